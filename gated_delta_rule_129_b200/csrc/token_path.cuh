// token_path.cuh -- the token path around the operator: the prologue that
// turns the projections' outputs into the operator's q, k, v, and the
// epilogue that normalises and gates its output.
//
// Page "Gated DeltaNet-2：将擦除与写入分开", section "词元路径与并行训练": q
// and k go through a short causal convolution, SiLU and L2 normalisation, v
// through the convolution and SiLU; the operator's output goes through RMS
// normalisation and an output gate of its own (not the write gate).  The
// linear projections around it need trained weights and are the caller's.
// Readings where the pages are silent: the convolution is depthwise over the
// H*d channels of a projection, causal inside each sequence (tokens before a
// sequence's start count as zero), of width W <= 8; both norms use eps = 1e-6;
// the output gate is sigmoid(g), like the erase and write gates.
//
// Both kernels are bound by HBM traffic; each lane owns a run of d/32
// channels (8 or 4 bytes of a bf16 row), fp32 arithmetic, a head's sums of
// squares by warp shuffles.  The prologue gives each warp one head of one
// projection over 32 consecutive tokens and slides the convolution window
// along them in registers; the epilogue gives each warp one (token, head).
#pragma once

#include "common.cuh"

namespace gdn2 {

constexpr int kTokThreads = 256;   // 8 warps, 8 (token, head) pairs per block
constexpr int kMaxConvWidth = 8;
constexpr float kTokEps = 1e-6f;

// A lane's run of channels of one row, moved as one vector access (4, 8 or
// 16 bytes: the run starts at a multiple of its own size).
template <int BYTES> struct VecT;
template <> struct VecT<4> { using T = uint32_t; };
template <> struct VecT<8> { using T = uint2; };
template <> struct VecT<16> { using T = uint4; };

template <typename IO, int D>
struct Row {
  static constexpr int PER = D / 32;   // channels per lane
  using V = typename VecT<PER * (int)sizeof(IO)>::T;
  union U { V vec; IO e[PER]; };
  float v[PER];
  __device__ __forceinline__ void load(const IO* p) {
    U u;
    u.vec = *reinterpret_cast<const V*>(p);
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] = to_f32(u.e[i]);
  }
  __device__ __forceinline__ void store(IO* p) const {
    U u;
#pragma unroll
    for (int i = 0; i < PER; ++i) u.e[i] = from_f32<IO>(v[i]);
    *reinterpret_cast<V*>(p) = u.vec;
  }
};

__device__ __forceinline__ float silu_f(float x) { return x / (1.f + expf(-x)); }

// Sequence bookkeeping of the prologue: the sequence that holds token t, as
// [start, next start).  Packed: the largest n with cu[n] <= t (empty
// sequences skipped); dense: rows of T.
__device__ __forceinline__ void seq_bounds(const int32_t* cu, int N, int T, int t, int& n, int& t0, int& t1) {
  if (!cu) {
    n = t / T;
    t0 = n * T;
    t1 = t0 + T;
    return;
  }
  int lo = 0, hi = N - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  n = lo;
  t0 = cu[lo];
  t1 = cu[lo + 1];
}

constexpr int kTokRun = 32;   // tokens per warp in the prologue

struct TokProArgs {
  const void *q_raw, *k_raw, *v_raw;
  const float *wq, *wk, *wv;
  int W;
  const int32_t* cu;
  int N, T, T_total, H;
  void *q, *k, *v;
};

// One warp: one head of one projection over a run of kTokRun consecutive
// tokens.  Each lane keeps its channels' taps and the last W - 1 input rows
// in registers and slides along the run, so every input row is read from
// memory once (plus W - 1 rows before the run); a sequence start inside the
// run clears the window.
template <typename IO, int D>
__device__ __forceinline__ void conv_run(const IO* __restrict__ x, const float* __restrict__ wt, IO* __restrict__ y,
                                         const TokProArgs& a, int h, int tb, bool l2, int lane) {
  constexpr int PER = D / 32;
  constexpr int WM = kMaxConvWidth;
  const int c0 = lane * PER;
  const int W = a.W;
  float tap[WM][PER];
#pragma unroll
  for (int i = 0; i < WM; ++i)
#pragma unroll
    for (int e = 0; e < PER; ++e) tap[i][e] = i < W ? wt[((size_t)h * D + c0 + e) * W + i] : 0.f;
  const int te = min(a.T_total, tb + kTokRun);
  int n, t0, t1;
  seq_bounds(a.cu, a.N, a.T, tb, n, t0, t1);
  t0 = max(t0, 0);   // (a malformed cu_seqlens must not send a read before the row)
  // win[i] = x_{t-i} for i = 1 .. WM-1 (zero before the sequence's start)
  float win[WM][PER];
#pragma unroll
  for (int i = 1; i < WM; ++i) {
    Row<IO, D> r;
    if (i < W && tb - i >= t0) {
      r.load(x + ((size_t)(tb - i) * a.H + h) * D + c0);
    } else {
#pragma unroll
      for (int e = 0; e < PER; ++e) r.v[e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) win[i][e] = r.v[e];
  }
  for (int t = tb; t < te; ++t) {
    if (t >= t1) {
      // a new sequence starts here (skip empty ones): nothing before it counts
      seq_bounds(a.cu, a.N, a.T, t, n, t0, t1);
#pragma unroll
      for (int i = 1; i < WM; ++i)
#pragma unroll
        for (int e = 0; e < PER; ++e) win[i][e] = 0.f;
    }
    Row<IO, D> r;
    r.load(x + ((size_t)t * a.H + h) * D + c0);
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = tap[0][e] * r.v[e];
#pragma unroll
    for (int i = 1; i < WM; ++i)
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] = fmaf(tap[i][e], win[i][e], acc[e]);
#pragma unroll
    for (int i = WM - 1; i > 1; --i)
#pragma unroll
      for (int e = 0; e < PER; ++e) win[i][e] = win[i - 1][e];
#pragma unroll
    for (int e = 0; e < PER; ++e) win[1][e] = r.v[e];
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      acc[e] = silu_f(acc[e]);
      ss = fmaf(acc[e], acc[e], ss);
    }
    if (l2) {
      const float rn = rsqrtf(warp_sum(ss) + kTokEps);
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] *= rn;
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) r.v[e] = acc[e];
    r.store(y + ((size_t)t * a.H + h) * D + c0);
  }
}

// grid: (token runs / 8, H, 3 projections); block: 8 warps, one run each
template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(kTokThreads)
token_prologue_kernel(const TokProArgs a) {
  const int lane = threadIdx.x & 31;
  const long long run = (long long)blockIdx.x * (kTokThreads / 32) + (threadIdx.x >> 5);
  const long long tb = run * kTokRun;
  if (tb >= a.T_total) return;
  const int h = blockIdx.y;
  switch (blockIdx.z) {
    case 0:
      conv_run<IO, DK>(static_cast<const IO*>(a.q_raw), a.wq, static_cast<IO*>(a.q), a, h, (int)tb, true, lane);
      break;
    case 1:
      conv_run<IO, DK>(static_cast<const IO*>(a.k_raw), a.wk, static_cast<IO*>(a.k), a, h, (int)tb, true, lane);
      break;
    default:
      conv_run<IO, DV>(static_cast<const IO*>(a.v_raw), a.wv, static_cast<IO*>(a.v), a, h, (int)tb, false, lane);
      break;
  }
}

struct TokEpiArgs {
  const void *o, *g;
  const float* weight;   // [dv]
  int T_total, H;
  void* out;
};

template <typename IO, int DV>
__global__ void __launch_bounds__(kTokThreads)
token_epilogue_kernel(const TokEpiArgs a) {
  constexpr int PER = DV / 32;
  const int lane = threadIdx.x & 31;
  const long long pair = (long long)blockIdx.x * (kTokThreads / 32) + (threadIdx.x >> 5);
  if (pair >= (long long)a.T_total * a.H) return;
  const size_t base = (size_t)pair * DV + lane * PER;
  Row<IO, DV> o, g;
  o.load(static_cast<const IO*>(a.o) + base);
  g.load(static_cast<const IO*>(a.g) + base);
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) ss = fmaf(o.v[e], o.v[e], ss);
  const float r = rsqrtf(warp_sum(ss) * (1.f / DV) + kTokEps);
#pragma unroll
  for (int e = 0; e < PER; ++e) o.v[e] = o.v[e] * r * a.weight[lane * PER + e] / (1.f + expf(-g.v[e]));
  o.store(static_cast<IO*>(a.out) + base);
}

}  // namespace gdn2
