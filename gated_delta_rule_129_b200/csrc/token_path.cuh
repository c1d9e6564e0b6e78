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
// squares by warp shuffles.  The prologue gives each block one head of one
// projection over a 64-token tile staged in shared memory (with the W - 1
// rows before it); the epilogue gives each warp one (token, head).
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

// __expf (the hardware exponential): its relative error, a few fp32 ulp, is
// far below what the bf16 outputs keep and below the fp32 path's tolerance.
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + __expf(-x)); }
__device__ __forceinline__ float silu_f(float x) { return x * sigmoid_f(x); }

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

// tokens per block in the prologue: 128 for bf16, 64 for fp32 rows (the
// same shared-memory footprint)
template <typename IO>
constexpr int tok_tile() { return 256 / (int)sizeof(IO); }

struct TokProArgs {
  const void *q_raw, *k_raw, *v_raw;
  const float *wq, *wk, *wv;
  int W;
  const int32_t* cu;
  int N, T, T_total, H;
  void *q, *k, *v;
};

// One block: one head of one projection over a tile of tok_tile<IO>() tokens.
// The tile's rows, the W - 1 rows before it and the head's taps are first
// copied to shared memory by all threads (16-byte loads, many in flight);
// then each warp computes its tokens from there, a lane per d/32 channels.
// A tap that reaches before the token's sequence start reads zero.
// WM: the taps held in registers (4 for widths up to 4, else 8).
template <typename IO, int D, int WM>
__device__ __forceinline__ void conv_tile(const IO* __restrict__ x, const float* __restrict__ wt, IO* __restrict__ y,
                                          const TokProArgs& a, int h, int tb, bool l2, uint8_t* smem) {
  constexpr int PER = D / 32;
  constexpr int ROWB = D * (int)sizeof(IO);                  // bytes of one row
  constexpr int TT = tok_tile<IO>();
  const int W = a.W;
  const int r0 = tb - (W - 1);                               // first row held
  const int nrows = min(a.T_total, tb + TT) - r0;
  float* s_tap = reinterpret_cast<float*>(smem + (TT + kMaxConvWidth - 1) * ROWB);   // [D][W]
  for (int i = threadIdx.x; i < D * W; i += kTokThreads) s_tap[i] = wt[(size_t)h * D * W + i];
  // copy rows [r0, r0 + nrows) of head h (rows before 0 left out)
  for (int i = threadIdx.x; i < nrows * (ROWB / 16); i += kTokThreads) {
    const int r = i / (ROWB / 16), u = i % (ROWB / 16);
    if (r0 + r >= 0)
      reinterpret_cast<uint4*>(smem + r * ROWB)[u] =
          *reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(x + ((size_t)(r0 + r) * a.H + h) * D) + u * 16);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c0 = lane * PER;
  float tap[WM][PER];
#pragma unroll
  for (int i = 0; i < WM; ++i)
#pragma unroll
    for (int e = 0; e < PER; ++e) tap[i][e] = i < W ? s_tap[(c0 + e) * W + i] : 0.f;
  constexpr int PW = TT / (kTokThreads / 32);                // tokens per warp
  const int tw = tb + warp * PW;
  if (tw >= a.T_total) return;
  int n, t0, t1;
  seq_bounds(a.cu, a.N, a.T, tw, n, t0, t1);
  t0 = max(t0, 0);
  // (4 tokens at a time: enough independent work per warp, and a body small
  // enough for the instruction cache)
#pragma unroll 4
  for (int u = 0; u < PW; ++u) {
    const int t = tw + u;
    if (t >= a.T_total) break;
    if (t >= t1) {
      seq_bounds(a.cu, a.N, a.T, t, n, t0, t1);
      t0 = max(t0, 0);
    }
    float acc[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) acc[e] = 0.f;
#pragma unroll
    for (int i = 0; i < WM; ++i) {
      if (i < W && t - i >= t0) {
        Row<IO, D> r;
        r.load(reinterpret_cast<const IO*>(smem + (t - i - r0) * ROWB) + c0);
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = fmaf(tap[i][e], r.v[e], acc[e]);
      }
    }
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
    Row<IO, D> o;
#pragma unroll
    for (int e = 0; e < PER; ++e) o.v[e] = acc[e];
    o.store(y + ((size_t)t * a.H + h) * D + c0);
  }
}

// rows of the tile and before it (as many bytes for bf16 and fp32), then the taps
constexpr int kTokSmem = (tok_tile<float>() + kMaxConvWidth - 1) * 128 * 4 + 128 * kMaxConvWidth * 4;

// grid: (token tiles, H, 3 projections)
template <typename IO, int DK, int DV, int WM>
__global__ void __launch_bounds__(kTokThreads)
token_prologue_kernel(const TokProArgs a) {
  __shared__ __align__(16) uint8_t smem[kTokSmem];
  const int tb = blockIdx.x * tok_tile<IO>(), h = blockIdx.y;
  switch (blockIdx.z) {
    case 0:
      conv_tile<IO, DK, WM>(static_cast<const IO*>(a.q_raw), a.wq, static_cast<IO*>(a.q), a, h, tb, true, smem);
      break;
    case 1:
      conv_tile<IO, DK, WM>(static_cast<const IO*>(a.k_raw), a.wk, static_cast<IO*>(a.k), a, h, tb, true, smem);
      break;
    default:
      conv_tile<IO, DV, WM>(static_cast<const IO*>(a.v_raw), a.wv, static_cast<IO*>(a.v), a, h, tb, false, smem);
      break;
  }
}

struct TokEpiArgs {
  const void *o, *g;
  const float* weight;   // [dv]
  int T_total, H;
  void* out;
};

constexpr int kEpiPairs = 1;   // (token, head) pairs per warp in the epilogue

template <typename IO, int DV>
__global__ void __launch_bounds__(kTokThreads)
token_epilogue_kernel(const TokEpiArgs a) {
  constexpr int PER = DV / 32;
  const int lane = threadIdx.x & 31;
  const long long p0 = ((long long)blockIdx.x * (kTokThreads / 32) + (threadIdx.x >> 5)) * kEpiPairs;
  const long long np = (long long)a.T_total * a.H;
  float wt[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) wt[e] = a.weight[lane * PER + e];
  Row<IO, DV> o[kEpiPairs], g[kEpiPairs];
#pragma unroll
  for (int u = 0; u < kEpiPairs; ++u) {
    if (p0 + u < np) {
      const size_t base = (size_t)(p0 + u) * DV + lane * PER;
      o[u].load(static_cast<const IO*>(a.o) + base);
      g[u].load(static_cast<const IO*>(a.g) + base);
    }
  }
#pragma unroll
  for (int u = 0; u < kEpiPairs; ++u) {
    if (p0 + u >= np) break;
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) ss = fmaf(o[u].v[e], o[u].v[e], ss);
    const float r = rsqrtf(warp_sum(ss) * (1.f / DV) + kTokEps);
#pragma unroll
    for (int e = 0; e < PER; ++e) o[u].v[e] = o[u].v[e] * r * wt[e] * sigmoid_f(g[u].v[e]);
    o[u].store(static_cast<IO*>(a.out) + (size_t)(p0 + u) * DV + lane * PER);
  }
}

}  // namespace gdn2
