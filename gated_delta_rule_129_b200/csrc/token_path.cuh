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
// Both kernels are bound by HBM traffic and written to issue few
// instructions per token: fp32 arithmetic, a row of d channels spread over a
// warp (prologue) or a half-warp (epilogue), a row's sum of squares by
// shuffles.  The prologue gives each block one head of one projection over a
// tile of tokens staged in shared memory by asynchronous copies (with the
// W - 1 rows before it); each warp then walks a run of the tile's tokens with
// the last W rows of its channels held in registers, so a token costs one
// shared-memory read and W fused multiply-adds per channel.  The epilogue
// gives each half-warp one (token, head) row, 16 bytes per lane for bf16.
#pragma once

#include "common.cuh"

namespace gdn2 {

constexpr int kTokThreads = 256;   // 8 warps
constexpr int kMaxConvWidth = 8;
constexpr float kTokEps = 1e-6f;

// PER consecutive elements of a row, loaded or stored as one or two vector
// accesses (the run starts at a multiple of its own size, up to 16 bytes).
template <int BYTES> struct VecT;
template <> struct VecT<4> { using T = uint32_t; };
template <> struct VecT<8> { using T = uint2; };
template <> struct VecT<16> { using T = uint4; };

template <typename IO, int PER>
struct Run {
  static constexpr int BYTES = PER * (int)sizeof(IO);
  static constexpr int NV = BYTES > 16 ? BYTES / 16 : 1;   // vector accesses
  using V = typename VecT<(BYTES > 16 ? 16 : BYTES)>::T;
  union U { V vec[NV]; IO e[PER]; };
  float v[PER];
  __device__ __forceinline__ void load(const IO* p) {
    U u;
#pragma unroll
    for (int j = 0; j < NV; ++j) u.vec[j] = reinterpret_cast<const V*>(p)[j];
#pragma unroll
    for (int i = 0; i < PER; ++i) v[i] = to_f32(u.e[i]);
  }
  __device__ __forceinline__ void store(IO* p) const {
    U u;
#pragma unroll
    for (int i = 0; i < PER; ++i) u.e[i] = from_f32<IO>(v[i]);
#pragma unroll
    for (int j = 0; j < NV; ++j) reinterpret_cast<V*>(p)[j] = u.vec[j];
  }
};

// Sigmoid with the hardware exponential and the fast divide: their relative
// errors, a few fp32 ulp, are far below what the bf16 outputs keep and below
// the fp32 path's tolerance.  Very negative x gives exp(-x) = inf and 0.
__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.f, 1.f + __expf(-x)); }
__device__ __forceinline__ float silu_f(float x) { return x * sigmoid_f(x); }

// sum over the 16 lanes of each half-warp
__device__ __forceinline__ float half_warp_sum(float v) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sequence bookkeeping of the prologue: the sequence that holds token t, as
// [start, next start).  Packed: the largest n with cu[n] <= t (empty
// sequences skipped); dense: rows of T.
__device__ __forceinline__ void seq_bounds(const int32_t* cu, int N, int T, int t, int& t0, int& t1) {
  if (!cu) {
    t0 = (t / T) * T;
    t1 = t0 + T;
    return;
  }
  int lo = 0, hi = N - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cu[mid] <= t) lo = mid; else hi = mid - 1;
  }
  t0 = cu[lo];
  t1 = cu[lo + 1];
}

// tokens per block in the prologue: 128 for bf16, 64 for fp32 rows (the
// same shared-memory footprint)
template <typename IO>
constexpr int tok_tile() { return 256 / (int)sizeof(IO); }

// One launch covers up to three projections of the same width d (grid z):
// q and k (L2-normalised) and v, or q and k alone, or v alone.
struct TokProArgs {
  const void* x[3];     // projections' outputs [T_total, H, d]
  const float* wt[3];   // taps [H * d, W]
  void* y[3];           // the operator's inputs [T_total, H, d]
  int l2[3];            // 1: L2-normalise the row
  const int32_t* cu;
  int N, T, T_total, H;
};

// rows of the tile and before it (as many bytes for bf16 and fp32)
constexpr int kTokSmem = (tok_tile<float>() + kMaxConvWidth - 1) * 128 * 4;

// grid: (token tiles, H, projections).  One block: one head of one projection
// over tok_tile<IO>() tokens; D channels, exactly W taps (tap i weighs token
// t - i; a tap that reaches before the token's sequence start reads zero).
template <typename IO, int D, int W>
__global__ void __launch_bounds__(kTokThreads)
token_prologue_kernel(const TokProArgs a) {
  constexpr int PER = D / 32;                                // channels per lane
  constexpr int ROWB = D * (int)sizeof(IO);                  // bytes of one row
  constexpr int TT = tok_tile<IO>();
  constexpr int PW = TT / (kTokThreads / 32);                // tokens per warp
  __shared__ __align__(16) uint8_t smem[kTokSmem];
  const int z = blockIdx.z, h = blockIdx.y, tb = blockIdx.x * TT;
  // (selects, not an index: a dynamic index would copy the arguments to local memory)
  const IO* __restrict__ x = static_cast<const IO*>(z == 0 ? a.x[0] : z == 1 ? a.x[1] : a.x[2]);
  const int r0 = tb - (W - 1);                               // first row held
  const int nrows = min(a.T_total, tb + TT) - r0;
  // stage rows [r0, r0 + nrows) of head h (rows before 0 left out), all in flight at once
  for (int i = threadIdx.x; i < nrows * (ROWB / 16); i += kTokThreads) {
    const int r = i / (ROWB / 16), u = i % (ROWB / 16);
    if (r0 + r >= 0)
      cp_async16(smem + r * ROWB + u * 16,
                 reinterpret_cast<const uint8_t*>(x + ((size_t)(r0 + r) * a.H + h) * D) + u * 16);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int c0 = lane * PER;
  // the lane's taps: PER * W consecutive floats of the [H * d, W] table
  float tap[W][PER];
  {
    const float* wp = (z == 0 ? a.wt[0] : z == 1 ? a.wt[1] : a.wt[2]) + ((size_t)h * D + c0) * W;
#pragma unroll
    for (int e = 0; e < PER; ++e)
#pragma unroll
      for (int i = 0; i < W; ++i) tap[i][e] = wp[e * W + i];
  }
  cp_async_wait_all();
  __syncthreads();
  const int ts = tb + warp * PW;                             // the warp's first token
  if (ts >= a.T_total) return;
  const bool l2 = (z == 0 ? a.l2[0] : z == 1 ? a.l2[1] : a.l2[2]) != 0;
  IO* __restrict__ y = static_cast<IO*>(z == 0 ? a.y[0] : z == 1 ? a.y[1] : a.y[2]);
  int t0, t1;
  seq_bounds(a.cu, a.N, a.T, ts, t0, t1);
  // win[i]: channels of row t - i for the current token t
  float win[W][PER];
#pragma unroll
  for (int i = 1; i < W; ++i) {
    if (ts - i >= t0) {
      Run<IO, PER> r;
      r.load(reinterpret_cast<const IO*>(smem + (ts - i - r0) * ROWB) + c0);
#pragma unroll
      for (int e = 0; e < PER; ++e) win[i][e] = r.v[e];
    } else {
#pragma unroll
      for (int e = 0; e < PER; ++e) win[i][e] = 0.f;
    }
  }
#pragma unroll 4
  for (int u = 0; u < PW; ++u) {
    const int t = ts + u;
    if (t >= a.T_total) break;
    if (t >= t1) {                                           // a sequence starts at t
      seq_bounds(a.cu, a.N, a.T, t, t0, t1);
#pragma unroll
      for (int i = 1; i < W; ++i)
#pragma unroll
        for (int e = 0; e < PER; ++e) win[i][e] = 0.f;
    }
    {
      Run<IO, PER> r;
      r.load(reinterpret_cast<const IO*>(smem + (t - r0) * ROWB) + c0);
#pragma unroll
      for (int e = 0; e < PER; ++e) win[0][e] = r.v[e];
    }
    Run<IO, PER> o;
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      float acc = tap[0][e] * win[0][e];
#pragma unroll
      for (int i = 1; i < W; ++i) acc = fmaf(tap[i][e], win[i][e], acc);
      o.v[e] = silu_f(acc);
      ss = fmaf(o.v[e], o.v[e], ss);
    }
    if (l2) {
      const float rn = rsqrtf(warp_sum(ss) + kTokEps);
#pragma unroll
      for (int e = 0; e < PER; ++e) o.v[e] *= rn;
    }
    o.store(y + ((size_t)t * a.H + h) * D + c0);
#pragma unroll
    for (int i = W - 1; i > 0; --i)
#pragma unroll
      for (int e = 0; e < PER; ++e) win[i][e] = win[i - 1][e];
  }
}

struct TokEpiArgs {
  const void *o, *g;
  const float* weight;   // [dv]
  long long rows;        // T_total * H
  void* out;
};

// grid: ceil(rows / (16 kEpiRows)); kEpiRows (token, head) rows of DV
// channels per half-warp, DV / 16 channels per lane.
constexpr int kEpiRows = 2;   // (token, head) rows per half-warp, loaded together

template <typename IO, int DV>
__global__ void __launch_bounds__(kTokThreads)
token_epilogue_kernel(const TokEpiArgs a) {
  constexpr int PER = DV / 16, HW = kTokThreads / 16;
  const int l16 = threadIdx.x & 15;
  const long long row0 = (long long)blockIdx.x * (HW * kEpiRows) + (threadIdx.x >> 4);
  Run<IO, PER> o[kEpiRows], g[kEpiRows];
#pragma unroll
  for (int u = 0; u < kEpiRows; ++u) {   // every load of the thread first
    const long long row = row0 + u * HW;
    const size_t base = (size_t)(row < a.rows ? row : 0) * DV + l16 * PER;   // shuffles below stay warp-wide
    o[u].load(static_cast<const IO*>(a.o) + base);
    g[u].load(static_cast<const IO*>(a.g) + base);
  }
  float wt[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) wt[e] = a.weight[l16 * PER + e];
#pragma unroll
  for (int u = 0; u < kEpiRows; ++u) {
    const long long row = row0 + u * HW;
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) ss = fmaf(o[u].v[e], o[u].v[e], ss);
    const float r = rsqrtf(half_warp_sum(ss) * (1.f / DV) + kTokEps);
#pragma unroll
    for (int e = 0; e < PER; ++e) o[u].v[e] = o[u].v[e] * r * wt[e] * sigmoid_f(g[u].v[e]);
    if (row < a.rows) o[u].store(static_cast<IO*>(a.out) + (size_t)row * DV + l16 * PER);
  }
}

}  // namespace gdn2
