// prep_simt.cuh -- gate preparation + intra-chunk WY factors, fp32 on CUDA cores.
//
// One CTA per (chunk, head).  This is the fp32-I/O path (the 1e-4 accuracy
// mode) and the portable baseline of the bf16 path; the tensor-core kernel in
// prep_tc.cuh computes the same factors.
//
// Per chunk of n <= 64 tokens (page "Gated DeltaNet-2：将擦除与写入分开",
// sections "在两个维度上独立控制" and "词元路径与并行训练"; the algebra below is the
// recurrence unrolled over one chunk):
//   g_i    = cumulative sum of log_alpha over the chunk          (fp32)
//   e_i    = b_i * k_i,  z_i = w_i * v_i
//   A_ij   = sum_c e_ic k_jc exp(g_ic - g_jc),   j < i
//   P_ij   = sum_c q_ic k_jc exp(g_ic - g_jc),   j <= i
//   (I + A) W  = E~ = e * exp(g)       forward substitution, fp32
//   (I + A) U~ = Z                     same solve
//   Kbar_i = k_i * exp(g_n - g_i)
//   Q_eff  = q * exp(g) - P W,   O_part = P U~
// Every decay factor has a non-positive exponent, so none can overflow.
// Rows past the chunk's last token are written as zeros.
#pragma once

#include "common.cuh"

namespace gdn2 {

template <typename IO, typename FT>
struct PrepArgs {
  const IO* q;
  const IO* k;
  const IO* v;
  const float* la;
  const float* b;
  const float* w;
  SeqMap map;
  int H;
  FT* W;
  FT* Ut;
  FT* Kbar;
  FT* Qeff;
  FT* Opart;
  float* gamma_last;
  float* colscale;   // affine set: column scale of Mp and Q_eff (1 here: stored unscaled)
  FT* Mp;  // affine factor set only: Kbar^T W   [., H, DK, DK]
  FT* Nc;  // affine factor set only: Kbar^T U~  [., H, DK, DV]
  float* Tm;  // optional (the backward's recompute): T = (I + A)^-1  [., H, 64, 64]
  float* Pm;  // optional: P, zero above the diagonal                 [., H, 64, 64]
};

constexpr int kPrepSimtThreads = 512;

template <int DK, int DV>
constexpr size_t prep_simt_smem_bytes() {
  return sizeof(float) * (size_t)(4 * kChunk * (DK + 1) + kChunk * (DV + 1) + 2 * kChunk * (kChunk + 1));
}

// AFFINE selects the factor set: false stores W, U~, Kbar (WY set); true
// stores Mp = Kbar^T W and Nc = Kbar^T U~ (the chunk's affine state map).
// One (chunk c, head h) per call; all kPrepSimtThreads threads take part.
template <int DK, int DV, typename IO, typename FT, bool AFFINE>
__device__ __forceinline__ void prep_simt_chunk(const PrepArgs<IO, FT>& a, int c, int h, float* smem) {
  static_assert(2 * (DK + DV) <= kPrepSimtThreads, "two threads per solve column");
  constexpr int LK = DK + 1, LV = DV + 1, LA = kChunk + 1;
  const int H = a.H;
  const ChunkPos pos = chunk_pos(a.map, c);
  const int len = pos.len;

  float* sg = smem;                 // [64][LK]  cumulative log-decay
  float* sk = sg + kChunk * LK;     // [64][LK]  k
  float* se = sk + kChunk * LK;     // [64][LK]  e, then E~, then W
  float* sq = se + kChunk * LK;     // [64][LK]  q, then Q~
  float* sz = sq + kChunk * LK;     // [64][LV]  z, then U~
  float* sA = sz + kChunk * LV;     // [64][LA]  A (strictly lower)
  float* sP = sA + kChunk * LA;     // [64][LA]  P (lower, diagonal included)
  const int tid = threadIdx.x;

  batched_copy<8, float4>(
      kChunk * DK, tid, kPrepSimtThreads,
      [&](int idx) {
        const int i = idx / DK, cc = idx % DK;
        if (i >= len) return make_float4(0.f, 0.f, 0.f, 0.f);
        const size_t off = ((size_t)(pos.t0 + i) * H + h) * DK + cc;
        return make_float4(to_f32(a.k[off]), to_f32(a.q[off]), a.b[off], a.la[off]);
      },
      [&](int idx, float4 r) {
        const int i = idx / DK, cc = idx % DK;
        sk[i * LK + cc] = r.x;
        se[i * LK + cc] = r.z * r.x;
        sq[i * LK + cc] = r.y;
        sg[i * LK + cc] = r.w;
      });
  batched_copy<8, float>(
      kChunk * DV, tid, kPrepSimtThreads,
      [&](int idx) {
        const int i = idx / DV, cc = idx % DV;
        if (i >= len) return 0.f;
        const size_t off = ((size_t)(pos.t0 + i) * H + h) * DV + cc;
        return a.w[off] * to_f32(a.v[off]);
      },
      [&](int idx, float z) { sz[(idx / DV) * LV + idx % DV] = z; });
  for (int idx = tid; idx < kChunk * LA; idx += kPrepSimtThreads) {
    sA[idx] = 0.f;
    sP[idx] = 0.f;
  }
  __syncthreads();
  // In-chunk cumulative sum, one thread per key channel.  Padded rows carry
  // log_alpha = 0, so g stays at g_{n-1} past the last token.
  if (tid < DK) {
    float acc = 0.f;
    for (int i = 0; i < kChunk; ++i) {
      acc += sg[i * LK + tid];
      sg[i * LK + tid] = acc;
    }
  }
  __syncthreads();
  // A and P on 2 x 2 blocks of (i, j) pairs of the lower triangle, a thread
  // per block, the key channels summed in registers.  exp(g_i - g_j) is taken
  // of min(g_i - g_j, 0), so the entries above the diagonal (masked below)
  // cannot overflow; its hardware exponential's error, a few ulp, is far
  // below the fp32 path's tolerance.
  {
    constexpr int NB = kChunk / 2;
    for (int t = tid; t < NB * (NB + 1) / 2; t += kPrepSimtThreads) {
      int bi = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
      while (bi * (bi + 1) / 2 > t) --bi;
      while ((bi + 1) * (bi + 2) / 2 <= t) ++bi;
      const int bj = t - bi * (bi + 1) / 2;
      const int i0 = 2 * bi, j0 = 2 * bj;
      if (i0 >= len) continue;   // rows past the last token stay zero
      float aa[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, pp[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll 4
      for (int cc = 0; cc < DK; ++cc) {
        const float gi[2] = {sg[i0 * LK + cc], sg[(i0 + 1) * LK + cc]};
        const float gj[2] = {sg[j0 * LK + cc], sg[(j0 + 1) * LK + cc]};
        const float ev[2] = {se[i0 * LK + cc], se[(i0 + 1) * LK + cc]};
        const float qv[2] = {sq[i0 * LK + cc], sq[(i0 + 1) * LK + cc]};
        const float kv[2] = {sk[j0 * LK + cc], sk[(j0 + 1) * LK + cc]};
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const float kd = kv[q] * __expf(fminf(gi[r] - gj[q], 0.f));
            aa[r][q] = fmaf(ev[r], kd, aa[r][q]);
            pp[r][q] = fmaf(qv[r], kd, pp[r][q]);
          }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int i = i0 + r, j = j0 + q;
          if (i < len && j <= i) {
            if (j < i) sA[i * LA + j] = aa[r][q];
            sP[i * LA + j] = pp[r][q];
          }
        }
    }
  }
  __syncthreads();
  // Kbar (kept in sk, rows past the last token zero) and gamma_last; E~ and
  // Q~ are formed in place.
  const size_t tile_k = ((size_t)c * H + h) * kChunk * DK;
  const size_t tile_v = ((size_t)c * H + h) * kChunk * DV;
  for (int idx = tid; idx < kChunk * DK; idx += kPrepSimtThreads) {
    const int i = idx / DK, cc = idx % DK;
    const float gi = sg[i * LK + cc];
    const float kb = i < len ? sk[i * LK + cc] * expf(sg[(kChunk - 1) * LK + cc] - gi) : 0.f;
    if constexpr (!AFFINE) a.Kbar[tile_k + idx] = from_f32<FT>(kb);
    const float gam = expf(gi);
    se[i * LK + cc] *= gam;
    sq[i * LK + cc] *= gam;
  }
  // (sg is still read above by other threads; Kbar replaces k only after a barrier)
  __syncthreads();
  for (int idx = tid; idx < kChunk * DK; idx += kPrepSimtThreads) {
    const int i = idx / DK, cc = idx % DK;
    sk[i * LK + cc] = i < len ? sk[i * LK + cc] * expf(sg[(kChunk - 1) * LK + cc] - sg[i * LK + cc]) : 0.f;
  }
  if (tid < DK) a.gamma_last[((size_t)c * H + h) * DK + tid] = expf(sg[(kChunk - 1) * LK + tid]);
  if (AFFINE && a.colscale && tid < DK) a.colscale[((size_t)c * H + h) * DK + tid] = 1.f;
  __syncthreads();
  // half of sum_{m0 <= m < i} A_im X_m,col: the terms m = m0 + half, m0 + half + 2,
  // ... (two partial sums, short dependency chains); the other half comes
  // from the neighbouring lane
  const int scol = tid >> 1, half = tid & 1;
  auto row_dot_half = [&](const float* X, int ld, int col, int i, int m0) {
    float s0 = 0.f, s1 = 0.f;
    int m = m0 + half;
    for (; m + 2 < i; m += 4) {
      s0 = fmaf(sA[i * LA + m], X[m * ld + col], s0);
      s1 = fmaf(sA[i * LA + m + 2], X[(m + 2) * ld + col], s1);
    }
    for (; m < i; m += 2) s0 = fmaf(sA[i * LA + m], X[m * ld + col], s0);
    return s0 + s1;
  };
  // Forward substitution, row by row: W_i = E~_i - sum_{j<i} A_ij W_j, and the
  // same for U~ with Z.  Two threads per column of [W | U~].
  for (int i = 1; i < len; ++i) {
    float part = 0.f;
    if (scol < DK) part = row_dot_half(se, LK, scol, i, 0);
    else if (scol < DK + DV) part = row_dot_half(sz, LV, scol - DK, i, 0);
    part += __shfl_xor_sync(0xffffffffu, part, 1);
    if (half == 0) {
      if (scol < DK) se[i * LK + scol] -= part;
      else if (scol < DK + DV) sz[i * LV + scol - DK] -= part;
    }
    __syncthreads();
  }
  // Q_eff = Q~ - P W and O_part = P U~ (P is lower triangular with diagonal).
  for (int idx = tid; idx < kChunk * DK; idx += kPrepSimtThreads) {
    const int i = idx / DK, cc = idx % DK;
    float acc = sq[i * LK + cc];
    for (int j = 0; j <= i && j < len; ++j) acc = fmaf(-sP[i * LA + j], se[j * LK + cc], acc);
    a.Qeff[tile_k + idx] = from_f32<FT>(acc);
    if constexpr (!AFFINE) a.W[tile_k + idx] = from_f32<FT>(se[i * LK + cc]);
  }
  for (int idx = tid; idx < kChunk * DV; idx += kPrepSimtThreads) {
    const int i = idx / DV, cc = idx % DV;
    float acc = 0.f;
    for (int j = 0; j <= i && j < len; ++j) acc = fmaf(sP[i * LA + j], sz[j * LV + cc], acc);
    a.Opart[tile_v + idx] = from_f32<FT>(acc);
    if constexpr (!AFFINE) a.Ut[tile_v + idx] = from_f32<FT>(sz[i * LV + cc]);
  }
  if (a.Tm) {
    // T = (I + A)^-1 explicitly, for the backward: rows in order, each row's
    // entries from the rows above it (T_ij = -A_ij - sum_{j<m<i} A_im T_mj),
    // written over A once every thread has read the row (unit diagonal and
    // zero upper part implied).  A is no longer needed for the factors.
    __syncthreads();
    for (int i = 1; i < len; ++i) {
      float part = scol < i ? row_dot_half(sA, LA, scol, i, scol + 1) : 0.f;
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      const float val = scol < i ? -sA[i * LA + scol] - part : 0.f;
      __syncthreads();
      if (scol < i && half == 0) sA[i * LA + scol] = val;
      __syncthreads();
    }
    const size_t tile_t = ((size_t)c * H + h) * kChunk * kChunk;
    for (int idx = tid; idx < kChunk * kChunk; idx += kPrepSimtThreads) {
      const int i = idx / kChunk, j = idx % kChunk;
      a.Tm[tile_t + idx] = j < i ? sA[i * LA + j] : (i == j ? 1.f : 0.f);
      a.Pm[tile_t + idx] = j <= i ? sP[i * LA + j] : 0.f;
    }
  }
  if constexpr (AFFINE) {
    // The chunk's affine state map: S' = diag(gamma) S - Mp S + Nc with
    // Mp = Kbar^T W and Nc = Kbar^T U~ (sums over the chunk's tokens).
    const size_t mat_k = ((size_t)c * H + h) * DK * DK;
    const size_t mat_v = ((size_t)c * H + h) * DK * DV;
    for (int idx = tid; idx < DK * DK; idx += kPrepSimtThreads) {
      const int m = idx / DK, kk = idx % DK;
      float acc = 0.f;
      for (int i = 0; i < len; ++i) acc = fmaf(sk[i * LK + m], se[i * LK + kk], acc);
      a.Mp[mat_k + idx] = from_f32<FT>(acc);
    }
    for (int idx = tid; idx < DK * DV; idx += kPrepSimtThreads) {
      const int m = idx / DV, j = idx % DV;
      float acc = 0.f;
      for (int i = 0; i < len; ++i) acc = fmaf(sk[i * LK + m], sz[i * LV + j], acc);
      a.Nc[mat_v + idx] = from_f32<FT>(acc);
    }
  }
}

template <int DK, int DV, typename IO, typename FT, bool AFFINE>
__global__ void __launch_bounds__(kPrepSimtThreads)
prep_simt_kernel(const PrepArgs<IO, FT> a) {
  extern __shared__ float smem[];
  const int c = blockIdx.x, h = blockIdx.y;
  if (c >= a.map.chunk_off[a.map.N]) return;
  prep_simt_chunk<DK, DV, IO, FT, AFFINE>(a, c, h, smem);
}

// Exact fallback for the chunks the tensor-core prep hands back (decay too
// steep for its single in-chunk reference point): list[0] is the count,
// list[1 + i] = c * H + h.  A fixed grid strides over the list.
template <int DK, int DV, typename IO, typename FT>
__global__ void __launch_bounds__(kPrepSimtThreads)
prep_fixup_kernel(const PrepArgs<IO, FT> a, const int32_t* list) {
  extern __shared__ float smem[];
  const int count = list[0];
  for (int i = blockIdx.x; i < count; i += gridDim.x) {
    const int e = list[1 + i];
    prep_simt_chunk<DK, DV, IO, FT, true>(a, e / a.H, e % a.H, smem);
    __syncthreads();
  }
}

}  // namespace gdn2
