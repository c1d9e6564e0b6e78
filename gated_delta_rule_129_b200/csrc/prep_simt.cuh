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
constexpr float kPrepFoldNats = 60.f;   // decay range (each side of the middle row) for the product form of A, P

template <int DK, int DV>
constexpr size_t prep_simt_smem_bytes() {
  return sizeof(float) * (size_t)(4 * kChunk * (DK + 1) + kChunk * (DV + 1) + 3 * kChunk * (kChunk + 1));
}

// AFFINE selects the factor set: false stores W, U~, Kbar (WY set); true
// stores Mp = Kbar^T W and Nc = Kbar^T U~ (the chunk's affine state map).
// One (chunk c, head h) per call; all kPrepSimtThreads threads take part.
template <int DK, int DV, typename IO, typename FT, bool AFFINE>
__device__ __forceinline__ void prep_simt_chunk(const PrepArgs<IO, FT>& a, int c, int h, float* smem) {
  static_assert(kPrepSimtThreads == 512 && (DK + DV) % 32 == 0, "16 warps; [W | U~] in 32-column groups");
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
  float* sT = sP + kChunk * LA;     // [64][LA]  T = (I + A)^-1 (lower, unit diagonal)
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  // the chunk's rows: eight threads per token, DK / 8 key and DV / 8 value
  // channels each, read as 16-byte vectors (rows past the last token zero)
  {
    static_assert(kPrepSimtThreads == 8 * kChunk, "eight threads per token row");
    constexpr int CK = DK / 8, CV = DV / 8;
    const int i = tid >> 3, ck = (tid & 7) * CK, cv = (tid & 7) * CV;
    float kv[CK], qv[CK], bv[CK], lv[CK], wv[CV], vv[CV];
    if (i < len) {
      const size_t ok = ((size_t)(pos.t0 + i) * H + h) * DK + ck, ov = ((size_t)(pos.t0 + i) * H + h) * DV + cv;
      ldg_vec<CK>(a.k + ok, kv);
      ldg_vec<CK>(a.q + ok, qv);
      ldg_vec<CK>(a.b + ok, bv);
      ldg_vec<CK>(a.la + ok, lv);
      ldg_vec<CV>(a.w + ov, wv);
      ldg_vec<CV>(a.v + ov, vv);
    } else {
#pragma unroll
      for (int e = 0; e < CK; ++e) kv[e] = qv[e] = bv[e] = lv[e] = 0.f;
#pragma unroll
      for (int e = 0; e < CV; ++e) wv[e] = vv[e] = 0.f;
    }
#pragma unroll
    for (int e = 0; e < CK; ++e) {
      sk[i * LK + ck + e] = kv[e];
      se[i * LK + ck + e] = bv[e] * kv[e];
      sq[i * LK + ck + e] = qv[e];
      sg[i * LK + ck + e] = lv[e];
    }
#pragma unroll
    for (int e = 0; e < CV; ++e) sz[i * LV + cv + e] = wv[e] * vv[e];
  }
  for (int idx = tid; idx < kChunk * LA; idx += kPrepSimtThreads) {
    sA[idx] = 0.f;
    sP[idx] = 0.f;
    sT[idx] = 0.f;
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
  // A and P.  Where the chunk's decay stays within kPrepFoldNats on each side
  // of its middle row r, exp(g_ic - g_jc) = exp(g_ic - g_rc) exp(g_rc - g_jc)
  // (both factors in fp32 range), so with e, q scaled by the first and k by
  // the second, A and P are plain products over the key channels.  Otherwise
  // each pair takes its own exponential.
  __shared__ int s_steep;
  if (tid == 0) s_steep = 0;
  __syncthreads();
  const int rref = min(kChunk / 2, len - 1);
  if (tid < DK) {
    const float g0 = sg[tid], gr = sg[rref * LK + tid], gl = sg[(kChunk - 1) * LK + tid];
    if (g0 - gr > kPrepFoldNats || gr - gl > kPrepFoldNats) atomicOr(&s_steep, 1);
  }
  __syncthreads();
  const bool fold = s_steep == 0;
  if (fold) {
    for (int idx = tid; idx < kChunk * DK; idx += kPrepSimtThreads) {
      const int i = idx / DK, cc = idx % DK;
      const float d = sg[i * LK + cc] - sg[rref * LK + cc];
      const float al = expf(d), be = expf(-d);
      se[i * LK + cc] *= al;
      sq[i * LK + cc] *= al;
      sk[i * LK + cc] *= be;
    }
    __syncthreads();
    // a thread per 2 x 4 block of (i, j) pairs: rows 2 (t / 16) + {0, 1},
    // columns 4 (t % 16) + {0 .. 3}; blocks wholly above the diagonal idle
    const int i0 = 2 * (tid / 16), j0 = 4 * (tid % 16);
    if (j0 <= i0 + 1 && i0 < len) {
      float2 aa[2][2], pp[2][2];   // columns j0 + 2 h, j0 + 2 h + 1 of row i0 + r
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) aa[r][hh] = pp[r][hh] = make_float2(0.f, 0.f);
#pragma unroll 4
      for (int cc = 0; cc < DK; ++cc) {
        const float ev[2] = {se[i0 * LK + cc], se[(i0 + 1) * LK + cc]};
        const float qv[2] = {sq[i0 * LK + cc], sq[(i0 + 1) * LK + cc]};
        float2 kv[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh)
          kv[hh] = make_float2(sk[(j0 + 2 * hh) * LK + cc], sk[(j0 + 2 * hh + 1) * LK + cc]);
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            aa[r][hh] = fma2s(ev[r], kv[hh], aa[r][hh]);
            pp[r][hh] = fma2s(qv[r], kv[hh], pp[r][hh]);
          }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = i0 + r, j = j0 + q;
          const float av = (q & 1) ? aa[r][q >> 1].y : aa[r][q >> 1].x;
          const float pv = (q & 1) ? pp[r][q >> 1].y : pp[r][q >> 1].x;
          if (i < len && j <= i) {
            if (j < i) sA[i * LA + j] = av;
            sP[i * LA + j] = pv;
          }
        }
    }
  } else {
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
  }
  __syncthreads();
  // Kbar (kept in sk, rows past the last token zero) and gamma_last; E~ and
  // Q~ are formed in place.
  const size_t tile_k = ((size_t)c * H + h) * kChunk * DK;
  const size_t tile_v = ((size_t)c * H + h) * kChunk * DV;
  // (in the product form e, q and k are held scaled: e exp(g) = (e exp(g - g_r))
  // exp(g_r), and Kbar = k exp(g_n - g) = (k exp(g_r - g)) exp(g_n - g_r))
  for (int idx = tid; idx < kChunk * DK; idx += kPrepSimtThreads) {
    const int i = idx / DK, cc = idx % DK;
    const float gi = sg[i * LK + cc], gn = sg[(kChunk - 1) * LK + cc], gr = sg[rref * LK + cc];
    const float kb = i < len ? sk[i * LK + cc] * expf(fold ? gn - gr : gn - gi) : 0.f;
    if constexpr (!AFFINE) a.Kbar[tile_k + idx] = from_f32<FT>(kb);
    const float gam = expf(fold ? gr : gi);
    se[i * LK + cc] *= gam;
    sq[i * LK + cc] *= gam;
  }
  // (sg is still read above by other threads; Kbar replaces k only after a barrier)
  __syncthreads();
  for (int idx = tid; idx < kChunk * DK; idx += kPrepSimtThreads) {
    const int i = idx / DK, cc = idx % DK;
    const float gn = sg[(kChunk - 1) * LK + cc];
    sk[i * LK + cc] = i < len ? sk[i * LK + cc] * expf(fold ? gn - sg[rref * LK + cc] : gn - sg[i * LK + cc]) : 0.f;
  }
  if (tid < DK) a.gamma_last[((size_t)c * H + h) * DK + tid] = expf(sg[(kChunk - 1) * LK + tid]);
  if (AFFINE && a.colscale && tid < DK) a.colscale[((size_t)c * H + h) * DK + tid] = 1.f;
  __syncthreads();
  // T = (I + A)^-1 by blocks: the four 16 x 16 diagonal blocks by forward
  // substitution (warps 0-3, lane l < 16 owns column l), then the merges
  // 16 -> 32 and 32 -> 64, each T21 = -T22 (A21 T11).  sT starts all zero.
  if (warp < 4) {
    const int I = 16 * warp, l = lane;
    float t[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc = 0.f;
#pragma unroll
      for (int m = 0; m < i; ++m) acc = fmaf(sA[(I + i) * LA + I + m], t[m], acc);   // t[m] = 0 for m < l
      t[i] = i < l ? 0.f : (i == l ? 1.f : -acc);
    }
    if (l < 16)
#pragma unroll
      for (int i = 0; i < 16; ++i) sT[(I + i) * LA + I + l] = t[i];
  }
  __syncthreads();
  {
    // 16 -> 32: blocks (1, 0) and (3, 2); a thread per entry of X, then of T21
    const int m = tid >> 8, r = (tid >> 4) & 15, cc = tid & 15;
    const int ra = 32 * m + 16, ca = 32 * m;   // A21 / T21 at rows ra.., columns ca..; T11 at ca, T22 at ra
    float x = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) x = fmaf(sA[(ra + r) * LA + ca + k], sT[(ca + k) * LA + ca + cc], x);
    float* X = sA + (ra + r) * LA + ca + cc;   // A21 is not read again: X goes over it
    __syncthreads();
    *X = x;
    __syncthreads();
    float y = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) y = fmaf(sT[(ra + r) * LA + ra + k], sA[(ra + k) * LA + ca + cc], y);
    sT[(ra + r) * LA + ca + cc] = -y;
  }
  __syncthreads();
  {
    // 32 -> 64: rows 32.., columns 0..; two entries per thread
    const int r = tid >> 4, c2 = 2 * (tid & 15);
    float x0 = 0.f, x1 = 0.f;
    for (int k = 0; k < 32; ++k) {
      const float av = sA[(32 + r) * LA + k];
      x0 = fmaf(av, sT[k * LA + c2], x0);
      x1 = fmaf(av, sT[k * LA + c2 + 1], x1);
    }
    __syncthreads();
    sA[(32 + r) * LA + c2] = x0;       // X over A21
    sA[(32 + r) * LA + c2 + 1] = x1;
    __syncthreads();
    float y0 = 0.f, y1 = 0.f;
    for (int k = 0; k < 32; ++k) {
      const float tv = sT[(32 + r) * LA + 32 + k];
      y0 = fmaf(tv, sA[(32 + k) * LA + c2], y0);
      y1 = fmaf(tv, sA[(32 + k) * LA + c2 + 1], y1);
    }
    sT[(32 + r) * LA + c2] = -y0;
    sT[(32 + r) * LA + c2 + 1] = -y1;
  }
  __syncthreads();
  // [W | U~] = T [E~ | Z] and then Q_eff = Q~ - P W, O_part = P U~: warp w takes
  // rows 4w .. 4w + 3, lane l the columns l + 32 e of [W | U~] (T and P are
  // lower triangular, so the sums stop at the tile's last row)
  constexpr int NE = (DK + DV) / 32;
  auto colp = [&](float* base_k, float* base_v, int m, int e) -> float* {
    const int col = lane + 32 * e;
    return col < DK ? base_k + m * LK + col : base_v + m * LV + (col - DK);
  };
  static_assert(NE % 2 == 0, "column pairs");
  {
    float2 acc[4][NE / 2];   // columns e = 2 e2, 2 e2 + 1 of row 4 w + r
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int e2 = 0; e2 < NE / 2; ++e2) acc[r][e2] = make_float2(0.f, 0.f);
    for (int m = 0; m < 4 * warp + 4; ++m) {
      float tv[4];
      float2 xv[NE / 2];
#pragma unroll
      for (int r = 0; r < 4; ++r) tv[r] = sT[(4 * warp + r) * LA + m];
#pragma unroll
      for (int e2 = 0; e2 < NE / 2; ++e2) xv[e2] = make_float2(*colp(se, sz, m, 2 * e2), *colp(se, sz, m, 2 * e2 + 1));
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int e2 = 0; e2 < NE / 2; ++e2) acc[r][e2] = fma2s(tv[r], xv[e2], acc[r][e2]);
    }
    __syncthreads();   // every thread has read E~ and Z
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int e = 0; e < NE; ++e) *colp(se, sz, 4 * warp + r, e) = (e & 1) ? acc[r][e >> 1].y : acc[r][e >> 1].x;
  }
  __syncthreads();
  {
    float2 acc[4][NE / 2];   // columns e = 2 e2, 2 e2 + 1 of row 4 w + r
    auto q0 = [&](int r, int e) { return lane + 32 * e < DK ? sq[(4 * warp + r) * LK + lane + 32 * e] : 0.f; };
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int e2 = 0; e2 < NE / 2; ++e2) acc[r][e2] = make_float2(q0(r, 2 * e2), q0(r, 2 * e2 + 1));
    for (int m = 0; m < 4 * warp + 4; ++m) {
      float pv[4], xv[NE];
#pragma unroll
      for (int r = 0; r < 4; ++r) pv[r] = sP[(4 * warp + r) * LA + m];
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        xv[e] = *colp(se, sz, m, e);
        if (lane + 32 * e < DK) xv[e] = -xv[e];   // Q_eff takes -P W
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int e2 = 0; e2 < NE / 2; ++e2) acc[r][e2] = fma2s(pv[r], make_float2(xv[2 * e2], xv[2 * e2 + 1]), acc[r][e2]);
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = 4 * warp + r;
#pragma unroll
      for (int e = 0; e < NE; ++e) {
        const int col = lane + 32 * e;
        const float av = (e & 1) ? acc[r][e >> 1].y : acc[r][e >> 1].x;
        if (col < DK) {
          a.Qeff[tile_k + i * DK + col] = from_f32<FT>(av);
          if constexpr (!AFFINE) a.W[tile_k + i * DK + col] = from_f32<FT>(se[i * LK + col]);
        } else {
          a.Opart[tile_v + i * DV + col - DK] = from_f32<FT>(av);
          if constexpr (!AFFINE) a.Ut[tile_v + i * DV + col - DK] = from_f32<FT>(sz[i * LV + col - DK]);
        }
      }
    }
  }
  if (a.Tm) {
    // T and P for the backward (T with its unit diagonal, zero above it)
    const size_t tile_t = ((size_t)c * H + h) * kChunk * kChunk;
    for (int idx = tid; idx < kChunk * kChunk; idx += kPrepSimtThreads) {
      const int i = idx / kChunk, j = idx % kChunk;
      a.Tm[tile_t + idx] = sT[i * LA + j];
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
