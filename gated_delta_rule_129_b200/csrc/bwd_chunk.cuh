// bwd_chunk.cuh -- gradients of the forward operator through the 64-token
// chunk form, fp32 on the CUDA cores (fp32 or bf16 inputs, dk and dv in
// {64, 128}).
//
// The pages train the operator chunk by chunk (page "Gated DeltaNet-2：将擦除与
// 写入分开", section "词元路径与并行训练") and note that its gradients flow
// through the already-gated keys and values; the per-token update is the one
// of section "在两个维度上独立控制".  Per (sequence, head) and chunk of n
// tokens with start state S0 and end state S1 the forward is (g the in-chunk
// cumulative log-decay, gamma = exp(g), g_n its last row):
//
//   E~ = b k gamma,  Z = w v,  A_ij = sum_c e_ic k_jc exp(g_ic - g_jc) (j < i),
//   P_ij likewise with q (j <= i),  T = (I + A)^-1,  W = T E~,  U~ = T Z,
//   U = U~ - W S0,  O = scale (Q~ S0 + P U),  S1 = diag(gamma_n) S0 + Kbar^T U
//
// with Q~ = q gamma and Kbar = k exp(g_n - g).  The backward runs in five
// steps, four launches (host: gdn2_chunk_bwd):
//   1. the CUDA-core prep recomputes every chunk's factors in fp32 (W, U~,
//      Kbar, Q_eff = Q~ - P W, gamma_n) and also stores T and P;
//   2. bwd_g_kernel forms G = scale Q_eff^T dO of every chunk (the outputs'
//      share of the state gradient, which does not depend on the state);
//   3. the CUDA-core walk recomputes the state at every chunk start (S0);
//   4. in other blocks of the same launch (bwd_walks_kernel: the two walks
//      are independent), the chunks are walked in reverse order: the gradient
//      reaching a chunk's start state is the transpose of the forward's
//      affine chunk map applied to the one reaching its end, plus G:
//      dS0 = gamma_n dS1 - W^T (Kbar dS1) + G
//      (dS1 of a sequence's last chunk is dhT; dh0 is dS0 of its first);
//   5. bwd_chunk_kernel then takes every (chunk, head) on its own, from S0,
//      dS1 and dO:
//        dQ~ = scale dO S0^T,  dP = scale dO U^T (j <= i),
//        dU = scale P^T dO + Kbar dS1,  dKbar = U dS1^T,  dW = -dU S0^T,
//        dT = dU Z^T + dW E~^T,  dZ = T^T dU,  dE~ = T^T dW,
//        dA = -T^T dT T^T (j < i),
//      then through the pairwise decays of A and P (per key channel c):
//        dE^D_ic = sum_j dA_ij k_jc D_ijc,  dQ^D_ic = sum_j dP_ij k_jc D_ijc,
//        dK^D_jc = sum_i (dA_ij e_ic + dP_ij q_ic) D_ijc,  D_ijc = exp(g_ic - g_jc),
//      and through the per-channel scales:
//        dq = dQ~ gamma + dQ^D,  dE = dE~ gamma + dE^D,  db = dE k,
//        dk = dKbar exp(g_n - g) + dK^D + dE b,  dv = dZ w,  dw = dZ v,
//        dg = dE~ E~ + dQ~ Q~ - dKbar Kbar + e dE^D + q dQ^D - k dK^D, and
//        the last row of dg also takes gamma_n rowsum(dS1 S0) + colsum(dKbar Kbar);
//        dlog_alpha is the reverse cumulative sum of dg over the chunk.
//      (The row and column sums of the decayed products reduce to the
//      elementwise terms above: sum_j of (dA_ij e_ic + dP_ij q_ic) k_jc D_ijc
//      is e dE^D + q dQ^D, and its sum over i is k dK^D.)
// Each token's gradients belong to one (chunk, head), so no output is summed
// across blocks.
#pragma once

#include "common.cuh"
#include "walk_simt.cuh"

namespace gdn2 {

// ------------------------------------------------ reverse state walk ----
constexpr int kBwdWalkThreads = 512;
constexpr int kBwdWalkCols = 32;   // value columns per CTA

struct BwdStateArgs {
  const float *W, *Kbar;          // fp32 factors [chunks, H, 64, DK]
  const float* gamma_last;        // [chunks, H, DK]
  const float* G;                 // [chunks, H, DK, DV]: scale Q_eff^T dO of each chunk
  SeqMap map;
  int H;
  const float* dhT;               // [N, H, DK, DV] or nullptr (zero)
  float* dS1;                     // out: [chunks, H, DK, DV], gradient at each chunk's end state
  float* X;                       // out: [chunks, H, 64, DV], Kbar dS1 of each chunk
  float* dh0;                     // out: [N, H, DK, DV]
  const int32_t* status;          // nonzero: malformed cu_seqlens (no chunks); dh0 = 0
};

// Shared memory, in bytes: two buffers of (Kbar with rows padded by 16 bytes,
// the G slice [DK][CS], gamma_n), one W tile, then dS [DK][CS] and
// X = Kbar dS [64][CS] in fp32.
template <int DK>
struct BwdDstateCfg {
  static constexpr int CS = kBwdWalkCols, LK = DK + 4;
  static constexpr int TILE = kChunk * LK * 4, GB = DK * CS * 4;
  static constexpr int OFF_KB = 0, OFF_G = TILE, OFF_GL = OFF_G + GB, BUF = OFF_GL + DK * 4;
  static constexpr int OFF_W = 2 * BUF, OFF_S = OFF_W + TILE, OFF_X = OFF_S + DK * CS * 4,
                       SMEM = OFF_X + kChunk * CS * 4;
  static_assert(SMEM <= 232448, "shared memory");
};

template <int DK>
constexpr size_t bwd_dstate_smem_bytes() {
  return (size_t)BwdDstateCfg<DK>::SMEM;
}

// The reverse walk of block `blk` (sequence, head, kBwdWalkCols value
// columns): the columns of dS evolve independently, since every step
// multiplies it from the left.  Kbar, the G slice and gamma_n (used first)
// are copied into one of two buffers a chunk ahead (in walk order), W (used
// last) into a single buffer as soon as the previous step has read it.
template <int DK, int DV>
__device__ __forceinline__ void bwd_dstate_cta(const BwdStateArgs& a, int blk, uint8_t* dsm) {
  using C = BwdDstateCfg<DK>;
  constexpr int CS = kBwdWalkCols, SL = DV / CS, LK = C::LK, NT = kBwdWalkThreads;
  const int H = a.H;
  const int sl = blk % SL;
  const int h = (blk / SL) % H;
  const int n = blk / (SL * H);
  const int j0 = sl * CS, tid = threadIdx.x;

  float* sdS = reinterpret_cast<float*>(dsm + C::OFF_S);   // [DK][CS]
  float* sX = reinterpret_cast<float*>(dsm + C::OFF_X);    // [64][CS]
  const float* sW = reinterpret_cast<const float*>(dsm + C::OFF_W);

  const size_t sbase = ((size_t)n * H + h) * DK * DV;
  const bool bad = *a.status != 0;
  for (int idx = tid; idx < DK * CS; idx += NT) {
    const int cc = idx / CS, j = idx % CS;
    sdS[idx] = (!bad && a.dhT) ? a.dhT[sbase + (size_t)cc * DV + j0 + j] : 0.f;
  }
  const int c_begin = a.map.chunk_off[n], c_end = a.map.chunk_off[n + 1];
  auto issue_b = [&](int c, int slot) {   // Kbar, the G slice, gamma_n of chunk c
    uint8_t* b = dsm + slot * C::BUF;
    const size_t ch = (size_t)c * H + h;
    stage_rows<DK * 4>(b + C::OFF_KB, LK * 4, a.Kbar + ch * kChunk * DK, DK * 4, kChunk, kChunk, tid, NT);
    stage_rows<CS * 4>(b + C::OFF_G, CS * 4, a.G + ch * DK * DV + j0, DV * 4, DK, DK, tid, NT);
    stage_rows<DK * 4>(b + C::OFF_GL, 0, a.gamma_last + ch * DK, 0, 1, 1, tid, NT);
  };
  auto issue_w = [&](int c) {   // W of chunk c
    stage_rows<DK * 4>(dsm + C::OFF_W, LK * 4, a.W + ((size_t)c * H + h) * kChunk * DK, DK * 4, kChunk, kChunk,
                       tid, NT);
  };
  // commit groups, oldest first: B(last), W(last), then per chunk c (in walk
  // order): B(c - 1) at its start and W(c - 1) at its end
  if (c_begin < c_end) issue_b(c_end - 1, 0);
  cp_async_commit();
  if (c_begin < c_end) issue_w(c_end - 1);
  cp_async_commit();

  constexpr int RS = DK / 32;                      // rows of dS per thread
  const int ri = tid / 16, cj = 2 * (tid % 16);    // X: rows 2 ri, 2 ri + 1; columns cj, cj + 1
  const int rs = RS * (tid / 16);                  // dS: rows rs .. rs + RS - 1; columns cj, cj + 1
  for (int c = c_end - 1, it = 0; c >= c_begin; --c, ++it) {
    if (c - 1 >= c_begin) issue_b(c - 1, (it + 1) & 1);
    cp_async_commit();
    cp_async_wait<2>();   // B(c) has landed
    __syncthreads();
    const uint8_t* b = dsm + (it & 1) * C::BUF;
    const float* sKb = reinterpret_cast<const float*>(b + C::OFF_KB);
    const float* sG = reinterpret_cast<const float*>(b + C::OFF_G);
    const float* sgl = reinterpret_cast<const float*>(b + C::OFF_GL);
    // the gradient reaching this chunk's end state
    const size_t cs = ((size_t)c * H + h) * DK * DV;
    for (int idx = tid; idx < DK * CS; idx += NT)
      a.dS1[cs + (size_t)(idx / CS) * DV + j0 + idx % CS] = sdS[idx];
    // X = Kbar dS1 on a 2 x 2 tile
    {
      float x[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll 2
      for (int c4 = 0; c4 < DK; c4 += 4) {   // four key rows of dS a step, Kbar read as vectors
        float kb[2][4];
#pragma unroll
        for (int r = 0; r < 2; ++r) load_vec<4>(sKb + (2 * ri + r) * LK + c4, kb[r]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 d = *reinterpret_cast<const float2*>(sdS + (c4 + e) * CS + cj);
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            x[r][0] = fmaf(kb[r][e], d.x, x[r][0]);
            x[r][1] = fmaf(kb[r][e], d.y, x[r][1]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        *reinterpret_cast<float2*>(sX + (2 * ri + r) * CS + cj) = make_float2(x[r][0], x[r][1]);
        *reinterpret_cast<float2*>(a.X + (((size_t)c * H + h) * kChunk + 2 * ri + r) * DV + j0 + cj) =
            make_float2(x[r][0], x[r][1]);
      }
    }
    cp_async_wait<1>();   // W(c) has landed
    __syncthreads();
    // dS0 = gamma_n dS1 - W^T X + G on an RS x 2 tile (rows of W and X past the
    // chunk's last token are zero); every thread rewrites only the entries of
    // dS it read
    {
      float s[RS][2];
#pragma unroll
      for (int r = 0; r < RS; ++r) {
        const float g = sgl[rs + r];
        const float2 gv = *reinterpret_cast<const float2*>(sG + (rs + r) * CS + cj);
        s[r][0] = fmaf(g, sdS[(rs + r) * CS + cj], gv.x);
        s[r][1] = fmaf(g, sdS[(rs + r) * CS + cj + 1], gv.y);
      }
#pragma unroll 4
      for (int i = 0; i < kChunk; ++i) {
        const float2 xv = *reinterpret_cast<const float2*>(sX + i * CS + cj);
        float wv[RS];
        load_vec<RS>(sW + i * LK + rs, wv);
#pragma unroll
        for (int r = 0; r < RS; ++r) {
          s[r][0] = fmaf(-wv[r], xv.x, s[r][0]);
          s[r][1] = fmaf(-wv[r], xv.y, s[r][1]);
        }
      }
#pragma unroll
      for (int r = 0; r < RS; ++r)
        *reinterpret_cast<float2*>(sdS + (rs + r) * CS + cj) = make_float2(s[r][0], s[r][1]);
    }
    __syncthreads();   // W and this chunk's buffer are free
    if (c - 1 >= c_begin) issue_w(c - 1);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();
  for (int idx = tid; idx < DK * CS; idx += NT) {
    const int cc = idx / CS, j = idx % CS;
    a.dh0[sbase + (size_t)cc * DV + j0 + j] = sdS[idx];
  }
}

// G = scale Q_eff^T dO of every (chunk, head): the outputs' share of the
// gradient reaching the chunk's start state, which does not depend on the
// state, so it is formed for all chunks at once before the reverse walk.
// grid (chunks, H); a thread holds 4 key rows x DK DV / 2048 value columns.
constexpr int kBwdGThreads = 512;

template <int DK, int DV, typename IO>
__global__ void __launch_bounds__(kBwdGThreads)
bwd_g_kernel(const float* __restrict__ Qeff, const void* dO_, SeqMap map, int H, float scale,
             float* __restrict__ G) {
  constexpr int RG = DK / 4, CG = kBwdGThreads / RG, CPT = DV / CG, LQ = DK + 4;
  static_assert(CPT == 2 || CPT == 4 || CPT == 8, "2, 4 or 8 value columns a thread");
  const int c = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  if (c >= map.chunk_off[map.N]) return;
  const ChunkPos pos = chunk_pos(map, c);
  const size_t ch = (size_t)c * H + h;
  extern __shared__ __align__(16) float gsm[];
  float* sQ = gsm;                                   // [64][LQ] Q_eff
  IO* sO = reinterpret_cast<IO*>(gsm + kChunk * LQ); // [64][DV] dO (rows past the end zero)
  const IO* dO = static_cast<const IO*>(dO_);
  stage_rows<DK * 4>(sQ, LQ * 4, Qeff + ch * kChunk * DK, DK * 4, kChunk, kChunk, tid, kBwdGThreads);
  stage_rows<DV * (int)sizeof(IO)>(sO, DV * sizeof(IO), dO + ((size_t)pos.t0 * H + h) * DV,
                                   (size_t)H * DV * sizeof(IO), kChunk, pos.len, tid, kBwdGThreads);
  cp_async_wait_all();
  __syncthreads();
  const int m0 = 4 * (tid / CG), j0 = CPT * (tid % CG);
  float2 acc[4][CPT / 2];   // columns j0 + 2 e2, j0 + 2 e2 + 1
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int e2 = 0; e2 < CPT / 2; ++e2) acc[r][e2] = make_float2(0.f, 0.f);
#pragma unroll 4
  for (int i = 0; i < kChunk; ++i) {
    float qv[4], ov[CPT];
    load_vec<4>(sQ + i * LQ + m0, qv);
#pragma unroll
    for (int e = 0; e < CPT; e += (CPT >= 4 ? 4 : 2)) {
      if constexpr (CPT >= 4) {
        float t4[4];
        load_vec<4>(sO + i * DV + j0 + e, t4);
#pragma unroll
        for (int u = 0; u < 4; ++u) ov[e + u] = t4[u];
      } else {
        float t2[2];
        load_vec<2>(sO + i * DV + j0 + e, t2);
        ov[e] = t2[0]; ov[e + 1] = t2[1];
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int e2 = 0; e2 < CPT / 2; ++e2)
        acc[r][e2] = fma2s(qv[r], make_float2(ov[2 * e2], ov[2 * e2 + 1]), acc[r][e2]);
  }
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int e2 = 0; e2 < CPT / 2; ++e2)
      *reinterpret_cast<float2*>(G + (ch * DK + m0 + r) * DV + j0 + 2 * e2) =
          make_float2(scale * acc[r][e2].x, scale * acc[r][e2].y);
}

template <int DK, int DV, typename IO>
constexpr size_t bwd_g_smem_bytes() {
  return sizeof(float) * (size_t)kChunk * (DK + 4) + (size_t)kChunk * DV * sizeof(IO);
}

// The two walks of the backward in one launch (they are independent): blocks
// [0, n_fwd) walk the chunks forward and store every chunk's start state,
// the others walk them in reverse for the state gradient.
template <int DK, int DV, typename IO>
__global__ void __launch_bounds__(kBwdWalkThreads)
bwd_walks_kernel(const WalkArgs<IO, float> wa, const BwdStateArgs ra, int n_fwd) {
  static_assert(kBwdWalkThreads == walk_simt_threads(kBwdWalkCols), "one block size for both walks");
  extern __shared__ __align__(16) uint8_t bsm[];
  if ((int)blockIdx.x < n_fwd) walk_simt_cta<DK, DV, IO, float, kBwdWalkCols>(wa, blockIdx.x, bsm);
  else bwd_dstate_cta<DK, DV>(ra, blockIdx.x - n_fwd, bsm);
}

// -------------------------------------------------- per-chunk gradients ----
constexpr int kBwdThreads = 512;
constexpr int kBwdVB = 64;            // value columns per pass of the value loop
constexpr float kBwdFoldNats = 60.f;  // decay range (each side of the reference row) for the product form

struct BwdChunkArgs {
  const void *q, *k, *v, *dO;     // io dtype, [T_total, H, d]
  const float *la, *b, *w;        // [T_total, H, d]
  const float *Tm, *Pm;           // [chunks, H, 64, 64]
  const float *S0, *dS1;          // [chunks, H, DK, DV]
  const float *U, *X;             // [chunks, H, 64, DV]: U = U~ - W S0 and Kbar dS1, from the two walks
  SeqMap map;
  int H;
  float scale;
  float *dq, *dk, *dla, *db;      // out: [T_total, H, DK]
  float *dv, *dw;                 // out: [T_total, H, DV]
};

// Shared-memory plan, in floats.  [64][DK] arrays have row stride LDK, 64 x 64
// ones and the transposed [d][64] ones LT, value tiles LVB: multiples of 4
// (float4 rows) that also spread a column's rows over the banks.
template <int DK, int DV, typename IO>
struct BwdCfg {
  static constexpr int LDK = DK + 4, LT = kChunk + 4, VB = kBwdVB, LVB = VB + 4;
  static constexpr int MAT = kChunk * LDK > DK * LT ? kChunk * LDK : DK * LT;   // one key-sized slot
  static constexpr int SQ = kChunk * LT;                                         // one pair-sized slot
  // T, and P (then dP), for the whole call
  static constexpr int OFF_T = 0, OFF_P = SQ, A0 = 2 * SQ;
  // the value loop: the pass's tiles (dO in io dtype)
  static constexpr int OFF_V = A0;
  static constexpr int OFF_S0T = OFF_V, OFF_D1T = OFF_S0T + VB * LDK, OFF_U = OFF_D1T + VB * LDK,
                       OFF_DU = OFF_U + kChunk * LVB, OFF_UT = OFF_DU + kChunk * LVB, OFF_ZT = OFF_UT + VB * LT,
                       OFF_DO = OFF_ZT + VB * LT,                                  // [64][VB] io
                       OFF_WS = OFF_DO + (kChunk * VB * (int)sizeof(IO) + 3) / 4,  // [64][VB] w (fp32)
                       OFF_VS = OFF_WS + kChunk * VB,                              // [64][VB] v (io)
                       END_V = OFF_VS + (kChunk * VB * (int)sizeof(IO) + 3) / 4;
  // after it, key-sized slots: g; k (k beta in the product form); q, then E~^T,
  // then T^T, then e alpha (product form) or q (pair by pair); dW, then dT /
  // dA and X; q alpha (product form) or e (pair by pair)
  static constexpr int S_G = A0, S_K = A0 + MAT, S_2 = A0 + 2 * MAT, S_3 = A0 + 3 * MAT, S_4 = A0 + 4 * MAT,
                       END_K = A0 + 5 * MAT;
  static constexpr int OFF_RED = (END_V > END_K ? END_V : END_K);   // [DK] x 2: rowsum(dS1 S0), colsum(dKbar Kbar)
  static constexpr int FLOATS = OFF_RED + 2 * DK + 4;
  static constexpr size_t SMEM = sizeof(float) * (size_t)FLOATS;
  // thread tiles: 64 x DK (4 columns, TMK rows), 64 x 64 (2 x 4), 64 x VB (2 x QN)
  static constexpr int CGK = DK / 4, TMK = kChunk * CGK / kBwdThreads, QN = VB / 16;
  static_assert(TMK * (kBwdThreads / CGK) == kChunk, "key tile");
  static_assert(kChunk * VB == 2 * QN * kBwdThreads && kChunk * kChunk == 8 * kBwdThreads, "value and pair tiles");
  static_assert(SMEM <= 232448, "shared memory");
};

template <typename IO>
__device__ __forceinline__ float ld_io(const void* p, size_t i) {
  return to_f32(static_cast<const IO*>(p)[i]);
}

template <int N>
__device__ __forceinline__ void unpack4(const float4 v, float (&o)[N], int at) {
  o[at] = v.x; o[at + 1] = v.y; o[at + 2] = v.z; o[at + 3] = v.w;
}

// Four consecutive values held as two packed pairs: element j, and the pairs
// of a float4.
__device__ __forceinline__ float pick4(const float2 (&v)[2], int j) {
  return (j & 2) ? ((j & 1) ? v[1].y : v[1].x) : ((j & 1) ? v[0].y : v[0].x);
}
__device__ __forceinline__ void pairs4(const float4 v, float2 (&o)[2]) {
  o[0] = make_float2(v.x, v.y);
  o[1] = make_float2(v.z, v.w);
}

template <int DK, int DV, typename IO>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_chunk_kernel(const BwdChunkArgs a) {
  using C = BwdCfg<DK, DV, IO>;
  constexpr int LDK = C::LDK, LT = C::LT, VB = C::VB, LVB = C::LVB, TMK = C::TMK, QN = C::QN;
  const int c = blockIdx.x, h = blockIdx.y;
  if (c >= a.map.chunk_off[a.map.N]) return;
  const int H = a.H, tid = threadIdx.x;
  const ChunkPos pos = chunk_pos(a.map, c);
  const int len = pos.len, t0 = pos.t0;
  const size_t ch = (size_t)c * H + h;
  const size_t tile_v = ch * kChunk * DV, tile_t = ch * kChunk * kChunk;
  const size_t st = ch * DK * DV;
  auto tok_k = [&](int i, int cc) { return ((size_t)(t0 + i) * H + h) * DK + cc; };
  auto tok_v = [&](int i, int j) { return ((size_t)(t0 + i) * H + h) * DV + j; };

  extern __shared__ __align__(16) float sm[];
  float* sT = sm + C::OFF_T;
  float* sP = sm + C::OFF_P;
  float* sgs = sm + C::OFF_RED;        // rowsum over v of dS1 * S0
  float* sdgn = sgs + DK;              // colsum over i of dKbar * Kbar

  // ------------------------------------------------ persistent tiles ----
  stage_rows<kChunk * 4>(sT, LT * 4, a.Tm + tile_t, kChunk * 4, kChunk, kChunk, tid, kBwdThreads);
  stage_rows<kChunk * 4>(sP, LT * 4, a.Pm + tile_t, kChunk * 4, kChunk, kChunk, tid, kBwdThreads);
  cp_async_commit();
  for (int i = tid; i < 2 * DK; i += kBwdThreads) sgs[i] = 0.f;

  // thread tiles
  const int rk0 = TMK * (tid / C::CGK), ck0 = 4 * (tid % C::CGK);   // 64 x DK
  const int rp0 = 2 * (tid / 16), cp0 = 4 * (tid % 16);             // 64 x 64
  const int rv = 2 * (tid / 16), cv = tid % 16;                     // 64 x VB: rows rv, rv + 1; columns cv + 16 q
  // accumulators of the four columns of a thread tile, as two packed pairs
  float2 accQ[TMK][2], accKb[TMK][2], accW[TMK][2], accP[2][2], accT[2][2];
#pragma unroll
  for (int ii = 0; ii < TMK; ++ii)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) accQ[ii][hh] = accKb[ii][hh] = accW[ii][hh] = make_float2(0.f, 0.f);
#pragma unroll
  for (int ii = 0; ii < 2; ++ii)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) accP[ii][hh] = accT[ii][hh] = make_float2(0.f, 0.f);

  // ---------------------------------------------------- value loop ----
  // per pass of VB value columns: U (from the forward walk) and
  // dU = scale P^T dO + Kbar dS1 (Kbar dS1 from the reverse walk), then dQ~,
  // dKbar, dW (key tiles), dP, dT (pair tiles) gather the pass's terms, and
  // dZ gives the pass's dv, dw.  (scale is applied to the sums of dO terms:
  // here for dU, when dQ~ and dP are used.)
  {
    float* sS0T = sm + C::OFF_S0T;   // [VB][LDK]
    float* sD1T = sm + C::OFF_D1T;   // [VB][LDK]
    float* sU = sm + C::OFF_U;       // [64][LVB], U
    float* sdU = sm + C::OFF_DU;     // [64][LVB], Kbar dS1 then dU
    float* sUT = sm + C::OFF_UT;     // [VB][LT]
    float* sZT = sm + C::OFF_ZT;     // [VB][LT]
    IO* sdO = reinterpret_cast<IO*>(sm + C::OFF_DO);   // [64][VB]
    float* sws = sm + C::OFF_WS;                          // [64][VB] w
    IO* svs = reinterpret_cast<IO*>(sm + C::OFF_VS);     // [64][VB] v
    for (int v0 = 0; v0 < DV; v0 += VB) {
      __syncthreads();  // the previous pass's readers are done
      stage_rows<VB * 4>(sU, LVB * 4, a.U + tile_v + v0, DV * 4, kChunk, kChunk, tid, kBwdThreads);
      stage_rows<VB * 4>(sdU, LVB * 4, a.X + tile_v + v0, DV * 4, kChunk, kChunk, tid, kBwdThreads);
      stage_rows<VB * (int)sizeof(IO)>(sdO, VB * sizeof(IO), static_cast<const IO*>(a.dO) + tok_v(0, v0),
                                       (size_t)H * DV * sizeof(IO), kChunk, len, tid, kBwdThreads);
      stage_rows<VB * 4>(sws, VB * 4, a.w + tok_v(0, v0), (size_t)H * DV * 4, kChunk, len, tid, kBwdThreads);
      stage_rows<VB * (int)sizeof(IO)>(svs, VB * sizeof(IO), static_cast<const IO*>(a.v) + tok_v(0, v0),
                                       (size_t)H * DV * sizeof(IO), kChunk, len, tid, kBwdThreads);
      cp_async_commit();
      // S0 and dS1 slices, transposed (two float4 of each a thread in flight at a time)
      constexpr int NS = DK * VB / 4 / kBwdThreads;
#pragma unroll
      for (int u0 = 0; u0 < NS; u0 += 2) {
        float4 s4[2], d4[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int idx = tid + (u0 + u) * kBwdThreads, cc = idx / (VB / 4), v4 = 4 * (idx % (VB / 4));
          s4[u] = *reinterpret_cast<const float4*>(a.S0 + st + (size_t)cc * DV + v0 + v4);
          d4[u] = *reinterpret_cast<const float4*>(a.dS1 + st + (size_t)cc * DV + v0 + v4);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int idx = tid + (u0 + u) * kBwdThreads, cc = idx / (VB / 4), v4 = 4 * (idx % (VB / 4));
          sS0T[(v4 + 0) * LDK + cc] = s4[u].x; sS0T[(v4 + 1) * LDK + cc] = s4[u].y;
          sS0T[(v4 + 2) * LDK + cc] = s4[u].z; sS0T[(v4 + 3) * LDK + cc] = s4[u].w;
          sD1T[(v4 + 0) * LDK + cc] = d4[u].x; sD1T[(v4 + 1) * LDK + cc] = d4[u].y;
          sD1T[(v4 + 2) * LDK + cc] = d4[u].z; sD1T[(v4 + 3) * LDK + cc] = d4[u].w;
        }
      }
      cp_async_wait<0>();
      __syncthreads();
      for (int idx = tid; idx < kChunk * VB; idx += kBwdThreads) {   // Z^T (rows past the end are zero)
        const int i = idx / VB, j = idx % VB;
        sZT[j * LT + i] = sws[idx] * to_f32(svs[idx]);
      }
      if (tid < DK) {
        float sacc = 0.f;
#pragma unroll 8
        for (int j = 0; j < VB; ++j) sacc = fmaf(sS0T[j * LDK + tid], sD1T[j * LDK + tid], sacc);
        sgs[tid] += sacc;
      }
      // dU = Kbar dS1 + scale P^T dO and U^T on 2 x QN tiles (rows rv, rv + 1;
      // columns cv + 16 q: a thread rewrites only the entries it reads)
      {
        float2 pd[QN];   // rows rv, rv + 1 of column cv + 16 q
#pragma unroll
        for (int q = 0; q < QN; ++q) pd[q] = make_float2(0.f, 0.f);
        for (int j = rv; j < kChunk; ++j) {   // P_{j, i} = 0 for j < i
          const float2 p = *reinterpret_cast<const float2*>(sP + j * LT + rv);
#pragma unroll
          for (int q = 0; q < QN; ++q) pd[q] = fma2s(to_f32(sdO[j * VB + cv + 16 * q]), p, pd[q]);
        }
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int q = 0; q < QN; ++q) {
            const int i = rv + r, j = cv + 16 * q;
            sUT[j * LT + i] = sU[i * LVB + j];
            sdU[i * LVB + j] = fmaf(a.scale, r ? pd[q].y : pd[q].x, sdU[i * LVB + j]);
          }
      }
      __syncthreads();
      // dQ~ += dO S0^T, dKbar += U dS1^T, dW += dU S0^T (negated later), four columns at a time
#pragma unroll 1
      for (int j4 = 0; j4 < VB; j4 += 4) {
        float2 sv[4][2], dv[4][2];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          pairs4(*reinterpret_cast<const float4*>(sS0T + (j4 + jj) * LDK + ck0), sv[jj]);
          pairs4(*reinterpret_cast<const float4*>(sD1T + (j4 + jj) * LDK + ck0), dv[jj]);
        }
#pragma unroll
        for (int ii = 0; ii < TMK; ++ii) {
          const int i = rk0 + ii;
          float o[4], uu[4], du[4];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) o[jj] = to_f32(sdO[i * VB + j4 + jj]);
          unpack4(*reinterpret_cast<const float4*>(sU + i * LVB + j4), uu, 0);
          unpack4(*reinterpret_cast<const float4*>(sdU + i * LVB + j4), du, 0);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              accQ[ii][hh] = fma2s(o[jj], sv[jj][hh], accQ[ii][hh]);
              accKb[ii][hh] = fma2s(uu[jj], dv[jj][hh], accKb[ii][hh]);
              accW[ii][hh] = fma2s(du[jj], sv[jj][hh], accW[ii][hh]);
            }
        }
      }
      // dP += dO U^T, dT += dU Z^T
#pragma unroll 1
      for (int j4 = 0; j4 < VB; j4 += 4) {
        float2 uv[4][2], zv[4][2];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          pairs4(*reinterpret_cast<const float4*>(sUT + (j4 + jj) * LT + cp0), uv[jj]);
          pairs4(*reinterpret_cast<const float4*>(sZT + (j4 + jj) * LT + cp0), zv[jj]);
        }
#pragma unroll
        for (int ii = 0; ii < 2; ++ii) {
          const int i = rp0 + ii;
          float o[4], du[4];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) o[jj] = to_f32(sdO[i * VB + j4 + jj]);
          unpack4(*reinterpret_cast<const float4*>(sdU + i * LVB + j4), du, 0);
#pragma unroll
          for (int jj = 0; jj < 4; ++jj)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              accP[ii][hh] = fma2s(o[jj], uv[jj][hh], accP[ii][hh]);
              accT[ii][hh] = fma2s(du[jj], zv[jj][hh], accT[ii][hh]);
            }
        }
      }
      // dZ = T^T dU on the 2 x QN tile, then dv = dZ w and dw = dZ v
      {
        float2 z[QN];   // rows rv, rv + 1 of column cv + 16 q
#pragma unroll
        for (int q = 0; q < QN; ++q) z[q] = make_float2(0.f, 0.f);
        for (int i = rv; i < kChunk; ++i) {   // T_{i, j} = 0 for i < j
          const float2 t = *reinterpret_cast<const float2*>(sT + i * LT + rv);
#pragma unroll
          for (int q = 0; q < QN; ++q) z[q] = fma2s(sdU[i * LVB + cv + 16 * q], t, z[q]);
        }
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int q = 0; q < QN; ++q)
            if (rv + r < len) {
              const int j = cv + 16 * q;
              const size_t o = tok_v(rv + r, v0 + j);
              const float zz = r ? z[q].y : z[q].x;
              a.dv[o] = zz * sws[(rv + r) * VB + j];
              a.dw[o] = zz * to_f32(svs[(rv + r) * VB + j]);
            }
      }
    }
  }
  __syncthreads();  // the value loop's tiles are dead

  // ------------------------------------- g, k, q; dq, dk and dg partials ----
  float* sg = sm + C::S_G;        // [64][LDK] cumulative log-decay
  float* sk = sm + C::S_K;        // [64][LDK] k
  float* sq = sm + C::S_2;        // [64][LDK] q
  float* sdP = sm + C::OFF_P;     // [64][LT], over P
  // the chunk's key-side rows: eight threads per token, DK / 8 channels each,
  // read as 16-byte vectors eight channels at a time (rows past the end zero)
  static_assert(kBwdThreads == 8 * kChunk, "eight threads per token row");
  const int ri8 = tid >> 3, ck8 = (tid & 7) * (DK / 8);
  auto row_pass = [&](auto&& body) {
#pragma unroll
    for (int c8 = ck8; c8 < ck8 + DK / 8; c8 += 8) body(ri8, c8, ri8 < len);
  };
  row_pass([&](int i, int c8, bool live) {
    float lv[8], kv[8], qv[8];
    if (live) {
      const size_t o = tok_k(i, c8);
      ldg_vec<8>(a.la + o, lv);
      ldg_vec<8>(static_cast<const IO*>(a.k) + o, kv);
      ldg_vec<8>(static_cast<const IO*>(a.q) + o, qv);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      sg[i * LDK + c8 + e] = live ? lv[e] : 0.f;
      sk[i * LDK + c8 + e] = live ? kv[e] : 0.f;
      sq[i * LDK + c8 + e] = live ? qv[e] : 0.f;
    }
  });
#pragma unroll
  for (int ii = 0; ii < 2; ++ii)
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
      sdP[(rp0 + ii) * LT + cp0 + jj] = cp0 + jj <= rp0 + ii ? a.scale * pick4(accP[ii], jj) : 0.f;
  __syncthreads();
  if (tid < DK) {   // in-chunk cumulative sum; padded rows keep g at its last value
    float acc = 0.f;
    for (int i = 0; i < kChunk; ++i) {
      acc += sg[i * LDK + tid];
      sg[i * LDK + tid] = acc;
    }
  }
  __syncthreads();
  float dg[TMK][4];
  {
    float colsum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int ii = 0; ii < TMK; ++ii) {
      const int i = rk0 + ii;
      float dqv[4], dkv[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int cc = ck0 + jj;
        const float g = sg[i * LDK + cc], gn = sg[(kChunk - 1) * LDK + cc];
        const float gam = expf(g), ks = expf(gn - g);
        const float dQt = a.scale * pick4(accQ[ii], jj), dKb = pick4(accKb[ii], jj);
        const float kb = sk[i * LDK + cc] * ks;   // Kbar
        dg[ii][jj] = dQt * sq[i * LDK + cc] * gam - dKb * kb;
        colsum[jj] = fmaf(dKb, kb, colsum[jj]);
        dqv[jj] = dQt * gam;
        dkv[jj] = dKb * ks;
      }
      if (i < len) {
        *reinterpret_cast<float4*>(a.dq + tok_k(i, ck0)) = make_float4(dqv[0], dqv[1], dqv[2], dqv[3]);
        *reinterpret_cast<float4*>(a.dk + tok_k(i, ck0)) = make_float4(dkv[0], dkv[1], dkv[2], dkv[3]);
      }
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) atomicAdd(sdgn + ck0 + jj, colsum[jj]);
  }
  __syncthreads();  // q is dead: its slot takes E~^T

  // ------------------------------ dT += dW E~^T, dE~ = T^T dW, dE~ terms ----
  {
    float* sEtT = sm + C::S_2;     // [DK][LT]
    float* sdW = sm + C::S_3;      // [64][LDK]
    row_pass([&](int i, int c8, bool live) {
      float bv[8];
      if (live) ldg_vec<8>(a.b + tok_k(i, c8), bv);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        sEtT[(c8 + e) * LT + i] = live ? bv[e] * sk[i * LDK + c8 + e] * expf(sg[i * LDK + c8 + e]) : 0.f;
    });
#pragma unroll
    for (int ii = 0; ii < TMK; ++ii)
      *reinterpret_cast<float4*>(sdW + (rk0 + ii) * LDK + ck0) =
          make_float4(-accW[ii][0].x, -accW[ii][0].y, -accW[ii][1].x, -accW[ii][1].y);
    __syncthreads();
#pragma unroll 4
    for (int cc = 0; cc < DK; ++cc) {
      float2 ev[2];
      pairs4(*reinterpret_cast<const float4*>(sEtT + cc * LT + cp0), ev);
#pragma unroll
      for (int ii = 0; ii < 2; ++ii) {
        const float wv = sdW[(rp0 + ii) * LDK + cc];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) accT[ii][hh] = fma2s(wv, ev[hh], accT[ii][hh]);
      }
    }
    float2 dEt[TMK][2];
#pragma unroll
    for (int ii = 0; ii < TMK; ++ii) dEt[ii][0] = dEt[ii][1] = make_float2(0.f, 0.f);
    for (int m = rk0; m < kChunk; ++m) {   // T_{m, i} = 0 for m < i
      float2 dv[2];
      pairs4(*reinterpret_cast<const float4*>(sdW + m * LDK + ck0), dv);
#pragma unroll
      for (int ii = 0; ii < TMK; ++ii) {
        const float t = sT[m * LT + rk0 + ii];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) dEt[ii][hh] = fma2s(t, dv[hh], dEt[ii][hh]);
      }
    }
#pragma unroll
    for (int ii = 0; ii < TMK; ++ii) {
      const int i = rk0 + ii;
      float dev[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int cc = ck0 + jj;
        dg[ii][jj] = fmaf(pick4(dEt[ii], jj), sEtT[cc * LT + i], dg[ii][jj]);
        dev[jj] = pick4(dEt[ii], jj) * expf(sg[i * LDK + cc]);
      }
      if (i < len) {   // dE so far (made db below) and dg so far
        *reinterpret_cast<float4*>(a.db + tok_k(i, ck0)) = make_float4(dev[0], dev[1], dev[2], dev[3]);
        *reinterpret_cast<float4*>(a.dla + tok_k(i, ck0)) = make_float4(dg[ii][0], dg[ii][1], dg[ii][2], dg[ii][3]);
      }
    }
  }
  __syncthreads();

  // ---------------------------------------------- dA = -T^T dT T^T ----
  float* sdA = sm + C::S_3;        // [64][LT] (first half of the slot)
  {
    float* sdT = sdA;              // dT, then dA over it
    float* sX = sm + C::S_3 + C::SQ;
    float* sTT = sm + C::S_2;      // [64][LT], T transposed
#pragma unroll
    for (int ii = 0; ii < 2; ++ii)
      *reinterpret_cast<float4*>(sdT + (rp0 + ii) * LT + cp0) =
          make_float4(accT[ii][0].x, accT[ii][0].y, accT[ii][1].x, accT[ii][1].y);
    for (int idx = tid; idx < kChunk * kChunk; idx += kBwdThreads) {
      const int i = idx / kChunk, j = idx % kChunk;
      sTT[j * LT + i] = sT[i * LT + j];
    }
    __syncthreads();
    float2 x[2][2];
#pragma unroll
    for (int ii = 0; ii < 2; ++ii) x[ii][0] = x[ii][1] = make_float2(0.f, 0.f);
#pragma unroll 4
    for (int m = 0; m < kChunk; ++m) {   // X = dT T^T
      float2 tv[2];
      pairs4(*reinterpret_cast<const float4*>(sTT + m * LT + cp0), tv);
#pragma unroll
      for (int ii = 0; ii < 2; ++ii) {
        const float d = sdT[(rp0 + ii) * LT + m];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) x[ii][hh] = fma2s(d, tv[hh], x[ii][hh]);
      }
    }
#pragma unroll
    for (int ii = 0; ii < 2; ++ii)
      *reinterpret_cast<float4*>(sX + (rp0 + ii) * LT + cp0) =
          make_float4(x[ii][0].x, x[ii][0].y, x[ii][1].x, x[ii][1].y);
    __syncthreads();
    float2 y[2][2];
#pragma unroll
    for (int ii = 0; ii < 2; ++ii) y[ii][0] = y[ii][1] = make_float2(0.f, 0.f);
#pragma unroll 4
    for (int m = 0; m < kChunk; ++m) {   // T^T X
      float2 xv[2];
      pairs4(*reinterpret_cast<const float4*>(sX + m * LT + cp0), xv);
#pragma unroll
      for (int ii = 0; ii < 2; ++ii) {
        const float t = sT[m * LT + rp0 + ii];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) y[ii][hh] = fma2s(t, xv[hh], y[ii][hh]);
      }
    }
#pragma unroll
    for (int ii = 0; ii < 2; ++ii)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
        sdA[(rp0 + ii) * LT + cp0 + jj] = cp0 + jj < rp0 + ii ? -pick4(y[ii], jj) : 0.f;   // strictly lower
  }
  // the chunk's decay range on each side of the reference row r (its middle
  // token, or its last one when shorter): the product form below scales rows
  // by exp(g_i - g_r) and exp(g_r - g_j), safe in fp32 while both ranges stay
  // within kBwdFoldNats
  const int rref = min(kChunk / 2, len - 1);
  __shared__ int s_steep;
  if (tid == 0) s_steep = 0;
  __syncthreads();
  if (tid < DK) {
    const float g0 = sg[tid], gr = sg[rref * LDK + tid], gl = sg[(kChunk - 1) * LDK + tid];
    if (g0 - gr > kBwdFoldNats || gr - gl > kBwdFoldNats) atomicOr(&s_steep, 1);
  }
  __syncthreads();

  if (!s_steep) {
    // -------------------- through the pairwise decays, as products ----
    // exp(g_ic - g_jc) = alpha_ic beta_jc with alpha = exp(g - g_r) and
    // beta = exp(g_r - g):  dE^D = alpha (dA (k beta)), dQ^D = alpha (dP (k beta)),
    // dK^D = beta (dA^T (e alpha) + dP^T (q alpha)).
    float* skb = sk;                  // k beta, over k
    float* sea = sm + C::S_2;         // e alpha
    float* sqa = sm + C::S_4;         // q alpha
    row_pass([&](int i, int c8, bool live) {
      float bv[8], qv[8];
      if (live) {
        ldg_vec<8>(a.b + tok_k(i, c8), bv);
        ldg_vec<8>(static_cast<const IO*>(a.q) + tok_k(i, c8), qv);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int cc = c8 + e;
        const float g = sg[i * LDK + cc], gr = sg[rref * LDK + cc], kv = sk[i * LDK + cc];
        const float al = expf(g - gr), be = expf(gr - g);
        sea[i * LDK + cc] = live ? bv[e] * kv * al : 0.f;
        sqa[i * LDK + cc] = live ? qv[e] * al : 0.f;
        skb[i * LDK + cc] = kv * be;
      }
    });
    __syncthreads();
    float2 ed[TMK][2], qd[TMK][2], kd[TMK][2];
#pragma unroll
    for (int ii = 0; ii < TMK; ++ii)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) ed[ii][hh] = qd[ii][hh] = kd[ii][hh] = make_float2(0.f, 0.f);
    for (int m = 0; m < rk0 + TMK; ++m) {   // dA, dP vanish for m > i
      float2 kbv[2];
      pairs4(*reinterpret_cast<const float4*>(skb + m * LDK + ck0), kbv);
#pragma unroll
      for (int ii = 0; ii < TMK; ++ii) {
        const float av = sdA[(rk0 + ii) * LT + m], pv = sdP[(rk0 + ii) * LT + m];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          ed[ii][hh] = fma2s(av, kbv[hh], ed[ii][hh]);
          qd[ii][hh] = fma2s(pv, kbv[hh], qd[ii][hh]);
        }
      }
    }
    for (int i = rk0; i < kChunk; ++i) {   // dA_{i, j}, dP_{i, j} vanish for i < j
      float2 ea[2], qa[2];
      float av[TMK], pv[TMK];
      pairs4(*reinterpret_cast<const float4*>(sea + i * LDK + ck0), ea);
      pairs4(*reinterpret_cast<const float4*>(sqa + i * LDK + ck0), qa);
#pragma unroll
      for (int ii = 0; ii < TMK; ++ii) {
        av[ii] = sdA[i * LT + rk0 + ii];
        pv[ii] = sdP[i * LT + rk0 + ii];
      }
#pragma unroll
      for (int ii = 0; ii < TMK; ++ii)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) kd[ii][hh] = fma2s(av[ii], ea[hh], fma2s(pv[ii], qa[hh], kd[ii][hh]));
    }
    // combine with the partials this thread wrote (same rows and columns)
#pragma unroll
    for (int ii = 0; ii < TMK; ++ii) {
      const int i = rk0 + ii;
      if (i >= len) continue;
      const size_t o = tok_k(i, ck0);
      float4 pq = *reinterpret_cast<const float4*>(a.dq + o), pe = *reinterpret_cast<const float4*>(a.db + o);
      float4 pk = *reinterpret_cast<const float4*>(a.dk + o), pg = *reinterpret_cast<const float4*>(a.dla + o);
      const float4 bv = *reinterpret_cast<const float4*>(a.b + o);
      float kv[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) kv[jj] = ld_io<IO>(a.k, o + jj);
      float fq[4], fe[4], fk[4], fg[4], bq[4];
      unpack4(pq, fq, 0); unpack4(pe, fe, 0); unpack4(pk, fk, 0); unpack4(pg, fg, 0); unpack4(bv, bq, 0);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int cc = ck0 + jj;
        const float g = sg[i * LDK + cc], gr = sg[rref * LDK + cc];
        const float al = expf(g - gr), be = expf(gr - g);
        const float edj = pick4(ed[ii], jj), qdj = pick4(qd[ii], jj), kdj = pick4(kd[ii], jj);
        const float edv = al * edj, qdv = al * qdj, kdv = be * kdj;
        const float dE = fe[jj] + edv;
        fq[jj] += qdv;
        fk[jj] += kdv + dE * bq[jj];
        // e dE^D + q dQ^D - k dK^D, each from the scaled operands
        fg[jj] += sea[i * LDK + cc] * edj + sqa[i * LDK + cc] * qdj - skb[i * LDK + cc] * kdj;
        fe[jj] = dE * kv[jj];
      }
      *reinterpret_cast<float4*>(a.dq + o) = make_float4(fq[0], fq[1], fq[2], fq[3]);
      *reinterpret_cast<float4*>(a.db + o) = make_float4(fe[0], fe[1], fe[2], fe[3]);
      *reinterpret_cast<float4*>(a.dk + o) = make_float4(fk[0], fk[1], fk[2], fk[3]);
      *reinterpret_cast<float4*>(a.dla + o) = make_float4(fg[0], fg[1], fg[2], fg[3]);
    }
  } else {
    // -------------- through the pairwise decays, pair by pair (steep) ----
    float* sq2 = sm + C::S_2;    // q again
    float* se = sm + C::S_4;     // e = b k
    row_pass([&](int i, int c8, bool live) {
      float bv[8], qv[8];
      if (live) {
        ldg_vec<8>(a.b + tok_k(i, c8), bv);
        ldg_vec<8>(static_cast<const IO*>(a.q) + tok_k(i, c8), qv);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        sq2[i * LDK + c8 + e] = live ? qv[e] : 0.f;
        se[i * LDK + c8 + e] = live ? bv[e] * sk[i * LDK + c8 + e] : 0.f;
      }
    });
    __syncthreads();
    // thread (channel cc, part p): the row sums of its channel over the
    // columns j of its part (j mod 2*PARTS in {p, 2*PARTS-1-p}: every part
    // gets as many pairs j <= i), summed over the parts by shuffles; the
    // column sums dK^D of those j stay in the thread
    constexpr int PARTS = kBwdThreads / DK, NJ = kChunk / PARTS, P2 = 2 * PARTS;
    const int cc = tid / PARTS, p = tid % PARTS;
    int jx[NJ];
    float kj[NJ], gj[NJ], dKD[NJ];
#pragma unroll
    for (int s = 0; s < NJ; ++s) {
      jx[s] = P2 * (s >> 1) + ((s & 1) ? (P2 - 1 - p) : p);
      kj[s] = sk[jx[s] * LDK + cc];
      gj[s] = sg[jx[s] * LDK + cc];
      dKD[s] = 0.f;
    }
    for (int i = 0; i < len; ++i) {
      const float ei = se[i * LDK + cc], qi = sq2[i * LDK + cc], gi = sg[i * LDK + cc];
      const int smax = 2 * (i / P2 + 1);   // slots whose j can be <= i (the same for the whole warp)
      float rE = 0.f, rQ = 0.f;
#pragma unroll
      for (int s = 0; s < NJ; ++s) {
        if (s < smax) {
          const int j = jx[s];
          // exp of a non-positive number where j <= i; dA and dP are zero elsewhere
          const float D = __expf(fminf(gi - gj[s], 0.f));
          const float av = sdA[i * LT + j] * D, pv = sdP[i * LT + j] * D;
          rE = fmaf(av, kj[s], rE);
          rQ = fmaf(pv, kj[s], rQ);
          dKD[s] = fmaf(av, ei, fmaf(pv, qi, dKD[s]));
        }
      }
#pragma unroll
      for (int o = 1; o < PARTS; o <<= 1) {
        rE += __shfl_xor_sync(0xffffffffu, rE, o);
        rQ += __shfl_xor_sync(0xffffffffu, rQ, o);
      }
      if (p == i % PARTS) {
        const size_t o = tok_k(i, cc);
        const float dE = a.db[o] + rE;
        a.dq[o] += rQ;
        a.db[o] = dE * sk[i * LDK + cc];
        a.dk[o] += dE * a.b[o];
        a.dla[o] += ei * rE + qi * rQ;
      }
    }
    __syncthreads();   // the row terms are in before the column terms touch the same rows
#pragma unroll
    for (int s = 0; s < NJ; ++s) {
      const int j = jx[s];
      if (j < len) {
        const size_t o = tok_k(j, cc);
        a.dk[o] += dKD[s];
        a.dla[o] -= kj[s] * dKD[s];
      }
    }
  }
  __syncthreads();
  // dlog_alpha: reverse cumulative sum of dg over the chunk; the last token
  // also carries the gradient of gamma_n.  PARTS adjacent lanes per channel,
  // each a run of 64 / PARTS rows: the run's values are loaded at once, summed
  // from the end, and offset by the totals of the runs after it (shuffles).
  {
    constexpr int PARTS = kBwdThreads / DK, R = kChunk / PARTS;
    const int cc = tid / PARTS, p = tid % PARTS, i0 = p * R;
    float v[R];
#pragma unroll
    for (int r = 0; r < R; ++r) v[r] = i0 + r < len ? a.dla[tok_k(i0 + r, cc)] : 0.f;
    float run = 0.f;
#pragma unroll
    for (int r = R - 1; r >= 0; --r) {
      run += v[r];
      v[r] = run;
    }
    float after = p == 0 ? expf(sg[(kChunk - 1) * LDK + cc]) * sgs[cc] + sdgn[cc] : 0.f;   // added to every row
    after = __shfl_sync(0xffffffffu, after, (tid & 31) - p);                             // the channel's first lane
#pragma unroll
    for (int d = 1; d < PARTS; ++d) {
      const float tot = __shfl_sync(0xffffffffu, run, ((tid & 31) + d) & 31);
      if (p + d < PARTS) after += tot;
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
      if (i0 + r < len) a.dla[tok_k(i0 + r, cc)] = v[r] + after;
  }
}

}  // namespace gdn2
