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
// with Q~ = q gamma and Kbar = k exp(g_n - g).  The backward runs in four
// launches (host: gdn2_chunk_bwd):
//   1. the CUDA-core prep recomputes every chunk's factors in fp32 (W, U~,
//      Kbar, Q_eff = Q~ - P W, gamma_n) and also stores T and P;
//   2. the CUDA-core walk recomputes the state at every chunk start (S0);
//   3. bwd_dstate_kernel walks the chunks in reverse order: the gradient
//      reaching a chunk's start state is the transpose of the forward's
//      affine chunk map applied to the one reaching its end, plus the
//      outputs' share:  dS0 = gamma_n dS1 - W^T (Kbar dS1) + scale Q_eff^T dO
//      (dS1 of a sequence's last chunk is dhT; dh0 is dS0 of its first);
//   4. bwd_chunk_kernel then takes every (chunk, head) on its own, from S0,
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

namespace gdn2 {

// ------------------------------------------------ reverse state walk ----
constexpr int kBwdWalkThreads = 256;
constexpr int kBwdWalkCols = 16;   // value columns per CTA

struct BwdStateArgs {
  const float *W, *Kbar, *Qeff;   // fp32 factors [chunks, H, 64, DK]
  const float* gamma_last;        // [chunks, H, DK]
  const void* dO;                 // [T_total, H, DV], io dtype
  SeqMap map;
  int H;
  float scale;
  const float* dhT;               // [N, H, DK, DV] or nullptr (zero)
  float* dS1;                     // out: [chunks, H, DK, DV], gradient at each chunk's end state
  float* dh0;                     // out: [N, H, DK, DV]
  const int32_t* status;          // nonzero: malformed cu_seqlens (no chunks); dh0 = 0
};

// Shared memory, in bytes: two chunk buffers (W, Kbar, Q_eff rows padded by
// 16 bytes, the dO slice, gamma_n), then dS [DK][CS] and X = Kbar dS [64][CS]
// in fp32.
template <int DK, typename IO>
struct BwdDstateCfg {
  static constexpr int CS = kBwdWalkCols, LK = DK + 4;
  static constexpr int TILE = kChunk * LK * 4, DOB = kChunk * CS * (int)sizeof(IO);
  static constexpr int OFF_W = 0, OFF_KB = TILE, OFF_QE = 2 * TILE, OFF_DO = 3 * TILE, OFF_GL = OFF_DO + DOB,
                       BUF = OFF_GL + DK * 4;
  static constexpr int OFF_S = 2 * BUF, OFF_X = OFF_S + DK * CS * 4, SMEM = OFF_X + kChunk * CS * 4;
  static_assert(SMEM <= 232448, "shared memory");
};

template <int DK>
constexpr size_t bwd_dstate_smem_bytes() {
  return (size_t)BwdDstateCfg<DK, float>::SMEM;   // bounds the bf16 plan
}

// One CTA per (sequence, head, kBwdWalkCols value columns): the columns of
// dS evolve independently, since every step multiplies it from the left.  The
// chunk's tiles are copied asynchronously into one of two buffers while the
// chunk after it (in walk order) is computed.
template <int DK, int DV, typename IO>
__global__ void __launch_bounds__(kBwdWalkThreads)
bwd_dstate_kernel(const BwdStateArgs a) {
  using C = BwdDstateCfg<DK, IO>;
  constexpr int CS = kBwdWalkCols, SL = DV / CS, LK = C::LK;
  const int H = a.H;
  const int sl = blockIdx.x % SL;
  const int h = (blockIdx.x / SL) % H;
  const int n = blockIdx.x / (SL * H);
  const int j0 = sl * CS, tid = threadIdx.x;

  extern __shared__ __align__(16) uint8_t dsm[];
  float* sdS = reinterpret_cast<float*>(dsm + C::OFF_S);   // [DK][CS]
  float* sX = reinterpret_cast<float*>(dsm + C::OFF_X);    // [64][CS]

  const IO* dO = static_cast<const IO*>(a.dO);
  const size_t sbase = ((size_t)n * H + h) * DK * DV;
  const bool bad = *a.status != 0;
  for (int idx = tid; idx < DK * CS; idx += kBwdWalkThreads) {
    const int cc = idx / CS, j = idx % CS;
    sdS[idx] = (!bad && a.dhT) ? a.dhT[sbase + (size_t)cc * DV + j0 + j] : 0.f;
  }
  const int c_begin = a.map.chunk_off[n], c_end = a.map.chunk_off[n + 1];
  const int s_begin = a.map.seq_begin(n), s_end = a.map.seq_end(n);
  auto issue = [&](int c, int slot) {
    uint8_t* b = dsm + slot * C::BUF;
    const size_t tk = ((size_t)c * H + h) * kChunk * DK;
    const int t0 = s_begin + (c - c_begin) * kChunk, len = min(kChunk, s_end - t0);
    stage_rows<DK * 4>(b + C::OFF_W, LK * 4, a.W + tk, DK * 4, kChunk, kChunk, tid, kBwdWalkThreads);
    stage_rows<DK * 4>(b + C::OFF_KB, LK * 4, a.Kbar + tk, DK * 4, kChunk, kChunk, tid, kBwdWalkThreads);
    stage_rows<DK * 4>(b + C::OFF_QE, LK * 4, a.Qeff + tk, DK * 4, kChunk, kChunk, tid, kBwdWalkThreads);
    stage_rows<CS * (int)sizeof(IO)>(b + C::OFF_DO, CS * sizeof(IO), dO + ((size_t)t0 * H + h) * DV + j0,
                                     (size_t)H * DV * sizeof(IO), kChunk, len, tid, kBwdWalkThreads);
    stage_rows<DK * 4>(b + C::OFF_GL, 0, a.gamma_last + ((size_t)c * H + h) * DK, 0, 1, 1, tid, kBwdWalkThreads);
  };
  if (c_begin < c_end) issue(c_end - 1, 0);
  cp_async_commit();

  constexpr int RS = DK / 32;                    // rows of dS per thread
  const int ri = tid / 8, cj = 2 * (tid % 8);    // X: rows 2 ri, 2 ri + 1; columns cj, cj + 1
  const int rs = RS * (tid / 8);                 // dS: rows rs .. rs + RS - 1; columns cj, cj + 1
  for (int c = c_end - 1, it = 0; c >= c_begin; --c, ++it) {
    if (c - 1 >= c_begin) issue(c - 1, (it + 1) & 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint8_t* b = dsm + (it & 1) * C::BUF;
    const float* sW = reinterpret_cast<const float*>(b + C::OFF_W);
    const float* sKb = reinterpret_cast<const float*>(b + C::OFF_KB);
    const float* sQe = reinterpret_cast<const float*>(b + C::OFF_QE);
    const IO* sdO = reinterpret_cast<const IO*>(b + C::OFF_DO);
    const float* sgl = reinterpret_cast<const float*>(b + C::OFF_GL);
    const int t0 = s_begin + (c - c_begin) * kChunk;
    const int len = min(kChunk, s_end - t0);
    // the gradient reaching this chunk's end state
    const size_t cs = ((size_t)c * H + h) * DK * DV;
    for (int idx = tid; idx < DK * CS; idx += kBwdWalkThreads)
      a.dS1[cs + (size_t)(idx / CS) * DV + j0 + idx % CS] = sdS[idx];
    // X = Kbar dS1 on a 2 x 2 tile
    {
      float x[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll 8
      for (int cc = 0; cc < DK; ++cc) {
        const float2 d = *reinterpret_cast<const float2*>(sdS + cc * CS + cj);
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const float kb = sKb[(2 * ri + r) * LK + cc];
          x[r][0] = fmaf(kb, d.x, x[r][0]);
          x[r][1] = fmaf(kb, d.y, x[r][1]);
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) *reinterpret_cast<float2*>(sX + (2 * ri + r) * CS + cj) = make_float2(x[r][0], x[r][1]);
    }
    __syncthreads();
    // dS0 = gamma_n dS1 - W^T X + Q_eff^T (scale dO) on an RS x 2 tile; every
    // thread rewrites only the entries of dS it read
    {
      float s[RS][2];
#pragma unroll
      for (int r = 0; r < RS; ++r) {
        const float g = sgl[rs + r];
        s[r][0] = g * sdS[(rs + r) * CS + cj];
        s[r][1] = g * sdS[(rs + r) * CS + cj + 1];
      }
#pragma unroll 4
      for (int i = 0; i < len; ++i) {
        const float2 xv = *reinterpret_cast<const float2*>(sX + i * CS + cj);
        const float o0 = a.scale * to_f32(sdO[i * CS + cj]), o1 = a.scale * to_f32(sdO[i * CS + cj + 1]);
#pragma unroll
        for (int r = 0; r < RS; ++r) {
          const float wv = sW[i * LK + rs + r], qv = sQe[i * LK + rs + r];
          s[r][0] = fmaf(qv, o0, fmaf(-wv, xv.x, s[r][0]));
          s[r][1] = fmaf(qv, o1, fmaf(-wv, xv.y, s[r][1]));
        }
      }
#pragma unroll
      for (int r = 0; r < RS; ++r)
        *reinterpret_cast<float2*>(sdS + (rs + r) * CS + cj) = make_float2(s[r][0], s[r][1]);
    }
    __syncthreads();   // this buffer is free for the chunk after next
  }
  cp_async_wait<0>();
  __syncthreads();
  for (int idx = tid; idx < DK * CS; idx += kBwdWalkThreads) {
    const int cc = idx / CS, j = idx % CS;
    a.dh0[sbase + (size_t)cc * DV + j0 + j] = sdS[idx];
  }
}

// -------------------------------------------------- per-chunk gradients ----
constexpr int kBwdThreads = 512;
constexpr int kBwdVB = 16;   // value columns per pass of the value loop

struct BwdChunkArgs {
  const void *q, *k, *v, *dO;     // io dtype, [T_total, H, d]
  const float *la, *b, *w;        // [T_total, H, d]
  const float *W, *Ut, *Kbar;     // fp32 factors [chunks, H, 64, d]
  const float *Tm, *Pm;           // [chunks, H, 64, 64]
  const float *S0, *dS1;          // [chunks, H, DK, DV]
  SeqMap map;
  int H;
  float scale;
  float *dq, *dk, *dla, *db;      // out: [T_total, H, DK]
  float *dv, *dw;                 // out: [T_total, H, DV]
};

// Shared-memory plan, in floats.  [64][DK] arrays have row stride LDK, 64 x 64
// ones and the transposed [d][64] ones LT, value tiles LVB; strides are
// multiples of 4 (float4 rows) and spread the rows over the banks.
template <int DK, int DV>
struct BwdCfg {
  static constexpr int LDK = DK + 4, LT = kChunk + 4, VB = kBwdVB, LVB = VB + 4;
  static constexpr int MAT = kChunk * LDK > DK * LT ? kChunk * LDK : DK * LT;   // one key-sized slot
  static constexpr int SQ = kChunk * LT;                                         // one pair-sized slot
  // the whole call: T and P
  static constexpr int OFF_T = 0, OFF_P = SQ, A0 = 2 * SQ;
  // the value loop
  static constexpr int OFF_W = A0, OFF_KB = A0 + kChunk * LDK, OFF_V = A0 + 2 * kChunk * LDK;
  static constexpr int OFF_S0 = OFF_V, OFF_S0T = OFF_S0 + DK * VB, OFF_D1 = OFF_S0T + VB * LDK,
                       OFF_D1T = OFF_D1 + DK * VB, OFF_DO = OFF_D1T + VB * LDK, OFF_U = OFF_DO + kChunk * LVB,
                       OFF_UT = OFF_U + kChunk * LVB, OFF_DU = OFF_UT + VB * LT, OFF_ZT = OFF_DU + kChunk * LVB,
                       END_V = OFF_ZT + VB * LT;
  // after it: g, k, then q / E~^T / q, dW / e, then dT / dA, X, dP
  static constexpr int OFF_G = A0, OFF_K = A0 + MAT, SLOT2 = A0 + 2 * MAT, SLOT3 = A0 + 3 * MAT,
                       OFF_DT = A0 + 4 * MAT, OFF_X = OFF_DT + SQ, OFF_DP = OFF_X + SQ, END_K = OFF_DP + SQ;
  static constexpr int OFF_RED = (END_V > END_K ? END_V : END_K);   // [DK] x 2: rowsum(dS1 S0), colsum(dKbar Kbar)
  static constexpr int FLOATS = OFF_RED + 2 * DK;
  static constexpr size_t SMEM = sizeof(float) * (size_t)FLOATS;
  // thread tiles: 64 x DK (4 columns, TMK rows), 64 x 64 (2 x 4), 64 x VB (1 x 2)
  static constexpr int CGK = DK / 4, TMK = kChunk * CGK / kBwdThreads;
  static_assert(TMK * (kBwdThreads / CGK) == kChunk, "key tile");
  static_assert(kChunk * VB == 2 * kBwdThreads && kChunk * kChunk == 8 * kBwdThreads, "value and pair tiles");
  static_assert(SMEM <= 232448, "shared memory");
};

template <typename IO>
__device__ __forceinline__ float ld_io(const void* p, size_t i) {
  return to_f32(static_cast<const IO*>(p)[i]);
}

template <int DK, int DV, typename IO>
__global__ void __launch_bounds__(kBwdThreads, 1)
bwd_chunk_kernel(const BwdChunkArgs a) {
  using C = BwdCfg<DK, DV>;
  constexpr int LDK = C::LDK, LT = C::LT, VB = C::VB, LVB = C::LVB, TMK = C::TMK;
  const int c = blockIdx.x, h = blockIdx.y;
  if (c >= a.map.chunk_off[a.map.N]) return;
  const int H = a.H, tid = threadIdx.x;
  const ChunkPos pos = chunk_pos(a.map, c);
  const int len = pos.len, t0 = pos.t0;
  const size_t ch = (size_t)c * H + h;
  const size_t tile_k = ch * kChunk * DK, tile_v = ch * kChunk * DV, tile_t = ch * kChunk * kChunk;
  const size_t st = ch * DK * DV;
  auto tok_k = [&](int i, int cc) { return ((size_t)(t0 + i) * H + h) * DK + cc; };
  auto tok_v = [&](int i, int j) { return ((size_t)(t0 + i) * H + h) * DV + j; };

  extern __shared__ __align__(16) float sm[];
  float* sT = sm + C::OFF_T;
  float* sP = sm + C::OFF_P;
  float* sgs = sm + C::OFF_RED;        // rowsum over v of dS1 * S0
  float* sdgn = sgs + DK;              // colsum over i of dKbar * Kbar

  // ------------------------------------------------ persistent tiles ----
  {
    float* sW = sm + C::OFF_W;
    float* sKb = sm + C::OFF_KB;
    for (int idx = tid; idx < kChunk * kChunk; idx += kBwdThreads) {
      const int i = idx / kChunk, j = idx % kChunk;
      sT[i * LT + j] = a.Tm[tile_t + idx];
      sP[i * LT + j] = a.Pm[tile_t + idx];
    }
    for (int idx = tid; idx < kChunk * DK / 4; idx += kBwdThreads) {
      const int i = idx / (DK / 4), c4 = 4 * (idx % (DK / 4));
      *reinterpret_cast<float4*>(sW + i * LDK + c4) = *reinterpret_cast<const float4*>(a.W + tile_k + i * DK + c4);
      *reinterpret_cast<float4*>(sKb + i * LDK + c4) = *reinterpret_cast<const float4*>(a.Kbar + tile_k + i * DK + c4);
    }
    for (int i = tid; i < 2 * DK; i += kBwdThreads) sgs[i] = 0.f;
  }

  // thread tiles
  const int rk0 = TMK * (tid / C::CGK), ck0 = 4 * (tid % C::CGK);   // 64 x DK
  const int rp0 = 2 * (tid / 16), cp0 = 4 * (tid % 16);             // 64 x 64
  const int rv = tid / 8, cv0 = 2 * (tid % 8);                      // 64 x VB
  float accQ[TMK][4], accKb[TMK][4], accW[TMK][4], accP[2][4], accT[2][4];
#pragma unroll
  for (int ii = 0; ii < TMK; ++ii)
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) accQ[ii][jj] = accKb[ii][jj] = accW[ii][jj] = 0.f;
#pragma unroll
  for (int ii = 0; ii < 2; ++ii)
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) accP[ii][jj] = accT[ii][jj] = 0.f;

  // ---------------------------------------------------- value loop ----
  {
    const float* sW = sm + C::OFF_W;
    const float* sKb = sm + C::OFF_KB;
    float* sS0 = sm + C::OFF_S0;     // [DK][VB]
    float* sS0T = sm + C::OFF_S0T;   // [VB][LDK]
    float* sD1 = sm + C::OFF_D1;     // [DK][VB]
    float* sD1T = sm + C::OFF_D1T;   // [VB][LDK]
    float* sdO = sm + C::OFF_DO;     // [64][LVB], scale * dO
    float* sU = sm + C::OFF_U;       // [64][LVB], U~ then U
    float* sUT = sm + C::OFF_UT;     // [VB][LT]
    float* sdU = sm + C::OFF_DU;     // [64][LVB]
    float* sZT = sm + C::OFF_ZT;     // [VB][LT]
    for (int v0 = 0; v0 < DV; v0 += VB) {
      __syncthreads();  // the previous pass's readers are done (and the persistent tiles written)
      for (int idx = tid; idx < DK * VB / 4; idx += kBwdThreads) {
        const int cc = idx / (VB / 4), v4 = 4 * (idx % (VB / 4));
        const float4 s = *reinterpret_cast<const float4*>(a.S0 + st + (size_t)cc * DV + v0 + v4);
        const float4 d = *reinterpret_cast<const float4*>(a.dS1 + st + (size_t)cc * DV + v0 + v4);
        *reinterpret_cast<float4*>(sS0 + cc * VB + v4) = s;
        *reinterpret_cast<float4*>(sD1 + cc * VB + v4) = d;
        sS0T[(v4 + 0) * LDK + cc] = s.x; sS0T[(v4 + 1) * LDK + cc] = s.y;
        sS0T[(v4 + 2) * LDK + cc] = s.z; sS0T[(v4 + 3) * LDK + cc] = s.w;
        sD1T[(v4 + 0) * LDK + cc] = d.x; sD1T[(v4 + 1) * LDK + cc] = d.y;
        sD1T[(v4 + 2) * LDK + cc] = d.z; sD1T[(v4 + 3) * LDK + cc] = d.w;
      }
      for (int idx = tid; idx < kChunk * VB; idx += kBwdThreads) {
        const int i = idx / VB, j = idx % VB;
        const bool live = i < len;
        sdO[i * LVB + j] = live ? a.scale * ld_io<IO>(a.dO, tok_v(i, v0 + j)) : 0.f;
        sZT[j * LT + i] = live ? a.w[tok_v(i, v0 + j)] * ld_io<IO>(a.v, tok_v(i, v0 + j)) : 0.f;
        sU[i * LVB + j] = a.Ut[tile_v + (size_t)i * DV + v0 + j];
      }
      __syncthreads();
      if (tid < DK) {
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < VB; ++j) s = fmaf(sS0[tid * VB + j], sD1[tid * VB + j], s);
        sgs[tid] += s;
      }
      // U = U~ - W S0 and dU = P^T (scale dO) + Kbar dS1, two columns of one row
      {
        float u0 = sU[rv * LVB + cv0], u1 = sU[rv * LVB + cv0 + 1], d0 = 0.f, d1 = 0.f;
#pragma unroll 4
        for (int cc = 0; cc < DK; ++cc) {
          const float wv = sW[rv * LDK + cc], kb = sKb[rv * LDK + cc];
          const float2 s = *reinterpret_cast<const float2*>(sS0 + cc * VB + cv0);
          const float2 d = *reinterpret_cast<const float2*>(sD1 + cc * VB + cv0);
          u0 = fmaf(-wv, s.x, u0); u1 = fmaf(-wv, s.y, u1);
          d0 = fmaf(kb, d.x, d0); d1 = fmaf(kb, d.y, d1);
        }
        for (int j = rv; j < kChunk; ++j) {   // P_{j, rv} = 0 for j < rv
          const float p = sP[j * LT + rv];
          const float2 o = *reinterpret_cast<const float2*>(sdO + j * LVB + cv0);
          d0 = fmaf(p, o.x, d0); d1 = fmaf(p, o.y, d1);
        }
        __syncthreads();   // every thread has read its U~ before any U is written
        sU[rv * LVB + cv0] = u0; sU[rv * LVB + cv0 + 1] = u1;
        sUT[cv0 * LT + rv] = u0; sUT[(cv0 + 1) * LT + rv] = u1;
        sdU[rv * LVB + cv0] = d0; sdU[rv * LVB + cv0 + 1] = d1;
      }
      __syncthreads();
      // dQ~ += (scale dO) S0^T, dKbar += U dS1^T, dW += dU S0^T (negated below)
#pragma unroll 4
      for (int j = 0; j < VB; ++j) {
        const float4 s = *reinterpret_cast<const float4*>(sS0T + j * LDK + ck0);
        const float4 d = *reinterpret_cast<const float4*>(sD1T + j * LDK + ck0);
        const float sv[4] = {s.x, s.y, s.z, s.w}, dv[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
        for (int ii = 0; ii < TMK; ++ii) {
          const float o = sdO[(rk0 + ii) * LVB + j], u = sU[(rk0 + ii) * LVB + j], du = sdU[(rk0 + ii) * LVB + j];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            accQ[ii][jj] = fmaf(o, sv[jj], accQ[ii][jj]);
            accKb[ii][jj] = fmaf(u, dv[jj], accKb[ii][jj]);
            accW[ii][jj] = fmaf(du, sv[jj], accW[ii][jj]);
          }
        }
      }
      // dP += (scale dO) U^T, dT += dU Z^T
#pragma unroll 4
      for (int j = 0; j < VB; ++j) {
        const float4 u = *reinterpret_cast<const float4*>(sUT + j * LT + cp0);
        const float4 z = *reinterpret_cast<const float4*>(sZT + j * LT + cp0);
        const float uv[4] = {u.x, u.y, u.z, u.w}, zv[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
        for (int ii = 0; ii < 2; ++ii) {
          const float o = sdO[(rp0 + ii) * LVB + j], du = sdU[(rp0 + ii) * LVB + j];
#pragma unroll
          for (int jj = 0; jj < 4; ++jj) {
            accP[ii][jj] = fmaf(o, uv[jj], accP[ii][jj]);
            accT[ii][jj] = fmaf(du, zv[jj], accT[ii][jj]);
          }
        }
      }
      // dZ = T^T dU (rows >= rv of column rv), then dv = dZ w and dw = dZ v
      {
        float z0 = 0.f, z1 = 0.f;
        for (int i = rv; i < kChunk; ++i) {
          const float t = sT[i * LT + rv];
          const float2 d = *reinterpret_cast<const float2*>(sdU + i * LVB + cv0);
          z0 = fmaf(t, d.x, z0); z1 = fmaf(t, d.y, z1);
        }
        if (rv < len) {
          const size_t o = tok_v(rv, v0 + cv0);
          a.dv[o] = z0 * a.w[o];
          a.dv[o + 1] = z1 * a.w[o + 1];
          a.dw[o] = z0 * ld_io<IO>(a.v, o);
          a.dw[o + 1] = z1 * ld_io<IO>(a.v, o + 1);
        }
      }
    }
  }
  __syncthreads();  // the value loop's tiles are dead

  // ------------------------------------- g, k, q; dq, dk and dg partials ----
  float* sg = sm + C::OFF_G;      // [64][LDK] cumulative log-decay
  float* sk = sm + C::OFF_K;      // [64][LDK] k
  float* sq = sm + C::SLOT2;      // [64][LDK] q
  float* sdP = sm + C::OFF_DP;    // [64][LT]
  for (int idx = tid; idx < kChunk * DK; idx += kBwdThreads) {
    const int i = idx / DK, cc = idx % DK;
    const bool live = i < len;
    sg[i * LDK + cc] = live ? a.la[tok_k(i, cc)] : 0.f;
    sk[i * LDK + cc] = live ? ld_io<IO>(a.k, tok_k(i, cc)) : 0.f;
    sq[i * LDK + cc] = live ? ld_io<IO>(a.q, tok_k(i, cc)) : 0.f;
  }
#pragma unroll
  for (int ii = 0; ii < 2; ++ii)
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
      sdP[(rp0 + ii) * LT + cp0 + jj] = cp0 + jj <= rp0 + ii ? accP[ii][jj] : 0.f;
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
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int cc = ck0 + jj;
        const float g = sg[i * LDK + cc], gn = sg[(kChunk - 1) * LDK + cc];
        const float gam = expf(g), ks = expf(gn - g);
        const float dQt = accQ[ii][jj], dKb = accKb[ii][jj];
        const float kb = sk[i * LDK + cc] * ks;   // Kbar
        dg[ii][jj] = dQt * sq[i * LDK + cc] * gam - dKb * kb;
        colsum[jj] = fmaf(dKb, kb, colsum[jj]);
        if (i < len) {
          a.dq[tok_k(i, cc)] = dQt * gam;
          a.dk[tok_k(i, cc)] = dKb * ks;
        }
      }
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) atomicAdd(sdgn + ck0 + jj, colsum[jj]);
  }
  __syncthreads();  // q is dead: its slot takes E~^T

  // ------------------------------ dT += dW E~^T, dE~ = T^T dW, dE~ terms ----
  {
    float* sEtT = sm + C::SLOT2;   // [DK][LT]
    float* sdW = sm + C::SLOT3;    // [64][LDK]
    for (int idx = tid; idx < kChunk * DK; idx += kBwdThreads) {
      const int i = idx / DK, cc = idx % DK;
      const float bv = i < len ? a.b[tok_k(i, cc)] : 0.f;
      sEtT[cc * LT + i] = bv * sk[i * LDK + cc] * expf(sg[i * LDK + cc]);
    }
#pragma unroll
    for (int ii = 0; ii < TMK; ++ii)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) sdW[(rk0 + ii) * LDK + ck0 + jj] = -accW[ii][jj];
    __syncthreads();
#pragma unroll 4
    for (int cc = 0; cc < DK; ++cc) {
      const float4 e = *reinterpret_cast<const float4*>(sEtT + cc * LT + cp0);
      const float ev[4] = {e.x, e.y, e.z, e.w};
#pragma unroll
      for (int ii = 0; ii < 2; ++ii) {
        const float wv = sdW[(rp0 + ii) * LDK + cc];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) accT[ii][jj] = fmaf(wv, ev[jj], accT[ii][jj]);
      }
    }
    float dEt[TMK][4];
#pragma unroll
    for (int ii = 0; ii < TMK; ++ii)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) dEt[ii][jj] = 0.f;
    for (int m = rk0; m < kChunk; ++m) {   // T_{m, i} = 0 for m < i
      const float4 d = *reinterpret_cast<const float4*>(sdW + m * LDK + ck0);
      const float dv[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
      for (int ii = 0; ii < TMK; ++ii) {
        const float t = sT[m * LT + rk0 + ii];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) dEt[ii][jj] = fmaf(t, dv[jj], dEt[ii][jj]);
      }
    }
#pragma unroll
    for (int ii = 0; ii < TMK; ++ii) {
      const int i = rk0 + ii;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int cc = ck0 + jj;
        dg[ii][jj] = fmaf(dEt[ii][jj], sEtT[cc * LT + i], dg[ii][jj]);
        if (i < len) {
          a.db[tok_k(i, cc)] = dEt[ii][jj] * expf(sg[i * LDK + cc]);   // dE so far; made db below
          a.dla[tok_k(i, cc)] = dg[ii][jj];                            // dg so far
        }
      }
    }
  }
  __syncthreads();

  // ---------------------------------------------- dA = -T^T dT T^T ----
  {
    float* sdT = sm + C::OFF_DT;   // [64][LT], then dA
    float* sX = sm + C::OFF_X;     // [64][LT]
    float* sTT = sm + C::SLOT3;    // [64][LT], T transposed
#pragma unroll
    for (int ii = 0; ii < 2; ++ii)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) sdT[(rp0 + ii) * LT + cp0 + jj] = accT[ii][jj];
    for (int idx = tid; idx < kChunk * kChunk; idx += kBwdThreads) {
      const int i = idx / kChunk, j = idx % kChunk;
      sTT[j * LT + i] = sT[i * LT + j];
    }
    __syncthreads();
    float x[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
    for (int m = 0; m < kChunk; ++m) {   // X = dT T^T
      const float4 t = *reinterpret_cast<const float4*>(sTT + m * LT + cp0);
      const float tv[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
      for (int ii = 0; ii < 2; ++ii) {
        const float d = sdT[(rp0 + ii) * LT + m];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) x[ii][jj] = fmaf(d, tv[jj], x[ii][jj]);
      }
    }
#pragma unroll
    for (int ii = 0; ii < 2; ++ii)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) sX[(rp0 + ii) * LT + cp0 + jj] = x[ii][jj];
    __syncthreads();
    float y[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
    for (int m = 0; m < kChunk; ++m) {   // T^T X
      const float4 xv4 = *reinterpret_cast<const float4*>(sX + m * LT + cp0);
      const float xv[4] = {xv4.x, xv4.y, xv4.z, xv4.w};
#pragma unroll
      for (int ii = 0; ii < 2; ++ii) {
        const float t = sT[m * LT + rp0 + ii];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) y[ii][jj] = fmaf(t, xv[jj], y[ii][jj]);
      }
    }
#pragma unroll
    for (int ii = 0; ii < 2; ++ii)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
        sdT[(rp0 + ii) * LT + cp0 + jj] = cp0 + jj < rp0 + ii ? -y[ii][jj] : 0.f;   // dA, strictly lower
  }
  __syncthreads();

  // ------------------------------- through the pairwise decays of A, P ----
  {
    const float* sdA = sm + C::OFF_DT;
    float* sq2 = sm + C::SLOT2;    // q again
    float* se = sm + C::SLOT3;     // e = b k
    for (int idx = tid; idx < kChunk * DK; idx += kBwdThreads) {
      const int i = idx / DK, cc = idx % DK;
      const bool live = i < len;
      sq2[i * LDK + cc] = live ? ld_io<IO>(a.q, tok_k(i, cc)) : 0.f;
      se[i * LDK + cc] = live ? a.b[tok_k(i, cc)] * sk[i * LDK + cc] : 0.f;
    }
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
  // also carries the gradient of gamma_n
  if (tid < DK && len > 0) {
    const float gn = sg[(kChunk - 1) * LDK + tid];
    float run = expf(gn) * sgs[tid] + sdgn[tid];
    for (int i = len - 1; i >= 0; --i) {
      const size_t o = tok_k(i, tid);
      run += a.dla[o];
      a.dla[o] = run;
    }
  }
}

}  // namespace gdn2
