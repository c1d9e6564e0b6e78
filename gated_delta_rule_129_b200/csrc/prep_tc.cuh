// prep_tc.cuh -- gate preparation + intra-chunk WY + the chunk's affine state
// map on the tensor cores (bf16 I/O, dk = 128, dv in {64, 128}).
//
// One CTA per (chunk, head); 8 compute warps + 1 producer warp (TMA loads and
// UMMA issue).  Per chunk of n <= 64 tokens (page "Gated DeltaNet-2：将擦除与写入分开",
// sections "在两个维度上独立控制" and "词元路径与并行训练"; the algebra is the
// recurrence unrolled over one chunk, written as products):
//
//  1. Gate prep (fp32).  The inputs stream in 32-channel slices through a
//     2-slot TMA ring; per slice: g = in-chunk cumulative sum of log_alpha,
//     and the bf16 operands, all with the decay folded in around one
//     reference token r = 32 of the chunk:
//        E^_i = b_i k_i exp(g_i - g_r),  Q^_i = q_i exp(g_i - g_r),
//        K^_j = k_j exp(g_r - g_j),      E~_i = b_i k_i exp(g_i),
//        Kbar_j = k_j exp(g_n - g_j),    Q~_i = q_i exp(g_i),  Z_i = w_i v_i.
//     For j <= i the product of the two factors is exp(g_i - g_j) <= 1; each
//     factor alone stays inside exp(+-80) as long as no 32-token stretch of a
//     channel decays by more than 80 nats.  A chunk that breaks this bound is
//     handed to the exact fp32 kernel (prep_fixup_kernel), pairwise per entry.
//  2. UMMA 1: [E^; Q^] . K^T  (M = 128, N = 64, K = 128) -> A (strictly lower
//     part of rows 0..63) and P (lower part with diagonal, rows 64..127).
//  3. T = (I + A)^-1 in fp32 on the CUDA cores (blocked forward substitution:
//     16 x 16 diagonal blocks, then the off-diagonal blocks by distance); T is
//     then split into bf16 hi + lo parts so the products keep ~16 bits of T.
//  4. UMMA 2: R = Kbar^T T (M = 128, N = 64, K = 64), V = P T (M = 64).
//  5. UMMA 3: Mp = R E~, Nc = R Z, P W = V E~, O_part = V Z, and the epilogue
//     writes Mp, Nc, Q_eff = Q~ - P W, O_part (bf16) and exp(g_n) (fp32).
// Rows past the chunk's last token are zero in every operand, so they add
// nothing; the padded rows of Q_eff and O_part come out as exact zeros.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc.cuh"

namespace gdn2 {

struct PrepTcArgs {
  CUtensorMap tm_q, tm_k, tm_v;    // bf16 [T_total, H, d], box {32 | dv/4, 1, 64}
  CUtensorMap tm_la, tm_b, tm_w;   // fp32 [T_total, H, d], box {32 | dv/4, 1, 64}
  SeqMap map;
  int H;
  __nv_bfloat16* Qeff;   // [max_chunks, H, 64, 128]
  __nv_bfloat16* Opart;  // [max_chunks, H, 64, DV]
  __nv_bfloat16* Mp;     // [max_chunks, H, 128, 128]
  __nv_bfloat16* Nc;     // [max_chunks, H, 128, DV]
  float* gamma_last;     // [max_chunks, H, 128]
  int32_t* fix_list;     // [0] = count, then c * H + h of handed-back chunks
  int* status;
};

template <int DV>
struct PrepTcCfg {
  static constexpr int DK = 128;
  static constexpr int KS = 32;             // key channels per slice
  static constexpr int VS = DV / 4;         // value channels per slice
  static constexpr int SLICES = 4;
  static constexpr int COMPUTE_WARPS = 8;
  static constexpr int THREADS = COMPUTE_WARPS * 32 + 32;
  // raw slot: la, b fp32 [64][32]; q, k bf16 [64][32]; v bf16 [64][VS]; w fp32 [64][VS]
  static constexpr int OFF_LA = 0, OFF_B = 8192, OFF_Q = 16384, OFF_K = 20480, OFF_V = 24576;
  static constexpr int OFF_W = OFF_V + kChunk * VS * 2;
  static constexpr int SLOT_BYTES = OFF_W + kChunk * VS * 4;
  static constexpr int SLOT_STRIDE = 36864;
  static constexpr int RING = 2 * SLOT_STRIDE;
  // operands (1024-aligned)
  static constexpr int OFF_X = RING;                 // [E^; Q^] K-major SW128, 2 panels x 128 rows
  static constexpr int OFF_KH = OFF_X + 32768;       // K^ K-major SW128, 2 panels x 64 rows
  static constexpr int OFF_ET = OFF_KH + 16384;      // E~ MN-major SW128 (rows = tokens), 2 panels
  static constexpr int OFF_Z = OFF_ET + 16384;       // Z  MN-major SW128, DV/64 panels
  static constexpr int OFF_KB = OFF_Z + 16384;       // Kbar^T MN-major SW128 A operand, 2 panels
  static constexpr int OFF_QT = OFF_KB + 16384;      // Q~ plain [64][128] bf16
  static constexpr int OFF_BAR = OFF_QT + 16384;
  // reuse of the ring after the slices: solve scratch and small operands
  static constexpr int LDA = 68;                     // fp32 row stride of A and T
  static constexpr int OFF_AS = 0, OFF_TS = 17408, OFF_PB = 35840, OFF_THI = 44032, OFF_TLO = 52224;
  static constexpr int OFF_XS = 60416;               // 3 x 16 x 16 fp32 block scratch
  // reuse of [E^; Q^] and K^ after UMMA 1
  static constexpr int OFF_RB = OFF_X, OFF_VB = OFF_X + 16384;
  static constexpr int SMEM = 1024 + OFF_BAR + 2048;  // barriers, flags, scan scratch
  static constexpr int TMEM_COLS = 512;
  static_assert(SLOT_BYTES <= SLOT_STRIDE, "slot fits");
  static_assert(OFF_XS + 3 * 256 * 4 <= RING, "solve scratch fits in the ring");
};

__device__ __forceinline__ void bar_compute() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// byte offset of the 16-byte unit holding elements [8u, 8u+8) of row `row`
// in an SW128 panel (rows of 64 bf16)
__device__ __forceinline__ uint32_t sw_unit(uint32_t row, uint32_t u) { return row * 128u + ((u ^ (row & 7u)) << 4); }

template <int DV>
__global__ void __launch_bounds__(PrepTcCfg<DV>::THREADS, 1)
prep_tc_kernel(const __grid_constant__ PrepTcArgs a) {
  using C = PrepTcCfg<DV>;
  constexpr int DK = C::DK;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);  // [2]
  uint64_t* empty = full + 2;                                       // [2]
  uint64_t* ops_ready = empty + 2;
  uint64_t* mma1_done = ops_ready + 1;
  uint64_t* t_ready = mma1_done + 1;
  uint64_t* mma2_done = t_ready + 1;
  uint64_t* rv_ready = mma2_done + 1;
  uint64_t* mma3_done = rv_ready + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(mma3_done + 1);
  int* s_flag = reinterpret_cast<int*>(tslot + 1);   // [0] hand back, [1] abort
  float* s_tot = reinterpret_cast<float*>(s_flag + 2);  // [8][32] segment totals
  float* s_er = s_tot + 256;                             // [32] exp(g_r)
  float* s_enr = s_er + 32;                              // [32] exp(g_n - g_r)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, h = blockIdx.y, H = a.H;
  if (c >= a.map.chunk_off[a.map.N]) return;  // uniform for the CTA
  const ChunkPos pos = chunk_pos(a.map, c);
  const int len = pos.len, t0 = pos.t0;

  if (tid == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], C::COMPUTE_WARPS);
    }
    tc::mbar_init(ops_ready, C::COMPUTE_WARPS);
    tc::mbar_init(mma1_done, 1);
    tc::mbar_init(t_ready, C::COMPUTE_WARPS);
    tc::mbar_init(mma2_done, 1);
    tc::mbar_init(rv_ready, C::COMPUTE_WARPS);
    tc::mbar_init(mma3_done, 1);
    s_flag[0] = 0;
    s_flag[1] = 0;
    tc::fence_mbar_init();
  }
  if (warp == C::COMPUTE_WARPS) {
    tc::tmem_alloc(tslot, C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tslot;
  volatile int* vflag = s_flag;

  if (warp == C::COMPUTE_WARPS) {
    // ------------------------------------------------- producer + UMMA issue --
    if (lane == 0) {
      auto load = [&](int s) {
        const int slot = s & 1;
        uint8_t* d = sm + slot * C::SLOT_STRIDE;
        tc::mbar_arrive_expect_tx(&full[slot], C::SLOT_BYTES);
        tc::tma_load_3d(d + C::OFF_LA, &a.tm_la, &full[slot], C::KS * s, h, t0);
        tc::tma_load_3d(d + C::OFF_B, &a.tm_b, &full[slot], C::KS * s, h, t0);
        tc::tma_load_3d(d + C::OFF_Q, &a.tm_q, &full[slot], C::KS * s, h, t0);
        tc::tma_load_3d(d + C::OFF_K, &a.tm_k, &full[slot], C::KS * s, h, t0);
        tc::tma_load_3d(d + C::OFF_V, &a.tm_v, &full[slot], C::VS * s, h, t0);
        tc::tma_load_3d(d + C::OFF_W, &a.tm_w, &full[slot], C::VS * s, h, t0);
      };
      bool ok = true;
      load(0);
      load(1);
      for (int s = 2; s < C::SLICES && ok; ++s) {
        ok = tc::mbar_wait(&empty[s & 1], ((s - 2) >> 1) & 1);
        if (ok) load(s);
      }
      const uint32_t X = tc::smem_u32(sm + C::OFF_X), KH = tc::smem_u32(sm + C::OFF_KH);
      const uint32_t ET = tc::smem_u32(sm + C::OFF_ET), ZZ = tc::smem_u32(sm + C::OFF_Z);
      const uint32_t KB = tc::smem_u32(sm + C::OFF_KB), PB = tc::smem_u32(sm + C::OFF_PB);
      const uint32_t THI = tc::smem_u32(sm + C::OFF_THI), TLO = tc::smem_u32(sm + C::OFF_TLO);
      const uint32_t RB = tc::smem_u32(sm + C::OFF_RB), VB = tc::smem_u32(sm + C::OFF_VB);
      const uint32_t SW = tc::kLayoutSW128;
      // UMMA 1: [E^; Q^] . K^T
      ok = ok && tc::mbar_wait(ops_ready, 0);
      if (ok && !vflag[0] && !vflag[1]) {
        tc::tc_fence_after();
        constexpr uint32_t id1 = tc::idesc_bf16(128, 64, false, false);
#pragma unroll
        for (int s = 0; s < DK / 16; ++s) {
          const uint32_t ko = (s >> 2), kk = (s & 3) * 32;
          tc::umma_f16(tbase, tc::sdesc(X + ko * 16384 + kk, 16, 1024, SW),
                       tc::sdesc(KH + ko * 8192 + kk, 16, 1024, SW), id1, s > 0);
        }
        tc::umma_commit(mma1_done);
        // UMMA 2: R = Kbar^T T (cols 64..127), V = P T (cols 128..191); T = hi + lo
        ok = tc::mbar_wait(t_ready, 0);
        if (ok) {
          tc::tc_fence_after();
          constexpr uint32_t idR = tc::idesc_bf16(128, 64, true, true);
          constexpr uint32_t idV = tc::idesc_bf16(64, 64, false, true);
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint32_t TT = part == 0 ? THI : TLO;
#pragma unroll
            for (int s = 0; s < 4; ++s) {
              tc::umma_f16(tbase + 64, tc::sdesc(KB + s * 2048, 8192, 1024, SW),
                           tc::sdesc(TT + s * 2048, 8192, 1024, SW), idR, part > 0 || s > 0);
              tc::umma_f16(tbase + 128, tc::sdesc(PB + s * 32, 16, 1024, SW),
                           tc::sdesc(TT + s * 2048, 8192, 1024, SW), idV, part > 0 || s > 0);
            }
          }
          tc::umma_commit(mma2_done);
        }
        // UMMA 3: Mp = R E~ (0..127), Nc = R Z (128..), P W = V E~ (256..), O_part = V Z (384..)
        ok = ok && tc::mbar_wait(rv_ready, 0);
        if (ok) {
          tc::tc_fence_after();
          constexpr uint32_t idM = tc::idesc_bf16(128, 128, false, true);
          constexpr uint32_t idN = tc::idesc_bf16(128, DV, false, true);
          constexpr uint32_t idQ = tc::idesc_bf16(64, 128, false, true);
          constexpr uint32_t idO = tc::idesc_bf16(64, DV, false, true);
#pragma unroll
          for (int s = 0; s < 4; ++s) {
            const uint64_t r_d = tc::sdesc(RB + s * 32, 16, 1024, SW);
            const uint64_t v_d = tc::sdesc(VB + s * 32, 16, 1024, SW);
            const uint64_t e_d = tc::sdesc(ET + s * 2048, 8192, 1024, SW);
            const uint64_t z_d = tc::sdesc(ZZ + s * 2048, 8192, 1024, SW);
            tc::umma_f16(tbase + 0, r_d, e_d, idM, s > 0);
            tc::umma_f16(tbase + 128, r_d, z_d, idN, s > 0);
            tc::umma_f16(tbase + 256, v_d, e_d, idQ, s > 0);
            tc::umma_f16(tbase + 384, v_d, z_d, idO, s > 0);
          }
          tc::umma_commit(mma3_done);
          tc::mbar_wait(mma3_done, 0);  // UMMAs done before TMEM is released
        }
      }
      if (!ok) {
        atomicExch(a.status, 8 /* GDN2_ERR_DEVICE_TIMEOUT */);
        vflag[1] = 1;
      }
      // every issued TMA load has landed before the CTA exits
      tc::mbar_wait(&full[0], 1);
      tc::mbar_wait(&full[1], 1);
    }
  } else {
    // ----------------------------------------------------------- compute --
    const int i_tok = tid >> 2, gq = tid & 3;     // build mapping: token, 8-channel group
    for (int s = 0; s < C::SLICES; ++s) {
      const int slot = s & 1;
      uint8_t* d = sm + slot * C::SLOT_STRIDE;
      float* la = reinterpret_cast<float*>(d + C::OFF_LA);   // becomes g
      if (!tc::mbar_wait(&full[slot], (s >> 1) & 1)) {
        atomicExch(a.status, 8);
        vflag[1] = 1;
        break;
      }
      // cumulative log-decay: lane = channel, warp = 8-token segment
      float loc[8];
      float acc = 0.f;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int tok = 8 * warp + t;
        acc += tok < len ? la[tok * 32 + lane] : 0.f;
        loc[t] = acc;
      }
      s_tot[warp * 32 + lane] = acc;
      bar_compute();
      float off = 0.f;
      for (int w2 = 0; w2 < warp; ++w2) off += s_tot[w2 * 32 + lane];
#pragma unroll
      for (int t = 0; t < 8; ++t) la[(8 * warp + t) * 32 + lane] = loc[t] + off;
      bar_compute();
      if (warp == 0) {
        const float g0 = la[lane], gr = la[32 * 32 + lane], gn = la[63 * 32 + lane];
        if (g0 - gr > 80.f || gr - gn > 80.f) atomicOr(s_flag, 1);
        s_er[lane] = __expf(gr);
        s_enr[lane] = __expf(gn - gr);
        a.gamma_last[((size_t)c * H + h) * DK + C::KS * s + lane] = expf(gn);
      }
      bar_compute();
      // operands for token i_tok, key channels cc0 .. cc0 + 7
      {
        const int i = i_tok, cl = 8 * gq, cc0 = C::KS * s + cl;
        const bool live = i < len;
        const float* gi = la + i * 32 + cl;
        const float* gr = la + 32 * 32 + cl;
        const float* bb = reinterpret_cast<const float*>(d + C::OFF_B) + i * 32 + cl;
        const uint4 kraw = *reinterpret_cast<const uint4*>(d + C::OFF_K + (i * 32 + cl) * 2);
        const uint4 qraw = *reinterpret_cast<const uint4*>(d + C::OFF_Q + (i * 32 + cl) * 2);
        const uint32_t kw[4] = {kraw.x, kraw.y, kraw.z, kraw.w};
        const uint32_t qw[4] = {qraw.x, qraw.y, qraw.z, qraw.w};
        uint32_t eh[4], qh[4], kh[4], et[4], kb[4], qt[4];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          float o_eh[2], o_qh[2], o_kh[2], o_et[2], o_kb[2], o_qt[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int m = 2 * p + e;
            const float kv = live ? (e ? bf16_hi_f(kw[p]) : bf16_lo_f(kw[p])) : 0.f;
            const float qv = live ? (e ? bf16_hi_f(qw[p]) : bf16_lo_f(qw[p])) : 0.f;
            const float bv = live ? bb[m] : 0.f;
            const float x = gi[m] - gr[m];
            const float E = __expf(x), F = __expf(-x);
            const float gam = s_er[cl + m] * E, kbf = s_enr[cl + m] * F;
            o_eh[e] = bv * kv * E;
            o_qh[e] = qv * E;
            o_kh[e] = kv * F;
            o_et[e] = bv * kv * gam;
            o_kb[e] = kv * kbf;
            o_qt[e] = qv * gam;
          }
          eh[p] = tc::pack_bf16(o_eh[0], o_eh[1]);
          qh[p] = tc::pack_bf16(o_qh[0], o_qh[1]);
          kh[p] = tc::pack_bf16(o_kh[0], o_kh[1]);
          et[p] = tc::pack_bf16(o_et[0], o_et[1]);
          kb[p] = tc::pack_bf16(o_kb[0], o_kb[1]);
          qt[p] = tc::pack_bf16(o_qt[0], o_qt[1]);
        }
        const uint32_t pnl = cc0 >> 6, u = (cc0 & 63) >> 3;
        *reinterpret_cast<uint4*>(sm + C::OFF_X + pnl * 16384 + sw_unit(i, u)) = make_uint4(eh[0], eh[1], eh[2], eh[3]);
        *reinterpret_cast<uint4*>(sm + C::OFF_X + pnl * 16384 + sw_unit(64 + i, u)) = make_uint4(qh[0], qh[1], qh[2], qh[3]);
        *reinterpret_cast<uint4*>(sm + C::OFF_KH + pnl * 8192 + sw_unit(i, u)) = make_uint4(kh[0], kh[1], kh[2], kh[3]);
        *reinterpret_cast<uint4*>(sm + C::OFF_ET + pnl * 8192 + sw_unit(i, u)) = make_uint4(et[0], et[1], et[2], et[3]);
        *reinterpret_cast<uint4*>(sm + C::OFF_KB + pnl * 8192 + sw_unit(i, u)) = make_uint4(kb[0], kb[1], kb[2], kb[3]);
        *reinterpret_cast<uint4*>(sm + C::OFF_QT + i * 256 + cc0 * 2) = make_uint4(qt[0], qt[1], qt[2], qt[3]);
        // Z = w * v for value channels vc0 .. vc0 + VS/4 - 1
        constexpr int VPT = C::VS / 4;
        const int vl = VPT * gq, vc0 = C::VS * s + vl;
        const float* ww = reinterpret_cast<const float*>(d + C::OFF_W) + i * C::VS + vl;
        const __nv_bfloat16* vv = reinterpret_cast<const __nv_bfloat16*>(d + C::OFF_V) + i * C::VS + vl;
        uint32_t zw[VPT / 2];
#pragma unroll
        for (int p = 0; p < VPT / 2; ++p) {
          const float z0 = live ? ww[2 * p] * __bfloat162float(vv[2 * p]) : 0.f;
          const float z1 = live ? ww[2 * p + 1] * __bfloat162float(vv[2 * p + 1]) : 0.f;
          zw[p] = tc::pack_bf16(z0, z1);
        }
        uint8_t* zdst = sm + C::OFF_Z + (vc0 >> 6) * 8192 + sw_unit(i, (vc0 & 63) >> 3) + (vc0 & 7) * 2;
        if constexpr (VPT == 8) *reinterpret_cast<uint4*>(zdst) = make_uint4(zw[0], zw[1], zw[2], zw[3]);
        else *reinterpret_cast<uint2*>(zdst) = make_uint2(zw[0], zw[1]);
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[slot]);
    }
    tc::fence_async_smem();
    tc::tc_fence_before();
    bar_compute();
    const bool skip = vflag[0] || vflag[1];
    if (skip && tid == 0 && !vflag[1]) {
      const int idx = atomicAdd(a.fix_list, 1);
      a.fix_list[1 + idx] = c * H + h;
    }
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(ops_ready);
    if (!skip) {
      const int q = warp & 3, half = warp >> 2;
      float* AS = reinterpret_cast<float*>(sm + C::OFF_AS);
      float* TS = reinterpret_cast<float*>(sm + C::OFF_TS);
      bool ok = tc::mbar_wait(mma1_done, 0);
      if (ok) {
        // ------------------------------------------ epilogue 1: A and P --
        tc::tc_fence_after();
        const int row = 32 * q + lane;       // 0..63 rows of A, 64..127 rows of P
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          float v[16];
          tc::tmem_ld16(tc::tmem_addr(tbase, 32 * q, 32 * half + 16 * m), v);
          tc::tmem_wait_ld();
          const int j0 = 32 * half + 16 * m;
          if (q < 2) {
            const int i = row;
#pragma unroll
            for (int e = 0; e < 16; ++e) AS[i * C::LDA + j0 + e] = (j0 + e < i) ? v[e] : 0.f;
          } else {
            const int i = row - 64;
            uint32_t pw[8];
#pragma unroll
            for (int e = 0; e < 16; e += 2)
              pw[e / 2] = tc::pack_bf16(j0 + e <= i ? v[e] : 0.f, j0 + e + 1 <= i ? v[e + 1] : 0.f);
            *reinterpret_cast<uint4*>(sm + C::OFF_PB + sw_unit(i, j0 >> 3)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            *reinterpret_cast<uint4*>(sm + C::OFF_PB + sw_unit(i, (j0 >> 3) + 1)) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
          }
        }
        bar_compute();
        // ------------------------------------------ T = (I + A)^-1, fp32 --
        if (warp < 4) {
          // diagonal block I = warp; lane l < 16 owns column l
          const int I = warp, l = lane;
          float t[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float accv = 0.f;
#pragma unroll
            for (int m = 0; m < i; ++m)
              if (m >= l) accv = fmaf(AS[(16 * I + i) * C::LDA + 16 * I + m], t[m], accv);
            t[i] = i < l ? 0.f : (i == l ? 1.f : -accv);
          }
          if (l < 16)
#pragma unroll
            for (int i = 0; i < 16; ++i) TS[(16 * I + i) * C::LDA + 16 * I + l] = t[i];
        } else {
          // zero the blocks above the diagonal
          for (int idx = tid - 128; idx < 64 * 64; idx += 128) {
            const int r = idx >> 6, cc = idx & 63;
            if ((cc >> 4) > (r >> 4)) TS[r * C::LDA + cc] = 0.f;
          }
        }
        bar_compute();
        float* XS = reinterpret_cast<float*>(sm + C::OFF_XS);
        for (int dist = 1; dist < 4; ++dist) {
          const int nblk = 4 - dist;
          // X_b = sum_{K=J}^{I-1} A_{I,K} T_{K,J}  for block b = (I = J + dist, J)
          for (int idx = tid; idx < nblk * 256; idx += 256) {
            const int J = idx >> 8, I = J + dist, r = (idx >> 4) & 15, cc = idx & 15;
            float accv = 0.f;
            for (int K = J; K < I; ++K)
#pragma unroll
              for (int m = 0; m < 16; ++m)
                accv = fmaf(AS[(16 * I + r) * C::LDA + 16 * K + m], TS[(16 * K + m) * C::LDA + 16 * J + cc], accv);
            XS[idx] = accv;
          }
          bar_compute();
          // T_{I,J} = -T_{I,I} X_b
          for (int idx = tid; idx < nblk * 256; idx += 256) {
            const int J = idx >> 8, I = J + dist, r = (idx >> 4) & 15, cc = idx & 15;
            float accv = 0.f;
#pragma unroll
            for (int m = 0; m < 16; ++m)
              accv = fmaf(TS[(16 * I + r) * C::LDA + 16 * I + m], XS[(J << 8) + m * 16 + cc], accv);
            TS[(16 * I + r) * C::LDA + 16 * J + cc] = -accv;
          }
          bar_compute();
        }
        // T -> bf16 hi + lo, MN-major SW128 (row i, 64 columns j)
        {
          const int i = tid >> 2, j0 = 16 * (tid & 3);
          uint32_t hw[8], lw[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const float x0 = TS[i * C::LDA + j0 + e], x1 = TS[i * C::LDA + j0 + e + 1];
            const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
            hw[e / 2] = tc::pack_bf16(__bfloat162float(h0), __bfloat162float(h1));
            lw[e / 2] = tc::pack_bf16(x0 - __bfloat162float(h0), x1 - __bfloat162float(h1));
          }
          const uint32_t u = j0 >> 3;
          *reinterpret_cast<uint4*>(sm + C::OFF_THI + sw_unit(i, u)) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(sm + C::OFF_THI + sw_unit(i, u + 1)) = make_uint4(hw[4], hw[5], hw[6], hw[7]);
          *reinterpret_cast<uint4*>(sm + C::OFF_TLO + sw_unit(i, u)) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
          *reinterpret_cast<uint4*>(sm + C::OFF_TLO + sw_unit(i, u + 1)) = make_uint4(lw[4], lw[5], lw[6], lw[7]);
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(t_ready);
        ok = tc::mbar_wait(mma2_done, 0);
      }
      if (ok) {
        // ---------------------------------------- epilogue 2: R and V -> bf16 --
        tc::tc_fence_after();
#pragma unroll
        for (int m = 0; m < 2; ++m) {
          const int j0 = 32 * half + 16 * m;
          float v[16];
          tc::tmem_ld16(tc::tmem_addr(tbase, 32 * q, 64 + j0), v);
          tc::tmem_wait_ld();
          uint32_t pw[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) pw[e / 2] = tc::pack_bf16(v[e], v[e + 1]);
          const int rr = 32 * q + lane;  // channel row of R
          *reinterpret_cast<uint4*>(sm + C::OFF_RB + sw_unit(rr, j0 >> 3)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
          *reinterpret_cast<uint4*>(sm + C::OFF_RB + sw_unit(rr, (j0 >> 3) + 1)) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
          tc::tmem_ld16(tc::tmem_addr(tbase, 32 * q, 128 + j0), v);
          tc::tmem_wait_ld();
          if (lane < 16) {
            const int i = 16 * q + lane;  // token row of V (M = 64 layout)
#pragma unroll
            for (int e = 0; e < 16; e += 2) pw[e / 2] = tc::pack_bf16(v[e], v[e + 1]);
            *reinterpret_cast<uint4*>(sm + C::OFF_VB + sw_unit(i, j0 >> 3)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            *reinterpret_cast<uint4*>(sm + C::OFF_VB + sw_unit(i, (j0 >> 3) + 1)) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
          }
        }
        tc::fence_async_smem();
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(rv_ready);
        ok = tc::mbar_wait(mma3_done, 0);
      }
      if (ok) {
        // ------------------------------------------- epilogue 3: outputs --
        tc::tc_fence_after();
        const size_t tile = (size_t)c * H + h;
        const int mrow = 32 * q + lane;  // key channel (Mp, Nc)
        // Mp: columns [64 half, 64 half + 64)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float v[16];
          const int c0 = 64 * half + 16 * m;
          tc::tmem_ld16(tc::tmem_addr(tbase, 32 * q, c0), v);
          tc::tmem_wait_ld();
          uint32_t pw[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) pw[e / 2] = tc::pack_bf16(v[e], v[e + 1]);
          uint4* dst = reinterpret_cast<uint4*>(a.Mp + (tile * DK + mrow) * DK + c0);
          dst[0] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
          dst[1] = make_uint4(pw[4], pw[5], pw[6], pw[7]);
        }
        // Nc: columns [DV/2 half, DV/2 half + DV/2)
#pragma unroll
        for (int m = 0; m < DV / 32; ++m) {
          float v[16];
          const int c0 = (DV / 2) * half + 16 * m;
          tc::tmem_ld16(tc::tmem_addr(tbase, 32 * q, 128 + c0), v);
          tc::tmem_wait_ld();
          uint32_t pw[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) pw[e / 2] = tc::pack_bf16(v[e], v[e + 1]);
          uint4* dst = reinterpret_cast<uint4*>(a.Nc + (tile * DK + mrow) * DV + c0);
          dst[0] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
          dst[1] = make_uint4(pw[4], pw[5], pw[6], pw[7]);
        }
        // Q_eff = Q~ - P W and O_part (M = 64 layout: token 16 q + lane, lane < 16)
        const int i = 16 * q + lane;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float v[16];
          const int c0 = 64 * half + 16 * m;
          tc::tmem_ld16(tc::tmem_addr(tbase, 32 * q, 256 + c0), v);
          tc::tmem_wait_ld();
          if (lane < 16) {
            const uint4 t0v = *reinterpret_cast<const uint4*>(sm + C::OFF_QT + i * 256 + c0 * 2);
            const uint4 t1v = *reinterpret_cast<const uint4*>(sm + C::OFF_QT + i * 256 + c0 * 2 + 16);
            const uint32_t qw[8] = {t0v.x, t0v.y, t0v.z, t0v.w, t1v.x, t1v.y, t1v.z, t1v.w};
            uint32_t pw[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              pw[e] = tc::pack_bf16(bf16_lo_f(qw[e]) - v[2 * e], bf16_hi_f(qw[e]) - v[2 * e + 1]);
            uint4* dst = reinterpret_cast<uint4*>(a.Qeff + (tile * kChunk + i) * DK + c0);
            dst[0] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            dst[1] = make_uint4(pw[4], pw[5], pw[6], pw[7]);
          }
        }
#pragma unroll
        for (int m = 0; m < DV / 32; ++m) {
          float v[16];
          const int c0 = (DV / 2) * half + 16 * m;
          tc::tmem_ld16(tc::tmem_addr(tbase, 32 * q, 384 + c0), v);
          tc::tmem_wait_ld();
          if (lane < 16) {
            uint32_t pw[8];
#pragma unroll
            for (int e = 0; e < 16; e += 2) pw[e / 2] = tc::pack_bf16(v[e], v[e + 1]);
            uint4* dst = reinterpret_cast<uint4*>(a.Opart + (tile * kChunk + i) * DV + c0);
            dst[0] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            dst[1] = make_uint4(pw[4], pw[5], pw[6], pw[7]);
          }
        }
      }
      if (!ok) {
        atomicExch(a.status, 8);
        vflag[1] = 1;
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == C::COMPUTE_WARPS) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace gdn2
