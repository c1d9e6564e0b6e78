// prep_tc.cuh -- gate preparation + intra-chunk WY + the chunk's affine state
// map on the tensor cores (bf16 I/O, dk = 128, dv in {64, 128}).
//
// Persistent CTAs walk a list of (chunk, head) tasks.  Warps 0-7 compute,
// warp 8 streams the inputs by TMA, warp 9 issues the UMMAs.  Per chunk of
// n <= 64 tokens (page "Gated DeltaNet-2：将擦除与写入分开", sections
// "在两个维度上独立控制" and "词元路径与并行训练"; the algebra is the recurrence
// unrolled over one chunk, written as products):
//
//  1. Gate prep (fp32).  The inputs stream in 32-channel slices through a
//     3-slot TMA ring that runs ahead across tasks; per slice: g = in-chunk
//     cumulative sum of log_alpha, and the bf16 operands, all with the decay
//     folded in around one reference token r = 32 of the chunk:
//        E^_i = b_i k_i exp(g_i - g_r),  Q^_i = q_i exp(g_i - g_r),
//        K^_j = k_j exp(g_r - g_j),      E~_i = b_i k_i exp(g_i),
//        Kbar_j = k_j exp(g_n - g_j),    Q~_i = q_i exp(g_i),  Z_i = w_i v_i.
//     For j <= i the product of the two factors is exp(g_i - g_j) <= 1; each
//     factor alone stays inside exp(+-80) as long as no 32-token stretch of a
//     channel decays by more than 80 nats.  A chunk that breaks this bound is
//     handed back for the exact fp32 kernel (prep_fixup_kernel).
//  2. UMMA 1: [E^; Q^] . K^T  (M = 128, N = 64, K = 128) -> A (strictly lower
//     part of rows 0..63) and P (lower part with diagonal, rows 64..127).
//  3. T = (I + A)^-1 in fp32 on the CUDA cores: the four 16 x 16 diagonal
//     blocks by forward substitution, then each block column below the
//     diagonal by a warp pair; T is split into bf16 hi + lo, stored side by
//     side as one operand so one UMMA applies both (~16 bits of T kept).
//  4. UMMA 2: [R_hi | R_lo] = Kbar^T [T_hi | T_lo], [V_hi | V_lo] = P [T_hi | T_lo].
//  5. UMMA 3: [Mp | Nc] = R [E~ | Z], [P W | O_part] = V [E~ | Z]; the epilogue
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
  // outputs, stored by TMA from SW128 staging: box {64, 128} (Mp, Nc), {64, 64} (Q_eff, O_part)
  CUtensorMap tm_Mp, tm_Nc, tm_Qe, tm_Op;
  SeqMap map;
  int H;
  __nv_bfloat16* Qeff;   // [max_chunks, H, 64, 128]   (holds Q~ between the two phases)
  __nv_bfloat16* Opart;  // [max_chunks, H, 64, DV]
  __nv_bfloat16* Mp;     // [max_chunks, H, 128, 128]
  __nv_bfloat16* Nc;     // [max_chunks, H, 128, DV]
  float* gamma_last;     // [max_chunks, H, 128]
  int32_t* fix_list;     // [0] = count, then c * H + h of handed-back chunks
  int* ready;            // optional [max_chunks * H]: 1 = factors written, 2 = handed back
  int* task_counter;     // optional: tasks taken dynamically (else static striding)
  int* status;
};

template <int DV>
struct PrepTcCfg {
  static constexpr int DK = 128;
  static constexpr int KS = 32;             // key channels per slice
  static constexpr int VS = DV / 4;         // value channels per slice
  static constexpr int SLICES = 4;
  static constexpr int NSLOT = 3;
  static constexpr int COMPUTE_WARPS = 8;
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9;
  static constexpr int THREADS = 10 * 32;
  // raw slot: la, b fp32 [64][32]; q, k bf16 [64][32]; v bf16 [64][VS]; w fp32 [64][VS]
  static constexpr int OFF_LA = 0, OFF_B = 8192, OFF_Q = 16384, OFF_K = 20480, OFF_V = 24576;
  static constexpr int OFF_W = OFF_V + kChunk * VS * 2;
  static constexpr int SLOT_BYTES = OFF_W + kChunk * VS * 4;
  static constexpr int SLOT_STRIDE = 36864;
  static constexpr int RING = NSLOT * SLOT_STRIDE;
  // operands (1024-aligned)
  static constexpr int OFF_X = RING;            // [E^; Q^] K-major SW128, 2 panels x 128 rows
  static constexpr int OFF_KH = OFF_X + 32768;  // K^ K-major SW128, 2 panels x 64 rows
  static constexpr int OFF_ET = OFF_KH + 16384; // E~ MN-major SW128 (rows = tokens), 2 panels
  static constexpr int OFF_Z = OFF_ET + 16384;  // Z right after E~: [E~ | Z] is one operand
  static constexpr int OFF_KB = OFF_Z + 16384;  // Kbar^T MN-major SW128 A operand, 2 panels
  static constexpr int OFF_T = OFF_KB + 16384;  // [T_hi | T_lo] MN-major SW128, 2 panels
  static constexpr int OFF_BAR = OFF_T + 16384;
  // reuse of [E^; Q^] and K^ (48 KiB) once UMMA 1 has read them
  static constexpr int LDA = 68;                // fp32 row stride of A and T
  static constexpr int OFF_AS = OFF_X, OFF_TS = OFF_X + 17408, OFF_XS = OFF_X + 34816;
  static constexpr int OFF_PB = OFF_X + 38912;  // P as K-major SW128 operand
  static constexpr int OFF_RB = OFF_X, OFF_VB = OFF_X + 16384;  // after UMMA 2
  // output staging once UMMA 3 has read every operand (SW128 panels of 64 columns)
  static constexpr int OFF_SMP = OFF_X, OFF_SNC = OFF_X + 32768, OFF_SQE = OFF_X + 65536, OFF_SOP = OFF_X + 81920;
  static_assert(OFF_SOP + 16384 <= OFF_BAR, "output staging fits in the operand area");
  static constexpr int SMEM = 1024 + OFF_BAR + 2048;
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t COL_D1 = 0, COL_R = 64, COL_V = 192, COL_MN = 0, COL_QO = 256;
  static_assert(SLOT_BYTES <= SLOT_STRIDE, "slot fits");
  static_assert(OFF_PB + 8192 <= OFF_X + 49152, "solve scratch fits in the freed operands");
  static_assert(SMEM <= 232448, "shared memory");
};

__device__ __forceinline__ void bar_compute() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ void bar_pair(int id) { asm volatile("bar.sync %0, 64;" ::"r"(id) : "memory"); }

// byte offset of the 16-byte unit holding elements [8u, 8u+8) of row `row`
// in an SW128 panel (rows of 64 bf16)
__device__ __forceinline__ uint32_t sw_unit(uint32_t row, uint32_t u) { return row * 128u + ((u ^ (row & 7u)) << 4); }

__device__ __forceinline__ void store8(uint8_t* p, const uint32_t (&w)[8], int at) {
  *reinterpret_cast<uint4*>(p) = make_uint4(w[at], w[at + 1], w[at + 2], w[at + 3]);
}

template <int DV>
__device__ void prep_tc_cta(const PrepTcArgs& a, uint8_t* sm, int cta_rank, int cta_count) {
  using C = PrepTcCfg<DV>;
  constexpr int DK = C::DK;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);  // [NSLOT]
  uint64_t* empty = full + C::NSLOT;                                // [NSLOT]
  uint64_t* ops_ready = empty + C::NSLOT;
  uint64_t* mma1_done = ops_ready + 1;
  uint64_t* t_ready = mma1_done + 1;
  uint64_t* mma2_done = t_ready + 1;
  uint64_t* rv_ready = mma2_done + 1;
  uint64_t* mma3_done = rv_ready + 1;
  uint64_t* task_full = mma3_done + 1;   // [2] task ids handed from producer to compute
  uint64_t* task_empty = task_full + 2;  // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(task_empty + 2);
  int* s_flag = reinterpret_cast<int*>(tslot + 1);   // [0] abort, [1] done, [2 + (task & 1)] hand back
  int* s_task = s_flag + 4;                          // [2] task ids
  float* s_tot = reinterpret_cast<float*>(s_task + 2);  // [8][32] segment totals
  float* s_er = s_tot + 256;                             // [32] exp(g_r)
  float* s_enr = s_er + 32;                              // [32] exp(g_n - g_r)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H;
  const int ntasks = a.map.chunk_off[a.map.N] * H;

  if (tid == 0) {
    for (int s = 0; s < C::NSLOT; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], C::COMPUTE_WARPS);
    }
    tc::mbar_init(ops_ready, C::COMPUTE_WARPS);
    tc::mbar_init(mma1_done, 1);
    tc::mbar_init(t_ready, C::COMPUTE_WARPS);
    tc::mbar_init(mma2_done, 1);
    tc::mbar_init(rv_ready, C::COMPUTE_WARPS);
    tc::mbar_init(mma3_done, 1);
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(&task_full[s], 1);
      tc::mbar_init(&task_empty[s], C::COMPUTE_WARPS);
    }
    s_flag[0] = s_flag[1] = s_flag[2] = s_flag[3] = 0;
    tc::fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tc::tmem_alloc(tslot, C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tslot;
  volatile int* vflag = s_flag;

  if (warp == C::PRODUCER_WARP) {
    // ---------------------------------------------------- input producer --
    // Takes tasks (dynamic counter or static stride), hands each task id to
    // the compute warps through a 2-entry mailbox, and streams its four input
    // slices through the ring.  A task id of -1 ends the CTA's work.
    if (lane == 0) {
      int gs = 0, nt = 0, k_static = 0;
      bool ok = true;
      while (ok) {
        int task;
        if (a.task_counter) task = atomicAdd(a.task_counter, 1);
        else task = cta_rank + cta_count * (k_static++);
        if (task >= ntasks) task = -1;
        const int mb = nt & 1;
        if (nt >= 2 && !tc::mbar_wait(&task_empty[mb], ((nt - 2) >> 1) & 1)) { ok = false; break; }
        s_task[mb] = task;
        tc::mbar_arrive(&task_full[mb]);
        ++nt;
        if (task < 0 || vflag[0]) break;
        const int c = task / H, h = task % H;
        const int t0 = chunk_pos(a.map, c).t0;
        for (int s = 0; s < C::SLICES; ++s, ++gs) {
          const int slot = gs % C::NSLOT, use = gs / C::NSLOT;
          if (use > 0 && !tc::mbar_wait(&empty[slot], (use - 1) & 1)) { ok = false; break; }
          uint8_t* d = sm + slot * C::SLOT_STRIDE;
          tc::mbar_arrive_expect_tx(&full[slot], C::SLOT_BYTES);
          tc::tma_load_3d(d + C::OFF_LA, &a.tm_la, &full[slot], C::KS * s, h, t0);
          tc::tma_load_3d(d + C::OFF_B, &a.tm_b, &full[slot], C::KS * s, h, t0);
          tc::tma_load_3d(d + C::OFF_Q, &a.tm_q, &full[slot], C::KS * s, h, t0);
          tc::tma_load_3d(d + C::OFF_K, &a.tm_k, &full[slot], C::KS * s, h, t0);
          tc::tma_load_3d(d + C::OFF_V, &a.tm_v, &full[slot], C::VS * s, h, t0);
          tc::tma_load_3d(d + C::OFF_W, &a.tm_w, &full[slot], C::VS * s, h, t0);
        }
      }
      if (!ok) {
        atomicExch(a.status, 8 /* GDN2_ERR_DEVICE_TIMEOUT */);
        vflag[0] = 1;
      }
      // every issued load has landed before the CTA can exit
      for (int g = gs > C::NSLOT ? gs - C::NSLOT : 0; g < gs; ++g)
        tc::mbar_wait(&full[g % C::NSLOT], (g / C::NSLOT) & 1);
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------- UMMA issue --
    // One round of three UMMA groups per task the compute warps did not hand
    // back; the compute warps arrive once more with s_flag[2] set when done.
    if (lane == 0) {
      const uint32_t X = tc::smem_u32(sm + C::OFF_X), KH = tc::smem_u32(sm + C::OFF_KH);
      const uint32_t EZ = tc::smem_u32(sm + C::OFF_ET), KB = tc::smem_u32(sm + C::OFF_KB);
      const uint32_t TT = tc::smem_u32(sm + C::OFF_T), PB = tc::smem_u32(sm + C::OFF_PB);
      const uint32_t RB = tc::smem_u32(sm + C::OFF_RB), VB = tc::smem_u32(sm + C::OFF_VB);
      const uint32_t SW = tc::kLayoutSW128;
      constexpr uint32_t id1 = tc::idesc_bf16(128, 64, false, false);
      constexpr uint32_t idR = tc::idesc_bf16(128, 128, true, true);
      constexpr uint32_t idV = tc::idesc_bf16(64, 128, false, true);
      constexpr uint32_t idM = tc::idesc_bf16(128, 128 + DV, false, true);
      constexpr uint32_t idQ = tc::idesc_bf16(64, 128 + DV, false, true);
      for (int ex = 0;; ++ex) {
        if (!tc::mbar_wait(ops_ready, ex & 1)) break;
        if (vflag[1] || vflag[0]) break;
        tc::tc_fence_after();
#pragma unroll
        for (int s = 0; s < DK / 16; ++s) {
          const uint32_t ko = (s >> 2), kk = (s & 3) * 32;
          tc::umma_f16(tbase + C::COL_D1, tc::sdesc(X + ko * 16384 + kk, 16, 1024, SW),
                       tc::sdesc(KH + ko * 8192 + kk, 16, 1024, SW), id1, s > 0);
        }
        tc::umma_commit(mma1_done);
        if (!tc::mbar_wait(t_ready, ex & 1) || vflag[0]) break;
        tc::tc_fence_after();
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t t_d = tc::sdesc(TT + s * 2048, 8192, 1024, SW);
          tc::umma_f16(tbase + C::COL_R, tc::sdesc(KB + s * 2048, 8192, 1024, SW), t_d, idR, s > 0);
          tc::umma_f16(tbase + C::COL_V, tc::sdesc(PB + s * 32, 16, 1024, SW), t_d, idV, s > 0);
        }
        tc::umma_commit(mma2_done);
        if (!tc::mbar_wait(rv_ready, ex & 1) || vflag[0]) break;
        tc::tc_fence_after();
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          const uint64_t ez_d = tc::sdesc(EZ + s * 2048, 8192, 1024, SW);
          tc::umma_f16(tbase + C::COL_MN, tc::sdesc(RB + s * 32, 16, 1024, SW), ez_d, idM, s > 0);
          tc::umma_f16(tbase + C::COL_QO, tc::sdesc(VB + s * 32, 16, 1024, SW), ez_d, idQ, s > 0);
        }
        tc::umma_commit(mma3_done);
      }
    }
  } else {
    // ----------------------------------------------------------- compute --
    const int q = warp & 3, half = warp >> 2;
    int gs = 0, ex = 0;
    bool alive = true;
    for (int nt = 0; alive; ++nt) {
      const int mb = nt & 1;
      if (!tc::mbar_wait(&task_full[mb], (nt >> 1) & 1)) {
        atomicExch(a.status, 8);
        vflag[0] = 1;
        break;
      }
      const int task = s_task[mb];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&task_empty[mb]);
      if (task < 0 || vflag[0]) break;
      const int c = task / H, h = task % H;
      const ChunkPos pos = chunk_pos(a.map, c);
      const int len = pos.len;
      const size_t tile = (size_t)c * H + h;
      volatile int* skipflag = vflag + 2 + (nt & 1);
      if (tid == 0) {
        *skipflag = 0;
        tc::tma_store_wait_read();  // previous task's output staging has been read
      }
      bar_compute();
      // ------------------------------------------------------ slices --
      for (int s = 0; s < C::SLICES; ++s, ++gs) {
        const int slot = gs % C::NSLOT;
        uint8_t* d = sm + slot * C::SLOT_STRIDE;
        float* la = reinterpret_cast<float*>(d + C::OFF_LA);   // becomes g
        if (!tc::mbar_wait(&full[slot], (gs / C::NSLOT) & 1)) {
          atomicExch(a.status, 8);
          vflag[0] = 1;
          alive = false;
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
          if (g0 - gr > 80.f || gr - gn > 80.f) *skipflag = 1;
          s_er[lane] = __expf(gr);
          s_enr[lane] = __expf(gn - gr);
          a.gamma_last[tile * DK + C::KS * s + lane] = expf(gn);
        }
        bar_compute();
        // operands for token i, key channels cc0 .. cc0 + 7
        {
          const int i = tid >> 2, gq = tid & 3, cl = 8 * gq, cc0 = C::KS * s + cl;
          const bool live = i < len;
          // 8 consecutive fp32 values per thread, read as two float4 (scalar
          // reads of 8 token rows 128 B apart would hit the same banks)
          float gi[8], gr[8], bb[8];
          {
            const float4* g4 = reinterpret_cast<const float4*>(la + i * 32 + cl);
            const float4* r4 = reinterpret_cast<const float4*>(la + 32 * 32 + cl);
            const float4* b4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(d + C::OFF_B) + i * 32 + cl);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const float4 x = g4[hh], y = r4[hh], z = b4[hh];
              gi[4 * hh] = x.x; gi[4 * hh + 1] = x.y; gi[4 * hh + 2] = x.z; gi[4 * hh + 3] = x.w;
              gr[4 * hh] = y.x; gr[4 * hh + 1] = y.y; gr[4 * hh + 2] = y.z; gr[4 * hh + 3] = y.w;
              bb[4 * hh] = z.x; bb[4 * hh + 1] = z.y; bb[4 * hh + 2] = z.z; bb[4 * hh + 3] = z.w;
            }
          }
          const uint4 kraw = *reinterpret_cast<const uint4*>(d + C::OFF_K + (i * 32 + cl) * 2);
          const uint4 qraw = *reinterpret_cast<const uint4*>(d + C::OFF_Q + (i * 32 + cl) * 2);
          const uint32_t kw[4] = {kraw.x, kraw.y, kraw.z, kraw.w};
          const uint32_t qw[4] = {qraw.x, qraw.y, qraw.z, qraw.w};
          uint32_t eh[8], kh[8], et[4], kb[4], qt[4];
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
            eh[4 + p] = tc::pack_bf16(o_qh[0], o_qh[1]);
            kh[p] = tc::pack_bf16(o_kh[0], o_kh[1]);
            et[p] = tc::pack_bf16(o_et[0], o_et[1]);
            kb[p] = tc::pack_bf16(o_kb[0], o_kb[1]);
            qt[p] = tc::pack_bf16(o_qt[0], o_qt[1]);
          }
          const uint32_t pnl = cc0 >> 6, u = (cc0 & 63) >> 3;
          store8(sm + C::OFF_X + pnl * 16384 + sw_unit(i, u), eh, 0);
          store8(sm + C::OFF_X + pnl * 16384 + sw_unit(64 + i, u), eh, 4);
          *reinterpret_cast<uint4*>(sm + C::OFF_KH + pnl * 8192 + sw_unit(i, u)) = make_uint4(kh[0], kh[1], kh[2], kh[3]);
          *reinterpret_cast<uint4*>(sm + C::OFF_ET + pnl * 8192 + sw_unit(i, u)) = make_uint4(et[0], et[1], et[2], et[3]);
          *reinterpret_cast<uint4*>(sm + C::OFF_KB + pnl * 8192 + sw_unit(i, u)) = make_uint4(kb[0], kb[1], kb[2], kb[3]);
          // Q~ waits in the Q_eff buffer until the last epilogue
          *reinterpret_cast<uint4*>(a.Qeff + (tile * kChunk + i) * DK + cc0) = make_uint4(qt[0], qt[1], qt[2], qt[3]);
          // Z = w * v for value channels vc0 .. vc0 + VS/4 - 1 (right after E~)
          constexpr int VPT = C::VS / 4;
          const int vl = VPT * gq, vc0 = C::VS * s + vl;
          float ww[VPT];
          uint32_t vw[VPT / 2];
          {
            const float4* w4 = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(d + C::OFF_W) + i * C::VS + vl);
#pragma unroll
            for (int hh = 0; hh < VPT / 4; ++hh) {
              const float4 x = w4[hh];
              ww[4 * hh] = x.x; ww[4 * hh + 1] = x.y; ww[4 * hh + 2] = x.z; ww[4 * hh + 3] = x.w;
            }
            const uint8_t* vsrc = d + C::OFF_V + (i * C::VS + vl) * 2;
            if constexpr (VPT == 8) {
              const uint4 x = *reinterpret_cast<const uint4*>(vsrc);
              vw[0] = x.x; vw[1] = x.y; vw[2] = x.z; vw[3] = x.w;
            } else {
              const uint2 x = *reinterpret_cast<const uint2*>(vsrc);
              vw[0] = x.x; vw[1] = x.y;
            }
          }
          uint32_t zw[VPT / 2];
#pragma unroll
          for (int p = 0; p < VPT / 2; ++p) {
            const float z0 = live ? ww[2 * p] * bf16_lo_f(vw[p]) : 0.f;
            const float z1 = live ? ww[2 * p + 1] * bf16_hi_f(vw[p]) : 0.f;
            zw[p] = tc::pack_bf16(z0, z1);
          }
          uint8_t* zdst = sm + C::OFF_Z + (vc0 >> 6) * 8192 + sw_unit(i, (vc0 & 63) >> 3) + (vc0 & 7) * 2;
          if constexpr (VPT == 8) *reinterpret_cast<uint4*>(zdst) = make_uint4(zw[0], zw[1], zw[2], zw[3]);
          else *reinterpret_cast<uint2*>(zdst) = make_uint2(zw[0], zw[1]);
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&empty[slot]);
      }
      if (!alive) break;
      tc::fence_async_smem();
      tc::tc_fence_before();
      bar_compute();
      if (*skipflag) {
        // decay too steep for one reference point: hand the chunk back
        if (tid == 0) {
          const int idx = atomicAdd(a.fix_list, 1);
          a.fix_list[1 + idx] = (int)tile;
          if (a.ready) tc::st_release_gpu(a.ready + tile, 2);
        }
        continue;
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(ops_ready);
      float* AS = reinterpret_cast<float*>(sm + C::OFF_AS);
      float* TS = reinterpret_cast<float*>(sm + C::OFF_TS);
      float* XS = reinterpret_cast<float*>(sm + C::OFF_XS);
      if (!tc::mbar_wait(mma1_done, ex & 1)) { alive = false; break; }
      // -------------------------------------------- epilogue 1: A and P --
      tc::tc_fence_after();
      {
        uint32_t r[32];
        tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, C::COL_D1 + 32 * half), r);
        tc::tmem_wait_ld();
        const int j0 = 32 * half;
        if (q < 2) {
          const int i = 32 * q + lane;
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            float4 v4;
            v4.x = (j0 + e < i) ? __uint_as_float(r[e]) : 0.f;
            v4.y = (j0 + e + 1 < i) ? __uint_as_float(r[e + 1]) : 0.f;
            v4.z = (j0 + e + 2 < i) ? __uint_as_float(r[e + 2]) : 0.f;
            v4.w = (j0 + e + 3 < i) ? __uint_as_float(r[e + 3]) : 0.f;
            *reinterpret_cast<float4*>(AS + i * C::LDA + j0 + e) = v4;
          }
        } else {
          const int i = 32 * q + lane - 64;
          uint32_t pw[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            pw[e / 2] = tc::pack_bf16(j0 + e <= i ? __uint_as_float(r[e]) : 0.f,
                                      j0 + e + 1 <= i ? __uint_as_float(r[e + 1]) : 0.f);
#pragma unroll
          for (int uu = 0; uu < 4; ++uu)
            *reinterpret_cast<uint4*>(sm + C::OFF_PB + sw_unit(i, (j0 >> 3) + uu)) =
                make_uint4(pw[4 * uu], pw[4 * uu + 1], pw[4 * uu + 2], pw[4 * uu + 3]);
        }
      }
      bar_compute();
      // ------------------------------------------- T = (I + A)^-1, fp32 --
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
        for (int idx = tid - 128; idx < 64 * 64; idx += 128) {
          const int rr = idx >> 6, cc = idx & 63;
          if ((cc >> 4) > (rr >> 4)) TS[rr * C::LDA + cc] = 0.f;
        }
      }
      bar_compute();
      // block column J below the diagonal, by warps J and J + 4 (64 threads):
      // thread (r = row in block, cg = 4-column group)
      if ((warp & 3) < 3) {
        const int J = warp & 3, pt = (warp >> 2) * 32 + lane;   // 0..63 within the pair
        const int r = pt >> 2, cg = pt & 3;
        float* X = XS + J * 256;
        for (int I = J + 1; I < 4; ++I) {
          float4 xa = make_float4(0.f, 0.f, 0.f, 0.f);
          for (int kb = J; kb < I; ++kb) {
            const float* arow = AS + (16 * I + r) * C::LDA + 16 * kb;
            const float* tcol = TS + (16 * kb) * C::LDA + 16 * J + 4 * cg;
            float av[16];
#pragma unroll
            for (int m = 0; m < 16; m += 4) {
              const float4 a4 = *reinterpret_cast<const float4*>(arow + m);
              av[m] = a4.x; av[m + 1] = a4.y; av[m + 2] = a4.z; av[m + 3] = a4.w;
            }
#pragma unroll
            for (int m = 0; m < 16; ++m) {
              const float4 tv = *reinterpret_cast<const float4*>(tcol + m * C::LDA);
              xa.x = fmaf(av[m], tv.x, xa.x); xa.y = fmaf(av[m], tv.y, xa.y);
              xa.z = fmaf(av[m], tv.z, xa.z); xa.w = fmaf(av[m], tv.w, xa.w);
            }
          }
          *reinterpret_cast<float4*>(X + r * 16 + 4 * cg) = xa;
          bar_pair(2 + J);
          float4 ta = make_float4(0.f, 0.f, 0.f, 0.f);
          float tr[16];
#pragma unroll
          for (int m = 0; m < 16; m += 4) {
            const float4 t4 = *reinterpret_cast<const float4*>(TS + (16 * I + r) * C::LDA + 16 * I + m);
            tr[m] = t4.x; tr[m + 1] = t4.y; tr[m + 2] = t4.z; tr[m + 3] = t4.w;
          }
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            const float tv = tr[m];
            const float4 xv = *reinterpret_cast<const float4*>(X + m * 16 + 4 * cg);
            ta.x = fmaf(tv, xv.x, ta.x); ta.y = fmaf(tv, xv.y, ta.y);
            ta.z = fmaf(tv, xv.z, ta.z); ta.w = fmaf(tv, xv.w, ta.w);
          }
          *reinterpret_cast<float4*>(TS + (16 * I + r) * C::LDA + 16 * J + 4 * cg) =
              make_float4(-ta.x, -ta.y, -ta.z, -ta.w);
          bar_pair(2 + J);
        }
      }
      bar_compute();
      // T -> [T_hi | T_lo], MN-major SW128 (row i, 64 columns j per panel)
      {
        const int i = tid >> 2, j0 = 16 * (tid & 3);
        uint32_t hw[8], lw[8];
        float tv[16];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 t4 = *reinterpret_cast<const float4*>(TS + i * C::LDA + j0 + e);
          tv[e] = t4.x; tv[e + 1] = t4.y; tv[e + 2] = t4.z; tv[e + 3] = t4.w;
        }
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const float x0 = tv[e], x1 = tv[e + 1];
          const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
          hw[e / 2] = tc::pack_bf16(__bfloat162float(h0), __bfloat162float(h1));
          lw[e / 2] = tc::pack_bf16(x0 - __bfloat162float(h0), x1 - __bfloat162float(h1));
        }
        const uint32_t u = j0 >> 3;
        store8(sm + C::OFF_T + sw_unit(i, u), hw, 0);
        store8(sm + C::OFF_T + sw_unit(i, u + 1), hw, 4);
        store8(sm + C::OFF_T + 8192 + sw_unit(i, u), lw, 0);
        store8(sm + C::OFF_T + 8192 + sw_unit(i, u + 1), lw, 4);
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(t_ready);
      if (!tc::mbar_wait(mma2_done, ex & 1)) { alive = false; break; }
      // ---------------------------------- epilogue 2: R, V = hi + lo -> bf16 --
      tc::tc_fence_after();
      {
        const int j0 = 32 * half;
        uint32_t rh[32], rl[32], pw[16];
        tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, C::COL_R + j0), rh);
        tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, C::COL_R + 64 + j0), rl);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          pw[e / 2] = tc::pack_bf16(__uint_as_float(rh[e]) + __uint_as_float(rl[e]),
                                    __uint_as_float(rh[e + 1]) + __uint_as_float(rl[e + 1]));
        const int m = 32 * q + lane;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu)
          *reinterpret_cast<uint4*>(sm + C::OFF_RB + sw_unit(m, (j0 >> 3) + uu)) =
              make_uint4(pw[4 * uu], pw[4 * uu + 1], pw[4 * uu + 2], pw[4 * uu + 3]);
        tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, C::COL_V + j0), rh);
        tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, C::COL_V + 64 + j0), rl);
        tc::tmem_wait_ld();
        if (lane < 16) {
          const int i = 16 * q + lane;
#pragma unroll
          for (int e = 0; e < 32; e += 2)
            pw[e / 2] = tc::pack_bf16(__uint_as_float(rh[e]) + __uint_as_float(rl[e]),
                                      __uint_as_float(rh[e + 1]) + __uint_as_float(rl[e + 1]));
#pragma unroll
          for (int uu = 0; uu < 4; ++uu)
            *reinterpret_cast<uint4*>(sm + C::OFF_VB + sw_unit(i, (j0 >> 3) + uu)) =
                make_uint4(pw[4 * uu], pw[4 * uu + 1], pw[4 * uu + 2], pw[4 * uu + 3]);
        }
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(rv_ready);
      // Q~ for this thread's output row, while UMMA 3 runs
      const int i_out = 16 * q + lane;
      uint4 qt_r[DK / 8];   // the row's 128 bf16 values of Q~
      if (half == 0 && lane < 16) {
        const uint4* src = reinterpret_cast<const uint4*>(a.Qeff + (tile * kChunk + i_out) * DK);
#pragma unroll
        for (int uu = 0; uu < DK / 8; ++uu) qt_r[uu] = src[uu];
      }
      if (!tc::mbar_wait(mma3_done, ex & 1)) { alive = false; break; }
      // ------------------------------------------- epilogue 3: outputs --
      // Results go to SW128 staging in the (now free) operand area and leave
      // by TMA bulk stores, so every global write is a whole tile row.
      tc::tc_fence_after();
      {
        const int m = 32 * q + lane;  // key channel row of Mp / Nc
        // half 0: Mp columns 0..127; half 1: Nc columns 0..DV-1 (TMEM 128..)
        const int ncols = half == 0 ? 128 : DV;
        uint8_t* stg = sm + (half == 0 ? C::OFF_SMP : C::OFF_SNC);
        for (int c0 = 0; c0 < ncols; c0 += 32) {
          uint32_t r[32], pw[16];
          tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, C::COL_MN + 128 * half + c0), r);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; e += 2) pw[e / 2] = tc::pack_bf16(__uint_as_float(r[e]), __uint_as_float(r[e + 1]));
          uint8_t* pnl = stg + (c0 >> 6) * 16384;
#pragma unroll
          for (int uu = 0; uu < 4; ++uu)
            *reinterpret_cast<uint4*>(pnl + sw_unit(m, ((c0 & 63) >> 3) + uu)) =
                make_uint4(pw[4 * uu], pw[4 * uu + 1], pw[4 * uu + 2], pw[4 * uu + 3]);
        }
        // token rows (M = 64 layout): half 0: Q_eff = Q~ - P W; half 1: O_part
        uint8_t* stt = sm + (half == 0 ? C::OFF_SQE : C::OFF_SOP);
        for (int c0 = 0; c0 < ncols; c0 += 32) {
          uint32_t r[32], pw[16];
          tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, C::COL_QO + 128 * half + c0), r);
          tc::tmem_wait_ld();
          if (lane < 16) {
            if (half == 0) {
              const uint32_t* qw = reinterpret_cast<const uint32_t*>(&qt_r[c0 / 8]);
#pragma unroll
              for (int e = 0; e < 32; e += 2)
                pw[e / 2] = tc::pack_bf16(bf16_lo_f(qw[e / 2]) - __uint_as_float(r[e]),
                                          bf16_hi_f(qw[e / 2]) - __uint_as_float(r[e + 1]));
            } else {
#pragma unroll
              for (int e = 0; e < 32; e += 2) pw[e / 2] = tc::pack_bf16(__uint_as_float(r[e]), __uint_as_float(r[e + 1]));
            }
            uint8_t* pnl = stt + (c0 >> 6) * 8192;
#pragma unroll
            for (int uu = 0; uu < 4; ++uu)
              *reinterpret_cast<uint4*>(pnl + sw_unit(i_out, ((c0 & 63) >> 3) + uu)) =
                  make_uint4(pw[4 * uu], pw[4 * uu + 1], pw[4 * uu + 2], pw[4 * uu + 3]);
          }
        }
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
      bar_compute();
      if (tid == 0) {
        tc::fence_async_global();  // Q~ went through global with generic stores
        const int rk = (int)tile * DK, rt = (int)tile * kChunk;
        for (int p = 0; p < 2; ++p) tc::tma_store_2d(&a.tm_Mp, sm + C::OFF_SMP + p * 16384, 64 * p, rk);
        for (int p = 0; p < DV / 64; ++p) tc::tma_store_2d(&a.tm_Nc, sm + C::OFF_SNC + p * 16384, 64 * p, rk);
        for (int p = 0; p < 2; ++p) tc::tma_store_2d(&a.tm_Qe, sm + C::OFF_SQE + p * 8192, 64 * p, rt);
        for (int p = 0; p < DV / 64; ++p) tc::tma_store_2d(&a.tm_Op, sm + C::OFF_SOP + p * 8192, 64 * p, rt);
        tc::tma_store_commit();
        if (a.ready) {
          // the factors must be in global memory before the flag says so
          tc::tma_store_wait_all();
          __threadfence();
          tc::st_release_gpu(a.ready + tile, 1);
        }
      }
      ++ex;
    }
    if (tid == 0) tc::tma_store_wait_all();
    if (!alive) {
      atomicExch(a.status, 8);
      vflag[0] = 1;
    }
    // release the UMMA warp
    vflag[1] = 1;
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(ops_ready);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

template <int DV>
__global__ void __launch_bounds__(PrepTcCfg<DV>::THREADS, 1)
prep_tc_kernel(const __grid_constant__ PrepTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  prep_tc_cta<DV>(a, sm, blockIdx.x, gridDim.x);
}

}  // namespace gdn2
