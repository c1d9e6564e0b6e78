// prep_tc.cuh -- gate preparation + intra-chunk WY + the chunk's affine state
// map on the tensor cores (bf16 I/O, dk = 128, dv in {64, 128}).
//
// Persistent CTAs walk a list of (chunk, head) tasks.  Warp roles:
//   warp 8      TMA producer: takes the tasks, streams each task's inputs
//               in four 32-channel slices through a 3-slot ring that runs
//               ahead across tasks, and puts the task id and its chunk's
//               length beside each slice (nobody else looks the chunk up);
//   warp 10     scan: per slice, the in-chunk cumulative sum g of log_alpha,
//               written in place as g - g_r, the per-channel constants
//               exp(g_r), exp(g_n - g_r), exp(g_n), and the decay-range check;
//   warp 9      UMMA issue (one elected lane);
//   warps 0-7   build the operands of each slice, then run the epilogues and
//               the triangular solve of the task;
//   warp 11     output stores (one lane): takes each task's staged tiles,
//               stores them by TMA, frees the staging for the next task's
//               builds once read, and publishes the task's ready flag once
//               its stores are complete, off the compute warps' path.
// Per chunk of n <= 64 tokens (page "Gated DeltaNet-2：将擦除与写入分开",
// sections "在两个维度上独立控制" and "词元路径与并行训练"; the algebra is the
// recurrence unrolled over one chunk, written as products):
//
//  1. Gate prep (fp32), with the decay folded in around one reference token
//     r = 32 of the chunk:
//        E^_i = b_i k_i exp(g_i - g_r),  Q^_i = q_i exp(g_i - g_r),
//        K^_j = k_j exp(g_r - g_j),      Z_i = w_i v_i.
//     For j <= i the product of the two factors is exp(g_i - g_j) <= 1; each
//     factor alone stays inside exp(+-60) as long as no 32-token stretch of a
//     channel decays by more than 60 nats (which keeps every fp32 product
//     below the accumulator's range).  A chunk that breaks this bound is
//     handed back for the exact fp32 kernel (prep_fixup_kernel).  The other
//     decayed operands are the same tensors scaled per channel,
//        E~ = E^ diag(exp(g_r)),  Q~ = Q^ diag(exp(g_r)),
//        Kbar = K^ diag(exp(g_n - g_r)),
//     so they are never built: exp(g_n - g_r) scales the rows of R in an
//     epilogue, and exp(g_r), a column scale of Mp and of Q_eff, is stored
//     beside them (colscale) and applied by the walk to the rows of the state
//     operand (Mp S = Mp' (diag(exp(g_r)) S), and likewise Q_eff S).
//  2. UMMA 1, accumulated slice by slice as the operands are built:
//     [E^; Q^] . K^T (M = 128, N = 64, K = 128) -> A (strictly lower part of
//     rows 0..63) and P (lower part with diagonal, rows 64..127).
//  3. T = (I + A)^-1 in fp32 on the CUDA cores: the four 16 x 16 diagonal
//     blocks by forward substitution, then two levels of block merges
//     [[T1, 0], [-T2 A21 T1, T2]] (16 -> 32 -> 64).  T is split into bf16
//     hi + lo, stored side by side as one operand (~16 bits of T kept).
//  4. UMMA 2: [R'_hi | R'_lo] = K^^T [T_hi | T_lo], [V_hi | V_lo] = P [T_hi | T_lo];
//     R = Kbar^T T = diag(exp(g_n - g_r)) R'.
//  5. UMMA 3: [Mp' | Nc] = R [E^ | Z], then [P W' | O_part] = [V; V] [E^ | Z]
//     (the 64 token rows twice, so they fill all four TMEM lane quarters);
//     the epilogue stages Mp', Nc, Q_eff' = Q^ - P W' and O_part (bf16) and
//     the store warp writes them by TMA; Mp = Mp' diag(exp(g_r)) and
//     Q_eff = Q_eff' diag(exp(g_r)).
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
  __nv_bfloat16* Qeff;   // [max_chunks, H, 64, 128]
  __nv_bfloat16* Opart;  // [max_chunks, H, 64, DV]
  __nv_bfloat16* Mp;     // [max_chunks, H, 128, 128]
  __nv_bfloat16* Nc;     // [max_chunks, H, 128, DV]
  float* gamma_last;     // [max_chunks, H, 128]
  float* colscale;       // [max_chunks, H, 128]: exp(g_r), the column scale of the stored Mp and Q_eff
  int32_t* fix_list;     // [0] = count, then c * H + h of handed-back chunks
  int* ready;            // optional [max_chunks * H], zeroed: 2 = factors written, 3 = handed back
  int* task_counter;     // optional: tasks taken dynamically (else static striding)
  int stop_at;           // with task_counter: a CTA given a later role stops taking tasks here
  int l2_prefetch;       // start each task's last input slice towards L2 when the task is taken
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
  static constexpr int PRODUCER_WARP = 8, MMA_WARP = 9, SCAN_WARP = 10, STORE_WARP = 11;
  static constexpr int THREADS = 12 * 32;
  // raw slot: la (-> g in place), b fp32 [64][32]; q, k bf16 [64][32]; v bf16 [64][VS]; w fp32 [64][VS].
  // The fp32 rows of 128 bytes (la, b, and w when VS = 32) arrive SW128-swizzled
  // (16-byte unit u of token row t at u ^ (t & 7)), so that the 8 lanes of a
  // float4 access, which span two token rows, hit distinct banks.
  static constexpr int OFF_LA = 0, OFF_B = 8192, OFF_Q = 16384, OFF_K = 20480, OFF_V = 24576;
  static constexpr int OFF_W = OFF_V + kChunk * VS * 2;
  static constexpr int SLOT_BYTES = OFF_W + kChunk * VS * 4;
  static constexpr int SLOT_STRIDE = 36864;
  static constexpr bool W_SWIZZLED = VS == 32;
  static constexpr int RING = NSLOT * SLOT_STRIDE;
  // Operands: four SW128 panel slots of 16 KiB (128 rows of 64 bf16), 1024-aligned.
  //   slot 0 / 1: rows 0..63 E^, rows 64..127 Q^ (channels 0..63 / 64..127)
  //   slot 2 / 3: rows 0..63 Z (value channels 0..63 / 64..127), rows 64..127 K^
  // so that [E^; Q^] (UMMA 1 A, M = 128), K^ (UMMA 1 B and, MN-major, the
  // UMMA 2 A operand) and [E^ | Z] (UMMA 3 B, MN-major) each have one panel
  // stride (16 KiB).
  static constexpr int OFF_X = RING;
  static constexpr int PANEL = 16384;
  static constexpr int OFF_Z = OFF_X + 2 * PANEL;
  static constexpr int OFF_KH = OFF_Z + 8192;
  // free area (48 KiB): solve scratch, then T, then R and V
  static constexpr int OFF_F = OFF_X + 4 * PANEL;
  static constexpr int OFF_BAR = OFF_F + 49152;
  static constexpr int LDA = 68;                // fp32 row stride of A and T: float4 rows, and a
  static constexpr int LDT = 68;                // column of 8 rows spans all 32 banks
  static constexpr int OFF_AS = OFF_F, OFF_TS = OFF_F + 17408, OFF_PB = OFF_F + 34816, OFF_XS = OFF_F + 43008;
  static constexpr int OFF_T = OFF_F;           // [T_hi | T_lo] MN-major SW128, over A once A is dead
  static constexpr int OFF_RB = OFF_F, OFF_VB = OFF_F + 16384;  // after UMMA 2: [R; V] K-major
  // output staging once UMMA 3 has read its operands (SW128 panels of 64
  // columns).  The first stores of a task (Mp, Nc) use the free area and
  // slot 2, the last ones (Q_eff, O_part) slots 1 and 3 only: the next
  // task's first two slices (which write slots 0 and 2) need only the first
  // stores to have left shared memory, its last two slices all of them.
  static constexpr int OFF_SMP0 = OFF_F, OFF_SMP1 = OFF_F + 16384;
  static constexpr int OFF_SNC0 = OFF_F + 32768, OFF_SNC1 = OFF_X + 2 * PANEL;
  static constexpr int OFF_SOP0 = OFF_X + 3 * PANEL, OFF_SOP1 = OFF_X + 3 * PANEL + 8192;
  static constexpr int OFF_SQE = OFF_X + PANEL;  // + p * 8192 (slot 1)
  static constexpr int OFF_QH = OFF_X + 8192;    // Q^, + p * PANEL
  static_assert(OFF_XS + 4096 <= OFF_BAR, "solve scratch fits in the free area");
  static_assert(OFF_VB + 16384 <= OFF_BAR, "the M = 128 read of V stays inside the free area");
  static_assert(64 * LDA * 4 <= OFF_TS - OFF_AS && 64 * LDT * 4 <= OFF_PB - OFF_TS, "A and T scratch");
  static constexpr int SMEM = 1024 + OFF_BAR + 3072;
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t COL_D1 = 0, COL_R = 64, COL_V = 192, COL_MN = 0, COL_QO = 256;
  static_assert(SLOT_BYTES <= SLOT_STRIDE, "slot fits");
  static_assert(SMEM <= 232448, "shared memory");
};

__device__ __forceinline__ void bar_compute() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ void bar_half(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

// byte offset of the 16-byte unit holding elements [8u, 8u+8) of row `row`
// in an SW128 panel (rows of 64 bf16)
__device__ __forceinline__ uint32_t sw_unit(uint32_t row, uint32_t u) { return row * 128u + ((u ^ (row & 7u)) << 4); }

__device__ __forceinline__ void store8(uint8_t* p, const uint32_t (&w)[8], int at) {
  *reinterpret_cast<uint4*>(p) = make_uint4(w[at], w[at + 1], w[at + 2], w[at + 3]);
}

__device__ __forceinline__ void load8f(const float* p, float (&v)[8]) {
  const float4 x = reinterpret_cast<const float4*>(p)[0], y = reinterpret_cast<const float4*>(p)[1];
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w; v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
}

// float index of channel c (0..31) of token row t in an SW128 fp32 tile
__device__ __forceinline__ int swf(int t, int c) { return t * 32 + ((((c >> 2) ^ (t & 7))) << 2) + (c & 3); }

// channels 8g .. 8g+7 of token row t of an SW128 fp32 tile (two 16-byte units)
__device__ __forceinline__ void load8f_sw(const float* tile, int t, int g, float (&v)[8]) {
  const float4 x = *reinterpret_cast<const float4*>(tile + t * 32 + (((2 * g) ^ (t & 7)) << 2));
  const float4 y = *reinterpret_cast<const float4*>(tile + t * 32 + (((2 * g + 1) ^ (t & 7)) << 2));
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w; v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
}

// `stopper`: this CTA takes no task once the shared counter has reached
// a.stop_at (it has another role to play after this one).
template <int DV>
__device__ void prep_tc_cta(const PrepTcArgs& a, uint8_t* sm, int cta_rank, int cta_count, bool stopper = false) {
  using C = PrepTcCfg<DV>;
  constexpr int DK = C::DK;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::OFF_BAR);  // [NSLOT] producer -> scan
  uint64_t* gready = full + C::NSLOT;                               // [NSLOT] scan -> build
  uint64_t* empty = gready + C::NSLOT;                              // [NSLOT] build -> producer
  uint64_t* built = empty + C::NSLOT;                               // [SLICES] build -> UMMA 1
  uint64_t* mma1_done = built + C::SLICES;
  uint64_t* t_ready = mma1_done + 1;
  uint64_t* mma2_done = t_ready + 1;
  uint64_t* rv_ready = mma2_done + 1;
  uint64_t* mma3_done = rv_ready + 1;
  uint64_t* fin = mma3_done + 1;
  uint64_t* mma2a_done = fin + 1;   // the R half of UMMA 2
  uint64_t* mma3a_done = mma2a_done + 1;  // the [Mp' | Nc] half of UMMA 3
  uint64_t* st_a = mma3a_done + 1;  // Mp and Nc staged (both half leaders)
  uint64_t* st_b = st_a + 1;        // Q_eff and O_part staged
  uint64_t* rd_a = st_b + 1;        // the store warp: Mp / Nc staging read
  uint64_t* rd_b = rd_a + 1;        // the store warp: all staging read
  uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + C::OFF_BAR + 256);
  int* s_flag = reinterpret_cast<int*>(tslot + 1);    // [0] abort, [1] done
  int* slot_task = s_flag + 2;                        // [NSLOT] task id of the slot's slice
  int* slot_skip = slot_task + C::NSLOT;              // [NSLOT] decay range exceeded
  int* s_store = slot_skip + C::NSLOT;                // [2] tile being stored (-1: none left), skip
  int* slot_len = s_store + 2;                        // [NSLOT] valid tokens of the slot's chunk
  float* s_enr = reinterpret_cast<float*>(sm + C::OFF_BAR + 512);  // [2][128] exp(g_n - g_r), by task parity

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H;
  const int ntasks = a.map.chunk_off[a.map.N] * H;

  if (tid == 0) {
    for (int s = 0; s < C::NSLOT; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&gready[s], 1);
      tc::mbar_init(&empty[s], C::COMPUTE_WARPS);
    }
    for (int s = 0; s < C::SLICES; ++s) tc::mbar_init(&built[s], C::COMPUTE_WARPS);
    tc::mbar_init(mma1_done, 1);
    tc::mbar_init(t_ready, C::COMPUTE_WARPS);
    tc::mbar_init(mma2_done, 1);
    tc::mbar_init(rv_ready, C::COMPUTE_WARPS);
    tc::mbar_init(mma3_done, 1);
    tc::mbar_init(fin, 1);
    tc::mbar_init(mma2a_done, 1);
    tc::mbar_init(mma3a_done, 1);
    tc::mbar_init(st_a, 2);
    tc::mbar_init(st_b, 1);
    tc::mbar_init(rd_a, 1);
    tc::mbar_init(rd_b, 1);
    s_flag[0] = s_flag[1] = 0;
    tc::fence_mbar_init();
  }
  if (warp == C::MMA_WARP) {
    tc::tmem_alloc(tslot, C::TMEM_COLS);
    // a CTA with a later role allocates again, so it keeps the permit
    if (!stopper) tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tslot;
  volatile int* vflag = s_flag;
  volatile int* vtask = slot_task;
  volatile int* vlen = slot_len;

  if (warp == C::PRODUCER_WARP) {
    // ---------------------------------------------------- input producer --
    // Takes tasks (dynamic counter or static stride) and streams the four
    // input slices of each through the ring, the task id beside each slice.
    // A slot holding task id -1 (no data) ends the CTA's work.
    if (lane == 0) {
      int gs = 0, k_static = 0;
      bool ok = true;
      for (bool more = true; more && ok;) {
        int task;
        if (a.task_counter) {
          task = (stopper && *reinterpret_cast<volatile int*>(a.task_counter) >= a.stop_at)
                     ? ntasks : atomicAdd(a.task_counter, 1);
        }
        else task = cta_rank + cta_count * (k_static++);
        if (task >= ntasks) task = -1;
        int h = 0, t0 = 0, tlen = 0;
        if (task >= 0) {
          h = task % H;
          const ChunkPos cp = chunk_pos(a.map, task / H);
          t0 = cp.t0;
          tlen = cp.len;
        }
        if (task >= 0 && a.l2_prefetch) {
          // the last slice is loaded only once this task's first slice has
          // been built (three slots, four slices): start it towards L2 now.
          // (Beside the walk in the fused launch this costs more than it
          // saves, and is left off there.)
          constexpr int s3 = C::SLICES - 1;
          tc::tma_prefetch_3d(&a.tm_la, C::KS * s3, h, t0);
          tc::tma_prefetch_3d(&a.tm_b, C::KS * s3, h, t0);
          tc::tma_prefetch_3d(&a.tm_q, C::KS * s3, h, t0);
          tc::tma_prefetch_3d(&a.tm_k, C::KS * s3, h, t0);
          tc::tma_prefetch_3d(&a.tm_v, C::VS * s3, h, t0);
          tc::tma_prefetch_3d(&a.tm_w, C::VS * s3, h, t0);
        }
        const int nsl = task < 0 ? 1 : C::SLICES;
        for (int s = 0; s < nsl; ++s, ++gs) {
          const int slot = gs % C::NSLOT, use = gs / C::NSLOT;
          if (use > 0 && !tc::mbar_wait(&empty[slot], (use - 1) & 1)) { ok = false; break; }
          if (vflag[0]) { more = false; break; }
          vtask[slot] = task;
          vlen[slot] = tlen;  // the consumers need not look the chunk up again
          if (task < 0) {
            tc::mbar_arrive(&full[slot]);
            more = false;
            ++gs;
            break;
          }
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
  } else if (warp == C::SCAN_WARP) {
    // -------------------------------------------------------------- scan --
    // g_t = sum of log_alpha over tokens <= t of the chunk (tokens past its
    // end count as 0), written over log_alpha as g_t - g_r.
    int s_in = 0, tpar = 0;
    for (int gs = 0;; ++gs) {
      const int slot = gs % C::NSLOT, use = gs / C::NSLOT;
      if (!tc::mbar_wait(&full[slot], use & 1)) {
        atomicExch(a.status, 8);
        vflag[0] = 1;
        break;
      }
      const int task = vtask[slot];
      if (task >= 0 && !vflag[0]) {
        const int c = task / H;
        const int len = vlen[slot];
        const size_t tile = (size_t)c * H + task % H;
        float* la = reinterpret_cast<float*>(sm + slot * C::SLOT_STRIDE + C::OFF_LA);
        // lane = (token quarter tq, channel group cg): tokens 16 tq .. 16 tq + 15
        // of channels 4 cg .. 4 cg + 3, one 16-byte unit of each SW128 row
        const int tq = lane >> 3, cg = lane & 7;
        auto unit = [&](int i) {
          const int t = 16 * tq + i;
          return reinterpret_cast<float4*>(la + t * 32 + ((cg ^ (t & 7)) << 2));
        };
        float4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = *unit(i);
        // running sums within the quarter (tokens past the chunk's end add 0)
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (16 * tq + i < len) {
            acc.x += v[i].x; acc.y += v[i].y; acc.z += v[i].z; acc.w += v[i].w;
          }
          v[i] = acc;
        }
        // the quarters' offsets: inclusive scan of the totals over tq, then
        // the previous quarter's value
        auto shfl_up4 = [](float4 a, int d) {
          return make_float4(__shfl_up_sync(0xffffffffu, a.x, d), __shfl_up_sync(0xffffffffu, a.y, d),
                             __shfl_up_sync(0xffffffffu, a.z, d), __shfl_up_sync(0xffffffffu, a.w, d));
        };
        auto shfl4 = [](float4 a, int src) {
          return make_float4(__shfl_sync(0xffffffffu, a.x, src), __shfl_sync(0xffffffffu, a.y, src),
                             __shfl_sync(0xffffffffu, a.z, src), __shfl_sync(0xffffffffu, a.w, src));
        };
        float4 inc = acc;
        {
          const float4 y = shfl_up4(inc, 8);
          if (tq >= 1) { inc.x += y.x; inc.y += y.y; inc.z += y.z; inc.w += y.w; }
          const float4 z = shfl_up4(inc, 16);
          if (tq >= 2) { inc.x += z.x; inc.y += z.y; inc.z += z.z; inc.w += z.w; }
        }
        float4 off = shfl_up4(inc, 8);
        if (tq == 0) off = make_float4(0.f, 0.f, 0.f, 0.f);
        // g at token 0 (quarter 0), r = 32 (quarter 2) and 63 (quarter 3)
        const float4 first = make_float4(v[0].x + off.x, v[0].y + off.y, v[0].z + off.z, v[0].w + off.w);
        const float4 last = make_float4(v[15].x + off.x, v[15].y + off.y, v[15].z + off.z, v[15].w + off.w);
        const float4 g0 = shfl4(first, cg), gr = shfl4(first, 16 + cg), gn = shfl4(last, 24 + cg);
        const bool bad = (g0.x - gr.x > 60.f) || (g0.y - gr.y > 60.f) || (g0.z - gr.z > 60.f) ||
                         (g0.w - gr.w > 60.f) || (gr.x - gn.x > 60.f) || (gr.y - gn.y > 60.f) ||
                         (gr.z - gn.z > 60.f) || (gr.w - gn.w > 60.f);
        // what the build needs: x_t = g_t - g_r, over log_alpha
#pragma unroll
        for (int i = 0; i < 16; ++i)
          *unit(i) = make_float4((v[i].x + off.x) - gr.x, (v[i].y + off.y) - gr.y, (v[i].z + off.z) - gr.z,
                                 (v[i].w + off.w) - gr.w);
        if (tq == 0) {
          const int ch = C::KS * s_in + 4 * cg;
          *reinterpret_cast<float4*>(s_enr + tpar * DK + ch) =
              make_float4(__expf(gn.x - gr.x), __expf(gn.y - gr.y), __expf(gn.z - gr.z), __expf(gn.w - gr.w));
          *reinterpret_cast<float4*>(a.gamma_last + tile * DK + ch) =
              make_float4(expf(gn.x), expf(gn.y), expf(gn.z), expf(gn.w));
          // published with the chunk's other factors: the store warp's fence
          // and release of the ready flag come after these writes through the
          // CTA's mbarrier chain (releases are cumulative)
          *reinterpret_cast<float4*>(a.colscale + tile * DK + ch) =
              make_float4(__expf(gr.x), __expf(gr.y), __expf(gr.z), __expf(gr.w));
        }
        const unsigned any = __ballot_sync(0xffffffffu, bad);
        if (lane == 0) slot_skip[slot] = any != 0u;
        s_in = (s_in + 1) & (C::SLICES - 1);
        if (s_in == 0) tpar ^= 1;
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&gready[slot]);
      if (task < 0 || vflag[0]) break;
    }
  } else if (warp == C::MMA_WARP) {
    // ------------------------------------------------------- UMMA issue --
    if (lane == 0) {
      const uint32_t X = tc::smem_u32(sm + C::OFF_X), KH = tc::smem_u32(sm + C::OFF_KH);
      const uint32_t TT = tc::smem_u32(sm + C::OFF_T), PB = tc::smem_u32(sm + C::OFF_PB);
      const uint32_t RB = tc::smem_u32(sm + C::OFF_RB), VB = tc::smem_u32(sm + C::OFF_VB);
      const uint32_t SW = tc::kLayoutSW128;
      constexpr uint32_t id1 = tc::idesc_bf16(128, 64, false, false);
      constexpr uint32_t idR = tc::idesc_bf16(128, 128, true, true);
      constexpr uint32_t idV = tc::idesc_bf16(64, 128, false, true);
      constexpr uint32_t idM = tc::idesc_bf16(128, 128 + DV, false, true);
      // M = 128 over [V; V] (epilogue 2 writes V twice): the 64 token rows
      // land in lanes 0..63 and again in 64..127, so all four TMEM lane
      // quarters hold them and all eight epilogue warps share the token rows
      constexpr uint32_t idQ = tc::idesc_bf16(128, 128 + DV, false, true);
      bool ok = true;
      for (int ex = 0; ok; ++ex) {
        // UMMA 1, two K-steps of 16 channels per slice as the slices are built
        for (int s = 0; s < C::SLICES; ++s) {
          if (!tc::mbar_wait(&built[s], ex & 1) || vflag[0]) { ok = false; break; }
          if (vflag[1]) break;
          tc::tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const uint32_t k = 2 * s + kk, ko = k >> 2, kb = (k & 3) * 32;
            tc::umma_f16(tbase + C::COL_D1, tc::sdesc(X + ko * C::PANEL + kb, 16, 1024, SW),
                         tc::sdesc(KH + ko * C::PANEL + kb, 16, 1024, SW), id1, k > 0);
          }
        }
        if (!ok || vflag[1]) break;
        tc::umma_commit(mma1_done);
        if (!tc::mbar_wait(t_ready, ex & 1) || vflag[0]) break;
        tc::tc_fence_after();
        // R first, committed on its own: its epilogue starts while V runs
#pragma unroll
        for (int s = 0; s < 4; ++s)
          tc::umma_f16(tbase + C::COL_R, tc::sdesc(KH + s * 2048, C::PANEL, 1024, SW),
                       tc::sdesc(TT + s * 2048, 8192, 1024, SW), idR, s > 0);
        tc::umma_commit(mma2a_done);
#pragma unroll
        for (int s = 0; s < 4; ++s)
          tc::umma_f16(tbase + C::COL_V, tc::sdesc(PB + s * 32, 16, 1024, SW), tc::sdesc(TT + s * 2048, 8192, 1024, SW),
                       idV, s > 0);
        tc::umma_commit(mma2_done);
        if (!tc::mbar_wait(rv_ready, ex & 1) || vflag[0]) break;
        tc::tc_fence_after();
        // [Mp' | Nc] first (its epilogue starts while the token rows run)
#pragma unroll
        for (int s = 0; s < 4; ++s)
          tc::umma_f16(tbase + C::COL_MN, tc::sdesc(RB + s * 32, 16, 1024, SW), tc::sdesc(X + s * 2048, C::PANEL, 1024, SW),
                       idM, s > 0);
        tc::umma_commit(mma3a_done);
#pragma unroll
        for (int s = 0; s < 4; ++s)
          tc::umma_f16(tbase + C::COL_QO, tc::sdesc(VB + s * 32, 16, 1024, SW), tc::sdesc(X + s * 2048, C::PANEL, 1024, SW),
                       idQ, s > 0);
        tc::umma_commit(mma3_done);
      }
      // nothing of ours is left in the tensor pipe when TMEM is released
      tc::umma_commit(fin);
      tc::mbar_wait(fin, 0);
    }
  } else if (warp == C::STORE_WARP) {
    // ----------------------------------------------------------- stores --
    // Per task: the Mp / Nc tiles once both half leaders have staged them,
    // the Q_eff / O_part tiles once the epilogue is done; the staging is
    // handed back as soon as the stores have read it, and the task's ready
    // flag (2 = factors written) is raised once its stores are complete.
    if (lane == 0) {
      volatile int* vst = s_store;
      bool ok = true;
      auto publish = [&](int t) {
        tc::fence_async_global();
        __threadfence();
        tc::red_add_release_gpu(a.ready + t, 2);
      };
      for (int ex = 0;; ++ex) {
        if (!tc::mbar_wait(st_a, ex & 1)) { ok = false; break; }
        const int tile = vst[0];
        const bool skip = vst[1] != 0;
        if (tile < 0) break;
        if (!skip) {
          const int rk = tile * DK;
          tc::tma_store_2d(&a.tm_Mp, sm + C::OFF_SMP0, 0, rk);
          tc::tma_store_2d(&a.tm_Mp, sm + C::OFF_SMP1, 64, rk);
          tc::tma_store_2d(&a.tm_Nc, sm + C::OFF_SNC0, 0, rk);
          if (DV == 128) tc::tma_store_2d(&a.tm_Nc, sm + C::OFF_SNC1, 64, rk);
          tc::tma_store_commit();
        }
        if (!tc::mbar_wait(st_b, ex & 1)) { ok = false; break; }
        if (!skip) {
          const int rt = tile * kChunk;
          for (int p = 0; p < 2; ++p) tc::tma_store_2d(&a.tm_Qe, sm + C::OFF_SQE + p * 8192, 64 * p, rt);
          for (int p = 0; p < DV / 64; ++p) tc::tma_store_2d(&a.tm_Op, sm + C::OFF_SOP0 + p * 8192, 64 * p, rt);
          tc::tma_store_commit();
        }
        tc::tma_store_wait_read_but_newest();
        tc::mbar_arrive(rd_a);
        tc::tma_store_wait_read();
        tc::mbar_arrive(rd_b);
        if (!skip && a.ready) {
          // the compute warps are building the next task by now and need
          // nothing more from this warp until its epilogue
          tc::tma_store_wait_all();
          publish(tile);
        }
      }
      tc::tma_store_wait_all();
      if (!ok) {
        atomicExch(a.status, 8);
        vflag[0] = 1;
      }
    }
  } else {
    // ----------------------------------------------------------- compute --
    const int q = warp & 3, half = warp >> 2;
    float* AS = reinterpret_cast<float*>(sm + C::OFF_AS);
    float* TS = reinterpret_cast<float*>(sm + C::OFF_TS);
    float* XS = reinterpret_cast<float*>(sm + C::OFF_XS);
    int gs = 0;
    bool alive = true;
    int ex = 0;
    for (;; ++ex) {
      int task = -1, len = 0;
      size_t tile = 0;
      bool skip = false;
      // ------------------------------------------------------ slices --
      for (int s = 0; s < C::SLICES; ++s, ++gs) {
        const int slot = gs % C::NSLOT;
        if (!tc::mbar_wait(&gready[slot], (gs / C::NSLOT) & 1)) { alive = false; break; }
        task = vtask[slot];
        if (task < 0 || vflag[0]) break;
        if (s == 0) {
          const int c = task / H;
          len = vlen[slot];
          tile = (size_t)c * H + task % H;
          // the previous task's first stores (Mp, Nc) have left slot 2
          if (ex > 0 && !tc::mbar_wait(rd_a, (ex - 1) & 1)) { alive = false; break; }
        } else if (s == 2) {
          // and its last ones (Q_eff, O_part) slots 1 and 3
          if (ex > 0 && !tc::mbar_wait(rd_b, (ex - 1) & 1)) { alive = false; break; }
        }
        skip |= reinterpret_cast<volatile int*>(slot_skip)[slot] != 0;
        uint8_t* d = sm + slot * C::SLOT_STRIDE;
        const float* g = reinterpret_cast<const float*>(d + C::OFF_LA);
        // operands for token i, key channels cc0 .. cc0 + 7
        const int i = tid >> 2, gq = tid & 3, cl = 8 * gq, cc0 = C::KS * s + cl;
        const bool live = i < len;
        {
          float gi[8], bb[8];   // gi: g_i - g_r
          load8f_sw(g, i, gq, gi);
          load8f_sw(reinterpret_cast<const float*>(d + C::OFF_B), i, gq, bb);
          const uint4 kraw = *reinterpret_cast<const uint4*>(d + C::OFF_K + (i * 32 + cl) * 2);
          const uint4 qraw = *reinterpret_cast<const uint4*>(d + C::OFF_Q + (i * 32 + cl) * 2);
          const uint32_t kw[4] = {kraw.x, kraw.y, kraw.z, kraw.w};
          const uint32_t qw[4] = {qraw.x, qraw.y, qraw.z, qraw.w};
          uint32_t eh[8], kh[4];
#pragma unroll
          for (int p = 0; p < 4; ++p) {
            float o_eh[2], o_qh[2], o_kh[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int m = 2 * p + e;
              const float kv = live ? (e ? bf16_hi_f(kw[p]) : bf16_lo_f(kw[p])) : 0.f;
              const float qv = live ? (e ? bf16_hi_f(qw[p]) : bf16_lo_f(qw[p])) : 0.f;
              const float bv = live ? bb[m] : 0.f;
              const float x = gi[m];
              const float E = __expf(x), F = __expf(-x);
              o_eh[e] = bv * kv * E;
              o_qh[e] = qv * E;
              o_kh[e] = kv * F;
            }
            eh[p] = tc::pack_bf16(o_eh[0], o_eh[1]);
            eh[4 + p] = tc::pack_bf16(o_qh[0], o_qh[1]);
            kh[p] = tc::pack_bf16(o_kh[0], o_kh[1]);
          }
          const uint32_t pnl = cc0 >> 6, u = (cc0 & 63) >> 3;
          store8(sm + C::OFF_X + pnl * C::PANEL + sw_unit(i, u), eh, 0);
          store8(sm + C::OFF_X + pnl * C::PANEL + sw_unit(64 + i, u), eh, 4);
          *reinterpret_cast<uint4*>(sm + C::OFF_KH + pnl * C::PANEL + sw_unit(i, u)) = make_uint4(kh[0], kh[1], kh[2], kh[3]);
        }
        {
          // Z = w * v for value channels vc0 .. vc0 + VS/4 - 1 (right after E~)
          constexpr int VPT = C::VS / 4;
          const int vl = VPT * gq, vc0 = C::VS * s + vl;
          float ww[VPT];
          uint32_t vw[VPT / 2];
          {
            const float* wt = reinterpret_cast<const float*>(d + C::OFF_W);
            if constexpr (C::W_SWIZZLED) {
              load8f_sw(wt, i, gq, *reinterpret_cast<float(*)[8]>(ww));
            } else {
              const float4* w4 = reinterpret_cast<const float4*>(wt + i * C::VS + vl);
#pragma unroll
              for (int hh = 0; hh < VPT / 4; ++hh) {
                const float4 x = w4[hh];
                ww[4 * hh] = x.x; ww[4 * hh + 1] = x.y; ww[4 * hh + 2] = x.z; ww[4 * hh + 3] = x.w;
              }
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
          uint8_t* zdst = sm + C::OFF_Z + (vc0 >> 6) * C::PANEL + sw_unit(i, (vc0 & 63) >> 3) + (vc0 & 7) * 2;
          if constexpr (VPT == 8) *reinterpret_cast<uint4*>(zdst) = make_uint4(zw[0], zw[1], zw[2], zw[3]);
          else *reinterpret_cast<uint2*>(zdst) = make_uint2(zw[0], zw[1]);
        }
        tc::fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          tc::mbar_arrive(&empty[slot]);
          tc::mbar_arrive(&built[s]);
        }
      }
      if (!alive || task < 0 || vflag[0]) break;
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
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(AS + i * C::LDA + j0 + e) =
                make_float4(j0 + e < i ? __uint_as_float(r[e]) : 0.f, j0 + e + 1 < i ? __uint_as_float(r[e + 1]) : 0.f,
                            j0 + e + 2 < i ? __uint_as_float(r[e + 2]) : 0.f, j0 + e + 3 < i ? __uint_as_float(r[e + 3]) : 0.f);
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
      // (a) diagonal 16 x 16 blocks by forward substitution (warps 0-3,
      //     lane l < 16 owns column l of block `warp`); warps 4-7 zero the
      //     two upper blocks the merges below read.
      if (warp < 4) {
        const int I = warp, l = lane;
        float t[16];
        t[0] = l == 0 ? 1.f : 0.f;
#pragma unroll
        for (int i = 1; i < 16; ++i) {
          float arow[16];
          load8f(AS + (16 * I + i) * C::LDA + 16 * I, *reinterpret_cast<float(*)[8]>(arow));
          load8f(AS + (16 * I + i) * C::LDA + 16 * I + 8, *reinterpret_cast<float(*)[8]>(arow + 8));
          // t[m] = 0 for m < l, so the sum may run over every m < i
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int m = 0; m < i; ++m) {
            if (m & 1) s1 = fmaf(arow[m], t[m], s1);
            else s0 = fmaf(arow[m], t[m], s0);
          }
          t[i] = i < l ? 0.f : (i == l ? 1.f : -(s0 + s1));
        }
        if (l < 16)
#pragma unroll
          for (int i = 0; i < 16; ++i) TS[(16 * I + i) * C::LDT + 16 * I + l] = t[i];
      } else {
        const int z = tid - 128;  // 0..127: two 16 x 16 blocks, 4 values each
        const int blk = z >> 6, rr = (z >> 2) & 15, cc = 4 * (z & 3);
        const int r0 = 32 * blk + rr, c0 = 32 * blk + 16 + cc;
        *reinterpret_cast<float4*>(TS + r0 * C::LDT + c0) = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      bar_compute();
      // (b) 16 -> 32: blocks (1,0) and (3,2); warps 0-3 and 4-7.
      {
        const int m = warp >> 2, ba = 2 * m, bb = 2 * m + 1;
        const int t = tid & 127, r = t >> 3, c = 2 * (t & 7);
        float* X2 = XS + m * 256;
        float x0 = 0.f, x1 = 0.f;
        float arow[16];
        load8f(AS + (16 * bb + r) * C::LDA + 16 * ba, *reinterpret_cast<float(*)[8]>(arow));
        load8f(AS + (16 * bb + r) * C::LDA + 16 * ba + 8, *reinterpret_cast<float(*)[8]>(arow + 8));
        const float* tcol = TS + (16 * ba) * C::LDT + 16 * ba + c;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float2 tv = *reinterpret_cast<const float2*>(tcol + k * C::LDT);
          x0 = fmaf(arow[k], tv.x, x0);
          x1 = fmaf(arow[k], tv.y, x1);
        }
        *reinterpret_cast<float2*>(X2 + r * 16 + c) = make_float2(x0, x1);
        bar_half(2 + m);
        float y0 = 0.f, y1 = 0.f;
        float trow[16];
        load8f(TS + (16 * bb + r) * C::LDT + 16 * bb, *reinterpret_cast<float(*)[8]>(trow));
        load8f(TS + (16 * bb + r) * C::LDT + 16 * bb + 8, *reinterpret_cast<float(*)[8]>(trow + 8));
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float2 xv = *reinterpret_cast<const float2*>(X2 + k * 16 + c);
          y0 = fmaf(trow[k], xv.x, y0);
          y1 = fmaf(trow[k], xv.y, y1);
        }
        *reinterpret_cast<float2*>(TS + (16 * bb + r) * C::LDT + 16 * ba + c) = make_float2(-y0, -y1);
      }
      bar_compute();
      // (c) 32 -> 64: block (1,0) of 32 x 32 blocks, T21 = -T22 (A21 T11).
      // Both products skip the zero triangle of their T factor, with the
      // triangle's bound uniform per warp: X = A21 T11 by (lane = row r,
      // warp = columns 4w..4w+3, k >= 4w), then T21 by (lane = column,
      // warp = rows 4w..4w+3, k <= 4w+3).  A row of A21 and of T22 is read
      // as float4 by one lane; the T11 / X values every lane needs are
      // broadcasts.
      {
        const int r = lane, c0 = 4 * warp;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int k0 = c0; k0 < 32; k0 += 4) {
          const float4 av = *reinterpret_cast<const float4*>(AS + (32 + r) * C::LDA + k0);
          const float a4[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float4 tv = *reinterpret_cast<const float4*>(TS + (k0 + k) * C::LDT + c0);
            x.x = fmaf(a4[k], tv.x, x.x); x.y = fmaf(a4[k], tv.y, x.y);
            x.z = fmaf(a4[k], tv.z, x.z); x.w = fmaf(a4[k], tv.w, x.w);
          }
        }
        *reinterpret_cast<float4*>(XS + r * 32 + c0) = x;
        bar_compute();
        const int col = lane, r0 = 4 * warp;
        float y[4] = {0.f, 0.f, 0.f, 0.f};
        for (int k0 = 0; k0 <= r0; k0 += 4) {
          float xv[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) xv[k] = XS[(k0 + k) * 32 + col];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 tv = *reinterpret_cast<const float4*>(TS + (32 + r0 + i) * C::LDT + 32 + k0);
            y[i] = fmaf(tv.x, xv[0], y[i]); y[i] = fmaf(tv.y, xv[1], y[i]);
            y[i] = fmaf(tv.z, xv[2], y[i]); y[i] = fmaf(tv.w, xv[3], y[i]);
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) TS[(32 + r0 + i) * C::LDT + col] = -y[i];
      }
      bar_compute();
      // T -> [T_hi | T_lo], MN-major SW128 (row i, 64 columns j per panel);
      // entries above the diagonal are zero.
      {
        const int i = tid >> 2, j0 = 16 * (tid & 3);
        uint32_t hw[8], lw[8];
        float tv[16];
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 t4 = *reinterpret_cast<const float4*>(TS + i * C::LDT + j0 + e);
          tv[e] = j0 + e <= i ? t4.x : 0.f;
          tv[e + 1] = j0 + e + 1 <= i ? t4.y : 0.f;
          tv[e + 2] = j0 + e + 2 <= i ? t4.z : 0.f;
          tv[e + 3] = j0 + e + 3 <= i ? t4.w : 0.f;
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
      if (!tc::mbar_wait(mma2a_done, ex & 1)) { alive = false; break; }
      // ------------- epilogue 2: R = exp(g_n - g_r) (R'_hi + R'_lo), V = V_hi + V_lo -> bf16 --
      tc::tc_fence_after();
      {
        const int j0 = 32 * half;
        const int m = 32 * q + lane;
        const float sc = s_enr[(ex & 1) * DK + m];
        uint32_t rh[32], rl[32], pw[16];
        tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, C::COL_R + j0), rh);
        tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, C::COL_R + 64 + j0), rl);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 2)
          pw[e / 2] = tc::pack_bf16(sc * (__uint_as_float(rh[e]) + __uint_as_float(rl[e])),
                                    sc * (__uint_as_float(rh[e + 1]) + __uint_as_float(rl[e + 1])));
        // R goes over T, which the V half of UMMA 2 reads
        if (!tc::mbar_wait(mma2_done, ex & 1)) alive = false;
        tc::tc_fence_after();
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
          // and again as rows 64..127, so the token rows of the M = 128
          // product below fill all four TMEM lane quarters
#pragma unroll
          for (int uu = 0; uu < 4; ++uu) {
            const uint4 v4 = make_uint4(pw[4 * uu], pw[4 * uu + 1], pw[4 * uu + 2], pw[4 * uu + 3]);
            *reinterpret_cast<uint4*>(sm + C::OFF_VB + sw_unit(i, (j0 >> 3) + uu)) = v4;
            *reinterpret_cast<uint4*>(sm + C::OFF_VB + 8192 + sw_unit(i, (j0 >> 3) + uu)) = v4;
          }
        }
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(rv_ready);
      if (!alive || !tc::mbar_wait(mma3a_done, ex & 1)) { alive = false; break; }
      // ------------------------------------------- epilogue 3: outputs --
      // Results go to SW128 staging in the (now free) operand area and leave
      // by TMA bulk stores, so every global write is a whole tile row.
      tc::tc_fence_after();
      {
        const int m = 32 * q + lane;  // key channel row of Mp / Nc
        // half 0: Mp' columns 0..127; half 1: Nc columns 0..DV-1 (TMEM 128..)
        const uint32_t colb = C::COL_MN + 128 * half;
        auto stage = [&](uint8_t* pnl, const uint32_t (&pk)[32]) {
#pragma unroll
          for (int uu = 0; uu < 8; ++uu)
            *reinterpret_cast<uint4*>(pnl + sw_unit(m, uu)) =
                make_uint4(pk[4 * uu], pk[4 * uu + 1], pk[4 * uu + 2], pk[4 * uu + 3]);
        };
        uint32_t r0[32], r1[32], pk[32];
        tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, colb), r0);
        tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, colb + 32), r1);
        tc::tmem_wait_ld_regs(r0);
        tc::tmem_wait_ld_regs(r1);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          pk[e] = tc::pack_bf16(__uint_as_float(r0[2 * e]), __uint_as_float(r0[2 * e + 1]));
          pk[16 + e] = tc::pack_bf16(__uint_as_float(r1[2 * e]), __uint_as_float(r1[2 * e + 1]));
        }
        const bool second = half == 0 || DV == 128;
        if (second) {
          // the second 64 columns load while the first are staged
          tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, colb + 64), r0);
          tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, colb + 96), r1);
        }
        stage(sm + (half == 0 ? C::OFF_SMP0 : C::OFF_SNC0), pk);
        if (second) {
          tc::tmem_wait_ld_regs(r0);
          tc::tmem_wait_ld_regs(r1);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            pk[e] = tc::pack_bf16(__uint_as_float(r0[2 * e]), __uint_as_float(r0[2 * e + 1]));
            pk[16 + e] = tc::pack_bf16(__uint_as_float(r1[2 * e]), __uint_as_float(r1[2 * e + 1]));
          }
          // the second panels (over V and Z) wait for the token-row half of
          // UMMA 3, which reads both
          if (!tc::mbar_wait(mma3_done, ex & 1)) alive = false;
          stage(sm + (half == 0 ? C::OFF_SMP1 : C::OFF_SNC1), pk);
        }
      }
      // this half's tile (Mp or Nc) is staged: it leaves (store warp) while
      // the token rows are finished
      tc::fence_async_smem();
      bar_half(2 + half);
      if ((tid & 127) == 0) {
        if (tid == 0) {
          s_store[0] = (int)tile;
          s_store[1] = skip ? 1 : 0;
        }
        tc::mbar_arrive(st_a);
      }
      {
        // token rows: lane quarters 0, 1 form Q_eff' = Q^ - P W' (columns
        // 0..127, in slot 1 from Q^ in slot 0 / 1), lane quarters 2, 3
        // (the same rows again) O_part (columns 128..); each half takes one
        // 64-column panel.
        const bool qside = q < 2;
        if (qside || DV == 128 || half == 0) {
          const int i_out = 32 * (q & 1) + lane;
          uint8_t* pnl = sm + (qside ? C::OFF_SQE : C::OFF_SOP0) + half * 8192;
          const uint8_t* qh = sm + C::OFF_QH + half * C::PANEL;
          auto pack_rows = [&](const uint32_t (&r)[32], int cc) {
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
              const uint32_t off = sw_unit(i_out, (cc >> 3) + uu);
              uint32_t pw[4];
              if (qside) {
                const uint4 qv = *reinterpret_cast<const uint4*>(qh + off);
                const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  pw[e] = tc::pack_bf16(bf16_lo_f(qw[e]) - __uint_as_float(r[8 * uu + 2 * e]),
                                        bf16_hi_f(qw[e]) - __uint_as_float(r[8 * uu + 2 * e + 1]));
              } else {
#pragma unroll
                for (int e = 0; e < 4; ++e)
                  pw[e] = tc::pack_bf16(__uint_as_float(r[8 * uu + 2 * e]), __uint_as_float(r[8 * uu + 2 * e + 1]));
              }
              *reinterpret_cast<uint4*>(pnl + off) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
            }
          };
          uint32_t ra[32], rb[32];
          const uint32_t col = C::COL_QO + (qside ? 0u : 128u) + 64u * half;
          if (!tc::mbar_wait(mma3_done, ex & 1)) alive = false;
          tc::tc_fence_after();
          tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, col), ra);
          tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * q, col + 32), rb);
          tc::tmem_wait_ld_regs(ra);
          pack_rows(ra, 0);
          tc::tmem_wait_ld_regs(rb);
          pack_rows(rb, 32);
        }
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
      bar_compute();
      if (tid == 0) {
        if (skip) {
          // decay too steep for one reference point: hand the chunk back
          const int idx = atomicAdd(a.fix_list, 1);
          a.fix_list[1 + idx] = (int)tile;
          if (a.ready) tc::st_release_gpu(a.ready + tile, 3);
        }
        tc::mbar_arrive(st_b);
      }
    }
    // no task left: the store warp finishes what it holds and ends (once it
    // has taken the last task's tile index)
    if ((tid & 127) == 0) {
      if (tid == 0) {
        if (ex > 0) tc::mbar_wait(rd_a, (ex - 1) & 1);
        s_store[0] = -1;
      }
      tc::mbar_arrive(st_a);
    }
    if (!alive) {
      atomicExch(a.status, 8);
      vflag[0] = 1;
    }
    // release the UMMA warp (it waits for slice 0 of a next task)
    vflag[1] = 1;
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&built[0]);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tbase, C::TMEM_COLS);
  }
  if (stopper && tid == 0) {
    // the shared memory is about to be laid out for the next role
    for (int s = 0; s < C::NSLOT; ++s) {
      tc::mbar_inval(&full[s]);
      tc::mbar_inval(&gready[s]);
      tc::mbar_inval(&empty[s]);
    }
    for (int s = 0; s < C::SLICES; ++s) tc::mbar_inval(&built[s]);
    tc::mbar_inval(mma1_done);
    tc::mbar_inval(t_ready);
    tc::mbar_inval(mma2_done);
    tc::mbar_inval(rv_ready);
    tc::mbar_inval(mma3_done);
    tc::mbar_inval(fin);
    tc::mbar_inval(mma2a_done);
    tc::mbar_inval(mma3a_done);
    tc::mbar_inval(st_a);
    tc::mbar_inval(st_b);
    tc::mbar_inval(rd_a);
    tc::mbar_inval(rd_b);
    tc::fence_async_smem();
  }
  if (stopper) __syncthreads();
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
