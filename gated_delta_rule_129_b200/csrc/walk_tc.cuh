// walk_tc.cuh -- inter-chunk state walk + chunk output on the tensor cores
// (bf16 I/O, dk = 128, dv in {64, 128}).
//
// One CTA per (sequence, head, 64-column value slice).  The columns of the
// state evolve independently (every update is a left product), so a head's
// dv columns are split over dv/64 CTAs; each CTA keeps its 128 x 64 slice of
// the state in fp32 registers for the whole walk (4 epilogue warps: warp w
// owns key rows 32w .. 32w+31, the TMEM lane quarter it may read; each thread
// one key row x 64 columns).  A bf16 copy of the slice in shared memory is the
// B operand of two UMMAs per chunk:
//
//   D_S = Mp' . S'      (M = 128 key rows,  K = 128, N = 64)
//   D_O = Q_eff' . S'   (M = 64 tokens,     K = 128, N = 64)
//
// where S' = diag(colscale) S is the bf16 operand (the prep stores Mp and
// Q_eff with their columns divided by colscale, so Mp S = Mp' S'),
//
// and then   S <- diag(gamma) S - D_S + Nc      (fp32, in registers)
//            O  = scale * (D_O + O_part)        (query reads the updated state)
//
// which is the recurrence over one 64-token chunk in its affine form (the
// factors Mp = Kbar^T W, Nc = Kbar^T U~, Q_eff = Q~ - P W, O_part = P U~ come
// from the prep kernel).  The serial dependency per chunk is one UMMA (D_S)
// plus one register epilogue; D_O is issued after D_S, double-buffered in
// TMEM, and the bf16 state operand is double-buffered in shared memory, so
// the output epilogue of chunk j overlaps the critical path of chunk j+1.
//
// Two TMA rings feed it: ring A (Mp, Q_eff; read only by the UMMAs, released
// by tcgen05.commit) and ring B (the CTA's Nc and O_part columns, gamma and
// colscale; read by the epilogue warps, released by them).  Warp roles: 0-3
// update the state (the serial chain), 4-7 write the outputs, one lane of
// warp 8 issues the UMMAs, one lane each of warps 9 and 10 streams ring A
// (and prefetches the chunks ahead into L2) and ring B by TMA,
// so nothing but the state update sits between two D_S products.  Every wait is bounded; on a
// timeout the CTA records GDN2_ERR_DEVICE_TIMEOUT in the status word, drains
// what it issued and exits.
//
// Map mode (MAP = true, the first level of the two-level chunk scan): the
// same walk over a range of chunks, started from [I | 0] instead of a state,
// on the dk + dv columns of [Phi | Psi] (the chunk's Nc is added to the Psi
// columns only), without outputs; at the end of the range the CTA writes its
// columns of Phi (dk x dk) and Psi (dk x dv), the range's affine state map
// S_end = Phi S_start + Psi.
//
// Run beside the prep CTAs in one launch (gdn2_fused_kernel), the two TMA
// warps wait for each chunk's ready flag before loading its factors; a chunk
// the prep handed back to the exact kernel ends the walk early and raises the
// redo flag, and the host-side sequence then re-runs the walk after the fixup.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc.cuh"

namespace gdn2 {

struct WalkTcArgs {
  CUtensorMap tm_Mp;   // Mp    [rows = max_chunks*H*128, 128] bf16, box {64, 128}, SW128
  CUtensorMap tm_Qe;   // Q_eff [rows = max_chunks*H*64,  128] bf16, box {64, 64},  SW128
  CUtensorMap tm_Nc;   // Nc    [rows = max_chunks*H*128, dv]  bf16, box {64, 128}, SW128
  CUtensorMap tm_Op;   // O_part[rows = max_chunks*H*64,  dv]  bf16, box {64, 64},  SW128
  CUtensorMap tm_g;    // gamma [rows = max_chunks*H,     128] fp32, box {128, 1}
  CUtensorMap tm_cs;   // colscale, same shape and box
  SeqMap map;
  int H;
  float scale;
  const float* h0;
  __nv_bfloat16* out;
  float* hT;
  float* chunk_states;
  int* status;
  const int* ready;    // optional [max_chunks * H]: wait for 2 (written); 3 = handed back
  int* redo;           // set when a handed-back chunk ended the walk early
  const int* gate;     // optional: the kernel does nothing unless *gate != 0
  unsigned long long wait_ns;  // limit of every bounded wait (0: the default, 2 s)
  float* phi;          // map mode: [ranges, H, dk, dk] fp32
  float* psi;          // map mode: [ranges, H, dk, dv] fp32
};

// The walk's wait limit: the host's choice, or 2 s.
__device__ __forceinline__ uint64_t walk_budget(const WalkTcArgs& a) {
  return a.wait_ns ? (uint64_t)a.wait_ns : 2000000000ull;
}

template <int DV>
struct WalkTcCfg {
  static constexpr int DK = 128;
  static constexpr int NSL = 64;                 // value columns per CTA
  static constexpr int SLICES = DV / NSL;
  static constexpr int EPI_WARPS = 4;              // state warps 0-3, output warps 4-7
  static constexpr int MMA_WARP = 8, TMA_A_WARP = 9, TMA_B_WARP = 10;
  static constexpr int THREADS = 11 * 32;
  static constexpr int STAGES_A = 2;
  static constexpr int STAGES_B = 3;
  static constexpr int PF = 4;                   // L2 prefetch distance in chunks
  static constexpr int MP_BYTES = DK * DK * 2;             // 32 KiB
  static constexpr int QE_BYTES = kChunk * DK * 2;         // 16 KiB
  static constexpr int A_BYTES = MP_BYTES + QE_BYTES;
  static constexpr int NC_BYTES = DK * NSL * 2;            // 16 KiB, SW128 rows of 64
  static constexpr int OP_BYTES = kChunk * NSL * 2;        // 8 KiB, SW128 rows of 64
  static constexpr int G_BYTES = DK * 4;                   // 512 B each: gamma, colscale
  static constexpr int B_BYTES = NC_BYTES + OP_BYTES + 2 * G_BYTES;
  static constexpr int B_STRIDE = (B_BYTES + 1023) / 1024 * 1024;
  // bf16 state operand, MN-major interleaved core matrices (8 key rows x 8
  // columns, 128 B): offset(kg, ng) = kg * S_LBO + ng * 128
  static constexpr int S_LBO = (NSL / 8) * 128;
  static constexpr int S_BYTES = DK * NSL * 2;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = 1024 + STAGES_A * A_BYTES + STAGES_B * B_STRIDE + 2 * S_BYTES + BAR_BYTES;
  static constexpr int TMEM_COLS = 256;  // D_S [0,64), D_O[0] [64,128), D_O[1] [128,192)
  static_assert(NSL == 64, "SW128 Nc / O_part rows hold 64 columns");
  static_assert(SMEM <= 232448, "shared memory");
};

__device__ __forceinline__ void set_timeout(int* status, int* s_abort) {
  atomicExch(status, 8 /* GDN2_ERR_DEVICE_TIMEOUT */);
  *reinterpret_cast<volatile int*>(s_abort) = 1;
}


// Bounded wait that also ends when the CTA winds down (abort flag): true once
// the phase has completed; a timeout is recorded in the status word.
__device__ __forceinline__ bool wwait(uint64_t* bar, uint32_t parity, int* status, int* s_abort,
                                      uint64_t budget_ns = 2000000000ull) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = tc::global_ns();
  for (uint32_t it = 1;; ++it) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    // the abort flag and the clock only every 8th poll, so that a completed
    // phase is seen soon after it completes
    if ((it & 7u) == 0) {
      if (*reinterpret_cast<volatile int*>(s_abort)) return false;
      if (tc::global_ns() - t0 > budget_ns) {
        set_timeout(status, s_abort);
        return false;
      }
    }
  }
}

// Bounded wait until chunk tile `t` is ready; false on a timeout or when the
// prep handed the chunk back (then the redo flag is raised).
__device__ __forceinline__ bool wait_chunk_ready(const WalkTcArgs& a, int t, int* s_abort) {
  const uint64_t t0 = tc::global_ns();
  for (;;) {
    const int r = tc::ld_acquire_gpu(a.ready + t);
    if (r == 2) break;
    if (r == 3) {
      atomicExch(a.redo, 1);
      *reinterpret_cast<volatile int*>(s_abort) = 1;
      return false;
    }
    if (*reinterpret_cast<volatile int*>(s_abort)) return false;
    if (tc::global_ns() - t0 > walk_budget(a)) {
      set_timeout(a.status, s_abort);
      return false;
    }
  }
  // the TMA loads that follow read what the flag published
  tc::fence_async_global();
  return true;
}

template <int DV, bool MAP = false>
__device__ void walk_tc_cta(const WalkTcArgs& a, uint8_t* sm, int cta) {
  using C = WalkTcCfg<DV>;
  constexpr int DK = C::DK, NSL = C::NSL;
  // column slices per range: dv / 64 of the state, or (dk + dv) / 64 of [Phi | Psi]
  constexpr int SLC = MAP ? (DK + DV) / NSL : C::SLICES;
  uint8_t* ringA = sm;
  uint8_t* ringB = ringA + C::STAGES_A * C::A_BYTES;
  uint8_t* sS = ringB + C::STAGES_B * C::B_STRIDE;          // [2][S_BYTES]
  uint64_t* fullA = reinterpret_cast<uint64_t*>(sS + 2 * C::S_BYTES);
  uint64_t* emptyA = fullA + C::STAGES_A;
  uint64_t* fullB = emptyA + C::STAGES_A;
  uint64_t* emptyB = fullB + C::STAGES_B;
  uint64_t* s_done = emptyB + C::STAGES_B;   // D_S of the current chunk is ready
  uint64_t* o_done = s_done + 1;             // D_O of the current chunk is ready
  uint64_t* s_ready = o_done + 1;            // bf16 state operand written
  uint64_t* o_free = s_ready + 1;            // [2] D_O buffer read by the output warps
  uint64_t* fin = o_free + 2;                // every issued UMMA has finished
  uint32_t* tslot = reinterpret_cast<uint32_t*>(fin + 1);
  int* s_abort = reinterpret_cast<int*>(tslot + 1);
  const uint64_t wb = walk_budget(a);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H;
  const int sl = cta % SLC;
  const int h = (cta / SLC) % H;
  const int n = cta / (SLC * H);
  // map mode: slices 0 .. dk/64 - 1 hold Phi (key columns), the rest Psi
  const bool phi_slice = MAP && sl < DK / NSL;
  const int col0 = MAP && !phi_slice ? (sl - DK / NSL) * NSL : sl * NSL;
  const bool use_nc = !phi_slice;
  constexpr uint32_t A_TX = MAP ? C::MP_BYTES : C::A_BYTES;
  const int c_begin = a.map.chunk_off[n];
  const int nch = a.map.chunk_off[n + 1] - c_begin;
  const int s_begin = a.map.seq_begin(n), s_end = a.map.seq_end(n);

  if (tid == 0) {
    for (int s = 0; s < C::STAGES_A; ++s) {
      tc::mbar_init(&fullA[s], 1);
      tc::mbar_init(&emptyA[s], 1);
    }
    for (int s = 0; s < C::STAGES_B; ++s) {
      tc::mbar_init(&fullB[s], 1);
      tc::mbar_init(&emptyB[s], (MAP ? 1 : 2) * C::EPI_WARPS);  // state (and output) warps
    }
    tc::mbar_init(s_done, 1);
    tc::mbar_init(o_done, 1);
    tc::mbar_init(s_ready, C::EPI_WARPS);
    tc::mbar_init(&o_free[0], C::EPI_WARPS);
    tc::mbar_init(&o_free[1], C::EPI_WARPS);
    tc::mbar_init(fin, 1);
    *s_abort = 0;
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

  if (warp < C::EPI_WARPS) {
    // ----------------------------------------------------- state update --
    const int row = 32 * warp + lane;  // key channel = TMEM lane
    const size_t sbase = ((size_t)n * H + h) * DK * DV + (size_t)row * DV + col0;
    float S[NSL];
    if (MAP) {
      // [I | 0]: this thread's row of the identity (Phi) or zeros (Psi)
#pragma unroll
      for (int i = 0; i < NSL; ++i) S[i] = phi_slice && row == col0 + i ? 1.f : 0.f;
    } else {
#pragma unroll
      for (int i = 0; i < NSL; i += 4) {
        const float4 v = a.h0 ? *reinterpret_cast<const float4*>(a.h0 + sbase + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        S[i] = v.x; S[i + 1] = v.y; S[i + 2] = v.z; S[i + 3] = v.w;
      }
    }
    // this thread's row in the interleaved operand: core matrix (row/8, g),
    // 16-byte line row%8
    const uint32_t srow = (row >> 3) * C::S_LBO + (row & 7) * 16;
    // the bf16 operand of the chunk that reads it: this row times its colscale
    auto store_state = [&](int buf, float cs) {
      uint8_t* base = sS + buf * C::S_BYTES + srow;
#pragma unroll
      for (int g = 0; g < NSL / 8; ++g) {
        uint4 pk;
        pk.x = tc::pack_bf16(cs * S[8 * g + 0], cs * S[8 * g + 1]);
        pk.y = tc::pack_bf16(cs * S[8 * g + 2], cs * S[8 * g + 3]);
        pk.z = tc::pack_bf16(cs * S[8 * g + 4], cs * S[8 * g + 5]);
        pk.w = tc::pack_bf16(cs * S[8 * g + 6], cs * S[8 * g + 7]);
        *reinterpret_cast<uint4*>(base + g * 128) = pk;
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(s_ready);
    };
    auto colscale_of = [&](int j) {   // row's colscale for chunk j (its ring B stage has landed)
      return reinterpret_cast<const float*>(ringB + (j % C::STAGES_B) * C::B_STRIDE + C::NC_BYTES + C::OP_BYTES +
                                            C::G_BYTES)[row];
    };
    if (nch > 0) {
      if (wwait(&fullB[0], 0, a.status, s_abort, wb)) store_state(0, colscale_of(0));
    }

    for (int j = 0; j < nch; ++j) {
      if (*reinterpret_cast<volatile int*>(s_abort)) break;
      const int c = c_begin + j;
      const int sb = j % C::STAGES_B;
      const uint8_t* stB = ringB + sb * C::B_STRIDE;
      if (a.chunk_states) {
        float* cs = a.chunk_states + ((size_t)c * H + h) * DK * DV + (size_t)row * DV + col0;
#pragma unroll
        for (int i = 0; i < NSL; i += 4) *reinterpret_cast<float4*>(cs + i) = make_float4(S[i], S[i + 1], S[i + 2], S[i + 3]);
      }
      if (!wwait(&fullB[sb], (j / C::STAGES_B) & 1, a.status, s_abort, wb)) break;
      // Nc row (64 bf16, SW128) and gamma before the product is ready
      const float gam = reinterpret_cast<const float*>(stB + C::NC_BYTES + C::OP_BYTES)[row];
      uint32_t ncw[NSL / 2];
#pragma unroll
      for (int u = 0; u < NSL / 8; ++u) {
        // (Phi columns of map mode take no Nc: zero words)
        const uint4 t = use_nc ? *reinterpret_cast<const uint4*>(stB + row * 128 + ((u ^ (row & 7)) << 4))
                               : make_uint4(0u, 0u, 0u, 0u);
        ncw[4 * u] = t.x; ncw[4 * u + 1] = t.y; ncw[4 * u + 2] = t.z; ncw[4 * u + 3] = t.w;
      }
      if (!wwait(s_done, j & 1, a.status, s_abort, wb)) break;
      tc::tc_fence_after();
      // S <- gamma * S - Mp S + Nc
      {
        uint32_t d0[32], d1[32];
        tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * warp, 0), d0);
        tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * warp, 32), d1);
        tc::tmem_wait_ld_regs(d0);
        tc::tmem_wait_ld_regs(d1);
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint32_t w2 = ncw[e / 2];
          S[e] = fmaf(gam, S[e], bf16_lo_f(w2) - __uint_as_float(d0[e]));
          S[e + 1] = fmaf(gam, S[e + 1], bf16_hi_f(w2) - __uint_as_float(d0[e + 1]));
        }
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const uint32_t w2 = ncw[16 + e / 2];
          S[32 + e] = fmaf(gam, S[32 + e], bf16_lo_f(w2) - __uint_as_float(d1[e]));
          S[32 + e + 1] = fmaf(gam, S[32 + e + 1], bf16_hi_f(w2) - __uint_as_float(d1[e + 1]));
        }
      }
      // D_O(j-1) read sS[(j+1)&1]; it was issued before D_S(j), so it is done.
      // The operand is for chunk j+1 (its stage lands before this one is released).
      float cs_next = 1.f;
      if (j + 1 < nch) {
        const int sn = (j + 1) % C::STAGES_B;
        if (!wwait(&fullB[sn], ((j + 1) / C::STAGES_B) & 1, a.status, s_abort, wb)) break;
        cs_next = colscale_of(j + 1);
      }
      store_state((j + 1) & 1, cs_next);
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&emptyB[sb]);
    }
    if (MAP && !*reinterpret_cast<volatile int*>(s_abort)) {
      float* dst = phi_slice ? a.phi + (((size_t)n * H + h) * DK + row) * DK + col0
                             : a.psi + (((size_t)n * H + h) * DK + row) * DV + col0;
#pragma unroll
      for (int i = 0; i < NSL; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(S[i], S[i + 1], S[i + 2], S[i + 3]);
    } else if (a.hT && !*reinterpret_cast<volatile int*>(s_abort)) {
#pragma unroll
      for (int i = 0; i < NSL; i += 4)
        *reinterpret_cast<float4*>(a.hT + sbase + i) = make_float4(S[i], S[i + 1], S[i + 2], S[i + 3]);
    }
  } else if (warp < 2 * C::EPI_WARPS) {
    if constexpr (!MAP) {  // no outputs in map mode
    // ---------------------------------------------------------- outputs --
    const int ow = warp - C::EPI_WARPS;   // TMEM lane quarter of this warp
    const int i_tok = 16 * ow + lane;     // token row of D_O (M = 64 layout), lane < 16
    for (int j = 0; j < nch; ++j) {
      if (*reinterpret_cast<volatile int*>(s_abort)) break;
      const int sb = j % C::STAGES_B;
      const uint8_t* stB = ringB + sb * C::B_STRIDE;
      if (!wwait(&fullB[sb], (j / C::STAGES_B) & 1, a.status, s_abort, wb) || !wwait(o_done, j & 1, a.status, s_abort, wb))
        break;
      tc::tc_fence_after();
      uint32_t d0[32], d1[32];
      tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * ow, (uint32_t)NSL * (1u + (j & 1))), d0);
      tc::tmem_ld32_nowait(tc::tmem_addr(tbase, 32 * ow, (uint32_t)NSL * (1u + (j & 1)) + 32), d1);
      tc::tmem_wait_ld_regs(d0);
      tc::tmem_wait_ld_regs(d1);
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&o_free[j & 1]);
      const int t0 = s_begin + j * kChunk;
      const int len = min(kChunk, s_end - t0);
      if (lane < 16 && i_tok < len) {
        const uint8_t* op = stB + C::NC_BYTES + i_tok * 128;
        uint4* dst = reinterpret_cast<uint4*>(a.out + ((size_t)(t0 + i_tok) * H + h) * DV + col0);
#pragma unroll
        for (int u = 0; u < NSL / 8; ++u) {
          const uint4 o4 = *reinterpret_cast<const uint4*>(op + ((u ^ (i_tok & 7)) << 4));
          const uint32_t ow4[4] = {o4.x, o4.y, o4.z, o4.w};
          const uint32_t* dd = u < 4 ? d0 + 8 * u : d1 + 8 * (u - 4);
          uint32_t pw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            pw[e] = tc::pack_bf16(a.scale * (__uint_as_float(dd[2 * e]) + bf16_lo_f(ow4[e])),
                                  a.scale * (__uint_as_float(dd[2 * e + 1]) + bf16_hi_f(ow4[e])));
          dst[u] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&emptyB[sb]);
    }
    }
  } else if (warp == C::MMA_WARP && lane == 0) {
    // --------------------------------------------------------- UMMA issue --
    constexpr uint32_t idS = tc::idesc_bf16(128, NSL, false, true);
    constexpr uint32_t idO = tc::idesc_bf16(64, NSL, false, true);
    const uint64_t mp_d0 = tc::sdesc(tc::smem_u32(ringA), 16, 1024, tc::kLayoutSW128);
    const uint64_t sb_d0 = tc::sdesc(tc::smem_u32(sS), C::S_LBO, 128, tc::kLayoutNone);
    for (int j = 0; j < nch; ++j) {
      const int st = j % C::STAGES_A;
      if (!wwait(&fullA[st], (j / C::STAGES_A) & 1, a.status, s_abort, wb) || !wwait(s_ready, j & 1, a.status, s_abort, wb))
        break;
      if (*reinterpret_cast<volatile int*>(s_abort)) break;
      tc::tc_fence_after();
      // descriptors: the start address sits in the low bits (16-byte units),
      // so a K-step is a 64-bit add of (byte offset >> 4)
      const uint64_t mp_d = mp_d0 + (uint64_t)((st * C::A_BYTES) >> 4);
      const uint64_t qe_d = mp_d + (uint64_t)(C::MP_BYTES >> 4);
      const uint64_t sb_d = sb_d0 + (uint64_t)(((j & 1) * C::S_BYTES) >> 4);
#pragma unroll
      for (int s = 0; s < DK / 16; ++s)
        tc::umma_f16(tbase, mp_d + (uint64_t)(((s / 4) * (DK * 128) + (s % 4) * 32) >> 4),
                     sb_d + (uint64_t)((s * 2 * C::S_LBO) >> 4), idS, s > 0);
      tc::umma_commit(s_done);
      if (MAP) {
        tc::umma_commit(&emptyA[st]);
        continue;
      }
      // the output warps have read D_O(j-1): keeps every o_done waiter within
      // one phase (and frees the D_O buffer D_O(j+1) will use)
      if (j >= 1 && !wwait(&o_free[(j - 1) & 1], ((j - 1) >> 1) & 1, a.status, s_abort, wb)) break;
#pragma unroll
      for (int s = 0; s < DK / 16; ++s)
        tc::umma_f16(tbase + (uint32_t)NSL * (1u + (j & 1)),
                     qe_d + (uint64_t)(((s / 4) * (kChunk * 128) + (s % 4) * 32) >> 4),
                     sb_d + (uint64_t)((s * 2 * C::S_LBO) >> 4), idO, s > 0);
      tc::umma_commit(o_done);
      tc::umma_commit(&emptyA[st]);
    }
    // every issued UMMA has finished before TMEM is released
    tc::umma_commit(fin);
    tc::mbar_wait(fin, 0);
  } else if (warp == C::TMA_A_WARP && lane == 0) {
    // ------------------------------------------------ ring A producer (TMA) --
    tc::prefetch_tmap(&a.tm_Mp);
    tc::prefetch_tmap(&a.tm_Qe);
    int loaded = 0;
    for (int j = 0; j < nch; ++j) {
      if (*reinterpret_cast<volatile int*>(s_abort)) break;
      const int c = c_begin + j, st = j % C::STAGES_A;
      // Pull chunk j + PF's factors into L2 (all of them: the ring B warp
      // only reads what this brings), if they are written by now; the rings
      // are shallow and the factors may have left L2.
      if (j + C::PF < nch) {
        const int cp = c + C::PF, tp = cp * H + h;
        if (!a.ready || tc::ld_acquire_gpu(a.ready + tp) == 2) {
          const int rm = tp * DK, rq = tp * kChunk;
          tc::tma_prefetch_2d(&a.tm_Mp, 0, rm);
          tc::tma_prefetch_2d(&a.tm_Mp, 64, rm);
          if (!MAP) {
            tc::tma_prefetch_2d(&a.tm_Qe, 0, rq);
            tc::tma_prefetch_2d(&a.tm_Qe, 64, rq);
            tc::tma_prefetch_2d(&a.tm_Op, col0, rq);
          }
          if (use_nc) tc::tma_prefetch_2d(&a.tm_Nc, col0, rm);
          tc::tma_prefetch_2d(&a.tm_g, 0, tp);
          tc::tma_prefetch_2d(&a.tm_cs, 0, tp);
        }
      }
      if (j >= C::STAGES_A && !wwait(&emptyA[st], ((j - C::STAGES_A) / C::STAGES_A) & 1, a.status, s_abort, wb)) break;
      if (a.ready && !wait_chunk_ready(a, c * H + h, s_abort)) break;
      uint8_t* dst = ringA + st * C::A_BYTES;
      tc::mbar_arrive_expect_tx(&fullA[st], A_TX);
      const int rm = (c * H + h) * DK, rq = (c * H + h) * kChunk;
      tc::tma_load_2d(dst, &a.tm_Mp, &fullA[st], 0, rm);
      tc::tma_load_2d(dst + DK * 128, &a.tm_Mp, &fullA[st], 64, rm);
      if (!MAP) {
        tc::tma_load_2d(dst + C::MP_BYTES, &a.tm_Qe, &fullA[st], 0, rq);
        tc::tma_load_2d(dst + C::MP_BYTES + kChunk * 128, &a.tm_Qe, &fullA[st], 64, rq);
      }
      ++loaded;
    }
    // every issued load has landed before the CTA releases its shared memory
    // (each stage holds at most one outstanding load)
    for (int j = loaded > C::STAGES_A ? loaded - C::STAGES_A : 0; j < loaded; ++j)
      tc::mbar_wait(&fullA[j % C::STAGES_A], (j / C::STAGES_A) & 1);
  } else if (warp == C::TMA_B_WARP && lane == 0) {
    // ------------------------------------------------ ring B producer (TMA) --
    tc::prefetch_tmap(&a.tm_Nc);
    tc::prefetch_tmap(&a.tm_Op);
    tc::prefetch_tmap(&a.tm_g);
    tc::prefetch_tmap(&a.tm_cs);
    int loaded = 0;
    for (int j = 0; j < nch; ++j) {
      if (*reinterpret_cast<volatile int*>(s_abort)) break;
      const int c = c_begin + j, st = j % C::STAGES_B;
      if (j >= C::STAGES_B && !wwait(&emptyB[st], ((j - C::STAGES_B) / C::STAGES_B) & 1, a.status, s_abort, wb)) break;
      if (a.ready && !wait_chunk_ready(a, c * H + h, s_abort)) break;
      uint8_t* dst = ringB + st * C::B_STRIDE;
      tc::mbar_arrive_expect_tx(&fullB[st], (use_nc ? C::NC_BYTES : 0) + (MAP ? 0 : C::OP_BYTES) + 2 * C::G_BYTES);
      if (use_nc) tc::tma_load_2d(dst, &a.tm_Nc, &fullB[st], col0, (c * H + h) * DK);
      if (!MAP) tc::tma_load_2d(dst + C::NC_BYTES, &a.tm_Op, &fullB[st], col0, (c * H + h) * kChunk);
      tc::tma_load_2d(dst + C::NC_BYTES + C::OP_BYTES, &a.tm_g, &fullB[st], 0, c * H + h);
      tc::tma_load_2d(dst + C::NC_BYTES + C::OP_BYTES + C::G_BYTES, &a.tm_cs, &fullB[st], 0, c * H + h);
      ++loaded;
    }
    for (int j = loaded > C::STAGES_B ? loaded - C::STAGES_B : 0; j < loaded; ++j)
      tc::mbar_wait(&fullB[j % C::STAGES_B], (j / C::STAGES_B) & 1);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == C::MMA_WARP) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

template <int DV, bool MAP = false>
__global__ void __launch_bounds__(WalkTcCfg<DV>::THREADS, 1)
walk_tc_kernel(const __grid_constant__ WalkTcArgs a) {
  if (a.gate && *a.gate == 0) return;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  walk_tc_cta<DV, MAP>(a, sm, blockIdx.x);
}

}  // namespace gdn2
