// walk_tc.cuh -- inter-chunk state walk + chunk output on the tensor cores
// (bf16 I/O, dk = 128, dv in {64, 128}).
//
// One CTA per (sequence, head).  The head's dk x dv state stays in fp32
// registers for the whole walk (16 epilogue warps; warp w owns key rows
// 32*(w%4) .. +31 and value columns (w/4)*dv/4 .. +dv/4, matching the TMEM
// lane quarter the warp may read).  A bf16 copy of the state in shared memory
// is the B operand of two UMMAs per chunk:
//
//   D_S = Mp . S        (M = 128 key rows,  K = 128, N = dv)
//   D_O = Q_eff . S     (M = 64 tokens,     K = 128, N = dv)
//
// and then   S <- diag(gamma) S - D_S + Nc      (fp32, in registers)
//            O  = scale * (D_O + O_part)        (query reads the updated state)
//
// which is the recurrence over one 64-token chunk in its affine form (the
// factors Mp = Kbar^T W, Nc = Kbar^T U~, Q_eff = Q~ - P W, O_part = P U~ come
// from the prep kernel).  The serial dependency per chunk is one UMMA plus
// one register epilogue.  Mp and Q_eff tiles are streamed by TMA through a
// 3-stage ring; Nc, O_part and gamma rows are prefetched into registers one
// chunk ahead.  D_O is double-buffered in TMEM so the output epilogue of
// chunk j overlaps the UMMA of chunk j+1.
//
// Warp 16 is the producer: one lane issues the TMA loads and the UMMAs.
// Every wait is bounded; on a timeout the CTA records GDN2_ERR_DEVICE_TIMEOUT
// in the status word, drains what it issued and exits.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "tc.cuh"

namespace gdn2 {

struct WalkTcArgs {
  CUtensorMap tm_Mp;   // [max_chunks*H*128 rows, 128] bf16, box {64, 128}, SW128
  CUtensorMap tm_Qe;   // [max_chunks*H*64 rows, 128]  bf16, box {64, 64},  SW128
  const __nv_bfloat16* Nc;     // [max_chunks, H, 128, DV]
  const __nv_bfloat16* Opart;  // [max_chunks, H, 64, DV]
  const float* gamma_last;     // [max_chunks, H, 128]
  SeqMap map;
  int H;
  float scale;
  const float* h0;
  __nv_bfloat16* out;
  float* hT;
  float* chunk_states;
  int* status;
};

template <int DV>
struct WalkTcCfg {
  static constexpr int DK = 128;
  static constexpr int EPI_WARPS = 16;
  static constexpr int THREADS = EPI_WARPS * 32 + 32;
  static constexpr int CPT = DV / 4;  // state columns per epilogue thread
  static constexpr int STAGES = 3;
  static constexpr int MP_BYTES = DK * DK * 2;
  static constexpr int QE_BYTES = kChunk * DK * 2;
  static constexpr int STAGE_BYTES = MP_BYTES + QE_BYTES;
  static constexpr int S_BYTES = DK * DV * 2;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = 1024 + STAGES * STAGE_BYTES + S_BYTES + BAR_BYTES;
  static constexpr int TMEM_COLS = DV == 128 ? 512 : 256;  // D_S, D_O[0], D_O[1]
  static_assert(CPT % 16 == 0, "whole 16-column TMEM loads per thread");
};

__device__ __forceinline__ void set_timeout(int* status, int* s_abort) {
  atomicExch(status, 8 /* GDN2_ERR_DEVICE_TIMEOUT */);
  *reinterpret_cast<volatile int*>(s_abort) = 1;
}

template <int DV>
__global__ void __launch_bounds__(WalkTcCfg<DV>::THREADS, 1)
walk_tc_kernel(const __grid_constant__ WalkTcArgs a) {
  using C = WalkTcCfg<DV>;
  constexpr int DK = C::DK, CPT = C::CPT;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sS = sm + C::STAGES * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sS + C::S_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* mma_done = empty + C::STAGES;
  uint64_t* s_ready = mma_done + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(s_ready + 1);
  int* s_abort = reinterpret_cast<int*>(tslot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int H = a.H;
  const int n = blockIdx.x / H, h = blockIdx.x % H;
  const int c_begin = a.map.chunk_off[n];
  const int nch = a.map.chunk_off[n + 1] - c_begin;
  const int s_begin = a.map.seq_begin(n), s_end = a.map.seq_end(n);

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      tc::mbar_init(&full[s], 1);
      tc::mbar_init(&empty[s], 1);
    }
    tc::mbar_init(mma_done, 1);
    tc::mbar_init(s_ready, C::EPI_WARPS);
    *s_abort = 0;
    tc::fence_mbar_init();
  }
  if (warp == C::EPI_WARPS) {
    tc::tmem_alloc(tslot, C::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tslot;

  if (warp < C::EPI_WARPS) {
    // ------------------------------------------------------------ epilogue --
    const int q = warp & 3, cg = warp >> 2;
    const int row = 32 * q + lane;  // key channel (TMEM lane)
    const int c0 = cg * CPT;        // first value column
    const size_t sbase = ((size_t)n * H + h) * DK * DV + (size_t)row * DV + c0;
    float S[CPT];
#pragma unroll
    for (int i = 0; i < CPT; i += 4) {
      float4 v = a.h0 ? *reinterpret_cast<const float4*>(a.h0 + sbase + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      S[i] = v.x; S[i + 1] = v.y; S[i + 2] = v.z; S[i + 3] = v.w;
    }
    // bf16 state operand, MN-major SW128: element (k = row, n = col) of panel
    // col / 64 at sw128_off(row, col % 64); this thread's columns are
    // CPT / 8 whole 16-byte units of one panel.
    uint8_t* srow = sS + (c0 / 64) * (DK * 128) + row * 128;
    const int u0 = (c0 % 64) / 8;
    auto store_state = [&]() {
#pragma unroll
      for (int u = 0; u < CPT / 8; ++u) {
        uint4 pk;
        pk.x = tc::pack_bf16(S[8 * u + 0], S[8 * u + 1]);
        pk.y = tc::pack_bf16(S[8 * u + 2], S[8 * u + 3]);
        pk.z = tc::pack_bf16(S[8 * u + 4], S[8 * u + 5]);
        pk.w = tc::pack_bf16(S[8 * u + 6], S[8 * u + 7]);
        *reinterpret_cast<uint4*>(srow + ((((u0 + u) ^ (row & 7)) << 4))) = pk;
      }
      tc::fence_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(s_ready);
    };
    store_state();

    // per-chunk row data, prefetched one chunk ahead
    uint32_t nc_r[CPT / 2], op_r[CPT / 2];  // bf16 pairs
    float gam = 0.f;
    auto prefetch = [&](int j) {
      const int c = c_begin + j;
      const size_t mat = ((size_t)c * H + h) * DK;
      const uint4* np = reinterpret_cast<const uint4*>(a.Nc + (mat + row) * DV + c0);
#pragma unroll
      for (int u = 0; u < CPT / 8; ++u) {
        const uint4 t = __ldg(np + u);
        nc_r[4 * u] = t.x; nc_r[4 * u + 1] = t.y; nc_r[4 * u + 2] = t.z; nc_r[4 * u + 3] = t.w;
      }
      gam = __ldg(a.gamma_last + mat + row);
      if (lane < 16) {
        const size_t orow = ((size_t)c * H + h) * kChunk + 16 * q + lane;
        const uint4* op = reinterpret_cast<const uint4*>(a.Opart + orow * DV + c0);
#pragma unroll
        for (int u = 0; u < CPT / 8; ++u) {
          const uint4 t = __ldg(op + u);
          op_r[4 * u] = t.x; op_r[4 * u + 1] = t.y; op_r[4 * u + 2] = t.z; op_r[4 * u + 3] = t.w;
        }
      }
    };
    if (nch > 0) prefetch(0);

    for (int j = 0; j < nch; ++j) {
      if (*reinterpret_cast<volatile int*>(s_abort)) break;
      const int c = c_begin + j;
      if (a.chunk_states) {
        float* cs = a.chunk_states + ((size_t)c * H + h) * DK * DV + (size_t)row * DV + c0;
#pragma unroll
        for (int i = 0; i < CPT; i += 4) *reinterpret_cast<float4*>(cs + i) = make_float4(S[i], S[i + 1], S[i + 2], S[i + 3]);
      }
      if (!tc::mbar_wait(mma_done, j & 1)) {
        set_timeout(a.status, s_abort);
        break;
      }
      tc::tc_fence_after();
      // state: S <- gamma * S - Mp S + Nc
#pragma unroll
      for (int m = 0; m < CPT / 16; ++m) {
        float d[16];
        tc::tmem_ld16(tc::tmem_addr(tbase, 32 * q, c0 + 16 * m), d);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int e = 16 * m + i;
          const uint32_t w2 = nc_r[e / 2];
          const float nv = __uint_as_float((e & 1) ? (w2 & 0xFFFF0000u) : (w2 << 16));
          S[e] = fmaf(gam, S[e], nv - d[i]);
        }
      }
      store_state();
      // output of chunk j from D_O[j & 1]: token rows 16 q + lane (lane < 16)
      const int t0 = s_begin + j * kChunk;
      const int len = min(kChunk, s_end - t0);
      const uint32_t ocol = (uint32_t)DV * (1u + (j & 1));
#pragma unroll
      for (int m = 0; m < CPT / 16; ++m) {
        float d[16];
        tc::tmem_ld16(tc::tmem_addr(tbase, 32 * q, ocol + c0 + 16 * m), d);
        tc::tmem_wait_ld();
        const int i_tok = 16 * q + lane;
        if (lane < 16 && i_tok < len) {
          uint32_t pw[8];
#pragma unroll
          for (int i = 0; i < 16; i += 2) {
            const int e = 16 * m + i;
            const uint32_t w2 = op_r[e / 2];
            const float o0 = a.scale * (d[i] + __uint_as_float(w2 << 16));
            const float o1 = a.scale * (d[i + 1] + __uint_as_float(w2 & 0xFFFF0000u));
            pw[i / 2] = tc::pack_bf16(o0, o1);
          }
          uint4* dst = reinterpret_cast<uint4*>(a.out + ((size_t)(t0 + i_tok) * H + h) * DV + c0 + 16 * m);
          dst[0] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
          dst[1] = make_uint4(pw[4], pw[5], pw[6], pw[7]);
        }
      }
      tc::tc_fence_before();
      if (j + 1 < nch) prefetch(j + 1);
    }
    if (a.hT && !*reinterpret_cast<volatile int*>(s_abort)) {
#pragma unroll
      for (int i = 0; i < CPT; i += 4)
        *reinterpret_cast<float4*>(a.hT + sbase + i) = make_float4(S[i], S[i + 1], S[i + 2], S[i + 3]);
    }
  } else if (lane == 0) {
    // ------------------------------------------------- producer + UMMA issue --
    tc::prefetch_tmap(&a.tm_Mp);
    tc::prefetch_tmap(&a.tm_Qe);
    auto load = [&](int j) {
      const int st = j % C::STAGES;
      const int c = c_begin + j;
      uint8_t* dst = sm + st * C::STAGE_BYTES;
      tc::mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
      const int rm = (c * H + h) * DK, rq = (c * H + h) * kChunk;
      tc::tma_load_2d(dst, &a.tm_Mp, &full[st], 0, rm);
      tc::tma_load_2d(dst + DK * 128, &a.tm_Mp, &full[st], 64, rm);
      tc::tma_load_2d(dst + C::MP_BYTES, &a.tm_Qe, &full[st], 0, rq);
      tc::tma_load_2d(dst + C::MP_BYTES + kChunk * 128, &a.tm_Qe, &full[st], 64, rq);
    };
    const int pre = nch < C::STAGES ? nch : C::STAGES;
    for (int j = 0; j < pre; ++j) load(j);
    int loaded = pre, committed = 0;
    constexpr uint32_t idS = tc::idesc_bf16(128, DV, false, true);
    constexpr uint32_t idO = tc::idesc_bf16(64, DV, false, true);
    const uint32_t sS_addr = tc::smem_u32(sS);
    bool ok = true;
    for (int j = 0; j < nch && ok; ++j) {
      const int st = j % C::STAGES;
      ok = tc::mbar_wait(&full[st], (j / C::STAGES) & 1) && tc::mbar_wait(s_ready, j & 1);
      if (!ok || *reinterpret_cast<volatile int*>(s_abort)) {
        if (!ok) set_timeout(a.status, s_abort);
        ok = false;
        break;
      }
      tc::tc_fence_after();
      const uint32_t mp = tc::smem_u32(sm + st * C::STAGE_BYTES);
      const uint32_t qe = mp + C::MP_BYTES;
#pragma unroll
      for (int s = 0; s < DK / 16; ++s) {
        const uint32_t koff = (s % 4) * 32;
        const uint64_t bd = tc::sdesc(sS_addr + s * 16 * 128, DK * 128, 1024, tc::kLayoutSW128);
        const uint64_t ad = tc::sdesc(mp + (s / 4) * (DK * 128) + koff, 16, 1024, tc::kLayoutSW128);
        tc::umma_f16(tbase, ad, bd, idS, s > 0);
      }
#pragma unroll
      for (int s = 0; s < DK / 16; ++s) {
        const uint32_t koff = (s % 4) * 32;
        const uint64_t bd = tc::sdesc(sS_addr + s * 16 * 128, DK * 128, 1024, tc::kLayoutSW128);
        const uint64_t ad = tc::sdesc(qe + (s / 4) * (kChunk * 128) + koff, 16, 1024, tc::kLayoutSW128);
        tc::umma_f16(tbase + (uint32_t)DV * (1u + (j & 1)), ad, bd, idO, s > 0);
      }
      tc::umma_commit(mma_done);
      tc::umma_commit(&empty[st]);
      committed = j + 1;
      if (loaded < nch) {
        // stage st is reused for chunk `loaded` once these UMMAs have read it
        if (!tc::mbar_wait(&empty[st], (j / C::STAGES) & 1)) {
          set_timeout(a.status, s_abort);
          ok = false;
          break;
        }
        load(loaded);
        ++loaded;
      }
    }
    // drain: every issued load has landed and every issued UMMA has finished
    // before the CTA releases its shared and tensor memory
    for (int j = committed; j < loaded; ++j) tc::mbar_wait(&full[j % C::STAGES], (j / C::STAGES) & 1);
    if (committed > 0) tc::mbar_wait(mma_done, (committed - 1) & 1);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == C::EPI_WARPS) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tbase, C::TMEM_COLS);
  }
}

}  // namespace gdn2
