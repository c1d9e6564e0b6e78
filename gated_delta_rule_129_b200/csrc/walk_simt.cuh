// walk_simt.cuh -- inter-chunk state walk fused with the chunk output, fp32
// on CUDA cores.
//
// One CTA per (sequence, head, value slice of DVS columns).  The columns of
// the state evolve independently once the chunk factors are known, because
// every update of S is a left multiplication (W S, diag(gamma) S, Kbar^T U).
// The state slice stays in shared memory, in fp32, for the whole walk.
//
// Per chunk with start state S (factors from the prep kernel):
//   U  = U~ - W S                            the per-token deltas z - r
//   O  = scale * (Q_eff S + O_part)          query reads the updated states
//   S <- diag(gamma_last) S + Kbar^T U       state at the next chunk start
// hT receives the final state; h0 (or zero) is the first start state.
//
// The chunk's tiles are copied to shared memory asynchronously: W, Q_eff,
// U~, O_part and gamma_n (used first) into one of two buffers a chunk ahead,
// Kbar (used last) into a single buffer as soon as the previous chunk's
// state update has read it.  Both products run on register tiles (a thread
// holds 2 x 2 of U and O, dk / 32 x 2 of S, and updates only the entries of
// S it read).
#pragma once

#include <type_traits>

#include "common.cuh"

namespace gdn2 {

template <typename IO, typename FT>
struct WalkArgs {
  const FT* W;
  const FT* Ut;
  const FT* Kbar;
  const FT* Qeff;
  const FT* Opart;
  const float* gamma_last;
  SeqMap map;
  int H;
  float scale;
  const float* h0;
  IO* out;              // nullptr: states only (the backward's recompute)
  float* hT;
  float* chunk_states;  // optional [max_chunks, H, DK, DV]
  float* U_out;         // optional [max_chunks, H, 64, DV]: every chunk's U (the backward)
};

// Value columns per CTA: 16 (256 threads) for the forward, where the walk has
// the GPU to itself; 32 (512 threads) beside the backward's reverse walk, so
// that both walks fit on the SMs at once.  A CTA has 16 threads per column.
constexpr int kWalkSimtDVS = 16;
constexpr int walk_simt_threads(int dvs) { return 16 * dvs; }

// Shared memory, in bytes: two buffers of (W, Q_eff with rows padded by 16
// bytes; the U~ and O_part slices; gamma_n), one Kbar tile, then S [DK][DVS]
// and U [64][DVS] in fp32.
template <int DK, typename FT, int DVS_>
struct WalkSimtCfg {
  static constexpr int DVS = DVS_;
  static constexpr int LKF = DK + 16 / (int)sizeof(FT);           // elements per padded row
  static constexpr int TILE = kChunk * LKF * (int)sizeof(FT);
  static constexpr int VSL = kChunk * DVS * (int)sizeof(FT);
  static constexpr int OFF_W = 0, OFF_QE = TILE, OFF_UT = 2 * TILE, OFF_OP = OFF_UT + VSL, OFF_GL = OFF_OP + VSL,
                       BUF = OFF_GL + DK * 4;
  static constexpr int OFF_KB = 2 * BUF, OFF_S = OFF_KB + TILE, OFF_U = OFF_S + DK * DVS * 4;
  static constexpr int SMEM = OFF_U + kChunk * DVS * 4;
  static_assert(SMEM <= 232448, "shared memory");
};

template <int DK, int DVS>
constexpr size_t walk_simt_smem_bytes() {
  return (size_t)WalkSimtCfg<DK, float, DVS>::SMEM;   // the fp32 plan bounds the bf16 one
}

// The walk of block `blk` (sequence, head, DVS value columns) with `wsm` its
// shared memory; all 16 DVS threads of the CTA take part.
template <int DK, int DV, typename IO, typename FT, int DVS>
__device__ __forceinline__ void walk_simt_cta(const WalkArgs<IO, FT>& a, int blk, uint8_t* wsm) {
  using C = WalkSimtCfg<DK, FT, DVS>;
  constexpr int SLICES = DV / DVS, LKF = C::LKF, NT = walk_simt_threads(DVS), HC = DVS / 2;
  const int H = a.H;
  const int sl = blk % SLICES;
  const int h = (blk / SLICES) % H;
  const int n = blk / (SLICES * H);
  const int j0 = sl * DVS;
  const int tid = threadIdx.x;

  float* sS = reinterpret_cast<float*>(wsm + C::OFF_S);   // [DK][DVS]
  float* sU = reinterpret_cast<float*>(wsm + C::OFF_U);   // [64][DVS]
  const FT* sKb = reinterpret_cast<const FT*>(wsm + C::OFF_KB);

  const size_t state_base = ((size_t)n * H + h) * DK * DV;
  for (int idx = tid; idx < DK * DVS; idx += NT) {
    const int cc = idx / DVS, j = idx % DVS;
    sS[idx] = a.h0 ? a.h0[state_base + (size_t)cc * DV + j0 + j] : 0.f;
  }
  const int c_begin = a.map.chunk_off[n], c_end = a.map.chunk_off[n + 1];
  const int s_begin = a.map.seq_begin(n), s_end = a.map.seq_end(n);
  constexpr int RB = DK * (int)sizeof(FT), SB = DVS * (int)sizeof(FT);
  auto issue_a = [&](int c) {   // W, Q_eff, U~, O_part, gamma_n of chunk c into buffer c & 1
    uint8_t* b = wsm + (c & 1) * C::BUF;
    const size_t tk = ((size_t)c * H + h) * kChunk * DK, tv = ((size_t)c * H + h) * kChunk * DV;
    stage_rows<RB>(b + C::OFF_W, LKF * sizeof(FT), a.W + tk, RB, kChunk, kChunk, tid, NT);
    if (a.out) stage_rows<RB>(b + C::OFF_QE, LKF * sizeof(FT), a.Qeff + tk, RB, kChunk, kChunk, tid, NT);
    stage_rows<SB>(b + C::OFF_UT, SB, a.Ut + tv + j0, DV * sizeof(FT), kChunk, kChunk, tid, NT);
    if (a.out) stage_rows<SB>(b + C::OFF_OP, SB, a.Opart + tv + j0, DV * sizeof(FT), kChunk, kChunk, tid, NT);
    stage_rows<DK * 4>(b + C::OFF_GL, 0, a.gamma_last + ((size_t)c * H + h) * DK, 0, 1, 1, tid, NT);
  };
  auto issue_k = [&](int c) {   // Kbar of chunk c
    stage_rows<RB>(wsm + C::OFF_KB, LKF * sizeof(FT), a.Kbar + ((size_t)c * H + h) * kChunk * DK, RB, kChunk, kChunk,
                   tid, NT);
  };
  // commit groups, oldest first: A(c_begin), K(c_begin), then per chunk c:
  // A(c + 1) at its start and K(c + 1) at its end (empty groups past the last)
  if (c_begin < c_end) issue_a(c_begin);
  cp_async_commit();
  if (c_begin < c_end) issue_k(c_begin);
  cp_async_commit();

  constexpr int RS = DK / 32;                      // rows of S per thread
  const int ri = tid / HC, cj = 2 * (tid % HC);    // U, O: rows 2 ri, 2 ri + 1; columns cj, cj + 1
  const int rs = RS * (tid / HC);                  // S: rows rs .. rs + RS - 1; columns cj, cj + 1
  for (int c = c_begin; c < c_end; ++c) {
    if (c + 1 < c_end) issue_a(c + 1);
    cp_async_commit();
    cp_async_wait<2>();   // A(c) has landed (K(c) and A(c + 1) may be in flight)
    __syncthreads();
    const uint8_t* b = wsm + (c & 1) * C::BUF;
    const FT* sW = reinterpret_cast<const FT*>(b + C::OFF_W);
    const FT* sQe = reinterpret_cast<const FT*>(b + C::OFF_QE);
    const FT* sUt = reinterpret_cast<const FT*>(b + C::OFF_UT);
    const FT* sOp = reinterpret_cast<const FT*>(b + C::OFF_OP);
    const float* sgl = reinterpret_cast<const float*>(b + C::OFF_GL);
    const int t0 = s_begin + (c - c_begin) * kChunk;
    const int len = min(kChunk, s_end - t0);
    if (a.chunk_states) {
      const size_t cs = ((size_t)c * H + h) * DK * DV;
      for (int idx = tid; idx < DK * DVS; idx += NT)
        a.chunk_states[cs + (size_t)(idx / DVS) * DV + j0 + idx % DVS] = sS[idx];
    }
    // U = U~ - W S and O = Q_eff S + O_part on a 2 x 2 tile (O only when it
    // is written: the backward's recompute needs the states and U alone)
    auto phase1 = [&](auto with_o) {
      constexpr bool WO = decltype(with_o)::value;
      float u[2][2], o[2][2];
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          u[r][q] = to_f32(sUt[(2 * ri + r) * DVS + cj + q]);
          o[r][q] = WO ? to_f32(sOp[(2 * ri + r) * DVS + cj + q]) : 0.f;
        }
#pragma unroll 2
      for (int c4 = 0; c4 < DK; c4 += 4) {   // four key rows of S a step, W and Q_eff read as vectors
        float wv[2][4], qv[2][4];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          load_vec<4>(sW + (2 * ri + r) * LKF + c4, wv[r]);
          if constexpr (WO) load_vec<4>(sQe + (2 * ri + r) * LKF + c4, qv[r]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 s = *reinterpret_cast<const float2*>(sS + (c4 + e) * DVS + cj);
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            u[r][0] = fmaf(-wv[r][e], s.x, u[r][0]); u[r][1] = fmaf(-wv[r][e], s.y, u[r][1]);
            if constexpr (WO) {
              o[r][0] = fmaf(qv[r][e], s.x, o[r][0]); o[r][1] = fmaf(qv[r][e], s.y, o[r][1]);
            }
          }
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = 2 * ri + r;
        *reinterpret_cast<float2*>(sU + i * DVS + cj) = make_float2(u[r][0], u[r][1]);
        if (a.U_out)
          *reinterpret_cast<float2*>(a.U_out + (((size_t)c * H + h) * kChunk + i) * DV + j0 + cj) =
              make_float2(u[r][0], u[r][1]);
        if (WO && i < len) {
          const size_t off = ((size_t)(t0 + i) * H + h) * DV + j0 + cj;
          a.out[off] = from_f32<IO>(a.scale * o[r][0]);
          a.out[off + 1] = from_f32<IO>(a.scale * o[r][1]);
        }
      }
    };
    if (a.out) phase1(std::true_type{});
    else phase1(std::false_type{});
    cp_async_wait<1>();   // K(c) has landed
    __syncthreads();
    // S <- diag(gamma_n) S + Kbar^T U on an RS x 2 tile (rows of Kbar and U
    // past the chunk's last token are zero)
    {
      float s[RS][2];
#pragma unroll
      for (int r = 0; r < RS; ++r) {
        const float g = sgl[rs + r];
        s[r][0] = g * sS[(rs + r) * DVS + cj];
        s[r][1] = g * sS[(rs + r) * DVS + cj + 1];
      }
#pragma unroll 4
      for (int i = 0; i < len; ++i) {
        const float2 uv = *reinterpret_cast<const float2*>(sU + i * DVS + cj);
        float kb[RS];
        load_vec<RS>(sKb + i * LKF + rs, kb);
#pragma unroll
        for (int r = 0; r < RS; ++r) {
          s[r][0] = fmaf(kb[r], uv.x, s[r][0]);
          s[r][1] = fmaf(kb[r], uv.y, s[r][1]);
        }
      }
#pragma unroll
      for (int r = 0; r < RS; ++r)
        *reinterpret_cast<float2*>(sS + (rs + r) * DVS + cj) = make_float2(s[r][0], s[r][1]);
    }
    __syncthreads();   // Kbar and this chunk's buffer are free
    if (c + 1 < c_end) issue_k(c + 1);
    cp_async_commit();
  }
  cp_async_wait<0>();
  __syncthreads();
  if (a.hT) {
    for (int idx = tid; idx < DK * DVS; idx += NT) {
      const int cc = idx / DVS, j = idx % DVS;
      a.hT[state_base + (size_t)cc * DV + j0 + j] = sS[idx];
    }
  }
}

template <int DK, int DV, typename IO, typename FT>
__global__ void __launch_bounds__(walk_simt_threads(kWalkSimtDVS))
walk_simt_kernel(const WalkArgs<IO, FT> a) {
  extern __shared__ __align__(16) uint8_t wsm[];
  walk_simt_cta<DK, DV, IO, FT, kWalkSimtDVS>(a, blockIdx.x, wsm);
}

}  // namespace gdn2
