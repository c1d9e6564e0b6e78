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
// The chunk's factor tiles are copied to shared memory asynchronously into
// one of two buffers while the previous chunk is computed; both products run
// on register tiles (a thread holds 2 x 2 of U and O, dk / 32 x 2 of S; every
// thread updates only the entries of S it read).
#pragma once

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
};

constexpr int kWalkSimtThreads = 256;
constexpr int kWalkSimtDVS = 16;

// Shared memory, in bytes: two chunk buffers (W, Kbar, Q_eff rows padded by
// 16 bytes; U~ and O_part slices; gamma_n), then S [DK][DVS] and U [64][DVS]
// in fp32.
template <int DK, typename FT>
struct WalkSimtCfg {
  static constexpr int LKF = DK + 16 / (int)sizeof(FT);           // elements per padded row
  static constexpr int TILE = kChunk * LKF * (int)sizeof(FT);
  static constexpr int VSL = kChunk * kWalkSimtDVS * (int)sizeof(FT);
  static constexpr int OFF_W = 0, OFF_KB = TILE, OFF_QE = 2 * TILE, OFF_UT = 3 * TILE, OFF_OP = OFF_UT + VSL,
                       OFF_GL = OFF_OP + VSL, BUF = OFF_GL + DK * 4;
  static constexpr int OFF_S = 2 * BUF, OFF_U = OFF_S + DK * kWalkSimtDVS * 4;
  static constexpr int SMEM = OFF_U + kChunk * kWalkSimtDVS * 4;
  static_assert(SMEM <= 232448, "shared memory");
};

template <int DK, int DV>
constexpr size_t walk_simt_smem_bytes() {
  return (size_t)WalkSimtCfg<DK, float>::SMEM;   // the fp32 plan bounds the bf16 one
}

template <int DK, int DV, typename IO, typename FT>
__global__ void __launch_bounds__(kWalkSimtThreads)
walk_simt_kernel(const WalkArgs<IO, FT> a) {
  using C = WalkSimtCfg<DK, FT>;
  constexpr int DVS = kWalkSimtDVS, SLICES = DV / DVS, LKF = C::LKF;
  const int H = a.H;
  const int sl = blockIdx.x % SLICES;
  const int h = (blockIdx.x / SLICES) % H;
  const int n = blockIdx.x / (SLICES * H);
  const int j0 = sl * DVS;
  const int tid = threadIdx.x;

  extern __shared__ __align__(16) uint8_t wsm[];
  float* sS = reinterpret_cast<float*>(wsm + C::OFF_S);   // [DK][DVS]
  float* sU = reinterpret_cast<float*>(wsm + C::OFF_U);   // [64][DVS]

  const size_t state_base = ((size_t)n * H + h) * DK * DV;
  for (int idx = tid; idx < DK * DVS; idx += kWalkSimtThreads) {
    const int cc = idx / DVS, j = idx % DVS;
    sS[idx] = a.h0 ? a.h0[state_base + (size_t)cc * DV + j0 + j] : 0.f;
  }
  const int c_begin = a.map.chunk_off[n], c_end = a.map.chunk_off[n + 1];
  const int s_begin = a.map.seq_begin(n), s_end = a.map.seq_end(n);
  auto issue = [&](int c) {   // chunk c's tiles into buffer c & 1
    uint8_t* b = wsm + (c & 1) * C::BUF;
    const size_t tk = ((size_t)c * H + h) * kChunk * DK, tv = ((size_t)c * H + h) * kChunk * DV;
    constexpr int RB = DK * (int)sizeof(FT), SB = DVS * (int)sizeof(FT);
    stage_rows<RB>(b + C::OFF_W, LKF * sizeof(FT), a.W + tk, RB, kChunk, kChunk, tid, kWalkSimtThreads);
    stage_rows<RB>(b + C::OFF_KB, LKF * sizeof(FT), a.Kbar + tk, RB, kChunk, kChunk, tid, kWalkSimtThreads);
    stage_rows<RB>(b + C::OFF_QE, LKF * sizeof(FT), a.Qeff + tk, RB, kChunk, kChunk, tid, kWalkSimtThreads);
    stage_rows<SB>(b + C::OFF_UT, SB, a.Ut + tv + j0, DV * sizeof(FT), kChunk, kChunk, tid, kWalkSimtThreads);
    stage_rows<SB>(b + C::OFF_OP, SB, a.Opart + tv + j0, DV * sizeof(FT), kChunk, kChunk, tid, kWalkSimtThreads);
    stage_rows<DK * 4>(b + C::OFF_GL, 0, a.gamma_last + ((size_t)c * H + h) * DK, 0, 1, 1, tid, kWalkSimtThreads);
  };
  if (c_begin < c_end) issue(c_begin);
  cp_async_commit();

  constexpr int RS = DK / 32;                     // rows of S per thread
  const int ri = tid / 8, cj = 2 * (tid % 8);     // U, O: rows 2 ri, 2 ri + 1; columns cj, cj + 1
  const int rs = RS * (tid / 8);                 // S: rows rs .. rs + RS - 1; columns cj, cj + 1
  for (int c = c_begin; c < c_end; ++c) {
    if (c + 1 < c_end) issue(c + 1);
    cp_async_commit();
    cp_async_wait<1>();   // this chunk's copies have landed (the next chunk's may be in flight)
    __syncthreads();
    const uint8_t* b = wsm + (c & 1) * C::BUF;
    const FT* sW = reinterpret_cast<const FT*>(b + C::OFF_W);
    const FT* sKb = reinterpret_cast<const FT*>(b + C::OFF_KB);
    const FT* sQe = reinterpret_cast<const FT*>(b + C::OFF_QE);
    const FT* sUt = reinterpret_cast<const FT*>(b + C::OFF_UT);
    const FT* sOp = reinterpret_cast<const FT*>(b + C::OFF_OP);
    const float* sgl = reinterpret_cast<const float*>(b + C::OFF_GL);
    const int t0 = s_begin + (c - c_begin) * kChunk;
    const int len = min(kChunk, s_end - t0);
    if (a.chunk_states) {
      const size_t cs = ((size_t)c * H + h) * DK * DV;
      for (int idx = tid; idx < DK * DVS; idx += kWalkSimtThreads)
        a.chunk_states[cs + (size_t)(idx / DVS) * DV + j0 + idx % DVS] = sS[idx];
    }
    // U = U~ - W S and O = Q_eff S + O_part on a 2 x 2 tile
    {
      float u[2][2], o[2][2];
#pragma unroll
      for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          u[r][q] = to_f32(sUt[(2 * ri + r) * DVS + cj + q]);
          o[r][q] = to_f32(sOp[(2 * ri + r) * DVS + cj + q]);
        }
#pragma unroll 2
      for (int c4 = 0; c4 < DK; c4 += 4) {   // four key rows of S a step, W and Q_eff read as vectors
        float wv[2][4], qv[2][4];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          load_vec<4>(sW + (2 * ri + r) * LKF + c4, wv[r]);
          load_vec<4>(sQe + (2 * ri + r) * LKF + c4, qv[r]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 s = *reinterpret_cast<const float2*>(sS + (c4 + e) * DVS + cj);
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            u[r][0] = fmaf(-wv[r][e], s.x, u[r][0]); u[r][1] = fmaf(-wv[r][e], s.y, u[r][1]);
            o[r][0] = fmaf(qv[r][e], s.x, o[r][0]); o[r][1] = fmaf(qv[r][e], s.y, o[r][1]);
          }
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int i = 2 * ri + r;
        *reinterpret_cast<float2*>(sU + i * DVS + cj) = make_float2(u[r][0], u[r][1]);
        if (a.out && i < len) {
          const size_t off = ((size_t)(t0 + i) * H + h) * DV + j0 + cj;
          a.out[off] = from_f32<IO>(a.scale * o[r][0]);
          a.out[off + 1] = from_f32<IO>(a.scale * o[r][1]);
        }
      }
    }
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
    __syncthreads();   // this buffer is free for chunk c + 2
  }
  cp_async_wait<0>();
  __syncthreads();
  if (a.hT) {
    for (int idx = tid; idx < DK * DVS; idx += kWalkSimtThreads) {
      const int cc = idx / DVS, j = idx % DVS;
      a.hT[state_base + (size_t)cc * DV + j0 + j] = sS[idx];
    }
  }
}

}  // namespace gdn2
