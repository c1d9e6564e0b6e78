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

template <int DK, int DV>
constexpr size_t walk_simt_smem_bytes() {
  return sizeof(float) * (size_t)(3 * kChunk * (DK + 1) + DK * kWalkSimtDVS + 3 * kChunk * kWalkSimtDVS + DK);
}

template <int DK, int DV, typename IO, typename FT>
__global__ void __launch_bounds__(kWalkSimtThreads)
walk_simt_kernel(const WalkArgs<IO, FT> a) {
  constexpr int DVS = kWalkSimtDVS;
  constexpr int SLICES = DV / DVS;
  constexpr int LK = DK + 1;
  const int H = a.H;
  const int sl = blockIdx.x % SLICES;
  const int h = (blockIdx.x / SLICES) % H;
  const int n = blockIdx.x / (SLICES * H);
  const int j0 = sl * DVS;
  const int tid = threadIdx.x;

  extern __shared__ float smem[];
  float* sW = smem;                 // [64][LK]
  float* sKb = sW + kChunk * LK;    // [64][LK]
  float* sQe = sKb + kChunk * LK;   // [64][LK]
  float* sS = sQe + kChunk * LK;    // [DK][DVS] state slice
  float* sUt = sS + DK * DVS;       // [64][DVS]
  float* sOp = sUt + kChunk * DVS;  // [64][DVS]
  float* sU = sOp + kChunk * DVS;   // [64][DVS]
  float* sgl = sU + kChunk * DVS;   // [DK]

  const size_t state_base = ((size_t)n * H + h) * DK * DV;
  for (int idx = tid; idx < DK * DVS; idx += kWalkSimtThreads) {
    const int cc = idx / DVS, j = idx % DVS;
    sS[idx] = a.h0 ? a.h0[state_base + (size_t)cc * DV + j0 + j] : 0.f;
  }
  const int c_begin = a.map.chunk_off[n], c_end = a.map.chunk_off[n + 1];
  const int s_begin = a.map.seq_begin(n), s_end = a.map.seq_end(n);
  for (int c = c_begin; c < c_end; ++c) {
    const int t0 = s_begin + (c - c_begin) * kChunk;
    const int len = min(kChunk, s_end - t0);
    const size_t tile_k = ((size_t)c * H + h) * kChunk * DK;
    const size_t tile_v = ((size_t)c * H + h) * kChunk * DV;
    __syncthreads();  // previous chunk's readers of the tiles are done
    for (int idx = tid; idx < kChunk * DK; idx += kWalkSimtThreads) {
      const int i = idx / DK, cc = idx % DK;
      sW[i * LK + cc] = to_f32(a.W[tile_k + idx]);
      sKb[i * LK + cc] = to_f32(a.Kbar[tile_k + idx]);
      sQe[i * LK + cc] = to_f32(a.Qeff[tile_k + idx]);
    }
    for (int idx = tid; idx < kChunk * DVS; idx += kWalkSimtThreads) {
      const int i = idx / DVS, j = idx % DVS;
      sUt[idx] = to_f32(a.Ut[tile_v + (size_t)i * DV + j0 + j]);
      sOp[idx] = to_f32(a.Opart[tile_v + (size_t)i * DV + j0 + j]);
    }
    if (tid < DK) sgl[tid] = a.gamma_last[((size_t)c * H + h) * DK + tid];
    if (a.chunk_states) {
      const size_t cs = ((size_t)c * H + h) * DK * DV;
      for (int idx = tid; idx < DK * DVS; idx += kWalkSimtThreads)
        a.chunk_states[cs + (size_t)(idx / DVS) * DV + j0 + idx % DVS] = sS[idx];
    }
    __syncthreads();
    for (int idx = tid; idx < kChunk * DVS; idx += kWalkSimtThreads) {
      const int i = idx / DVS, j = idx % DVS;
      float u = sUt[idx], o = sOp[idx];
#pragma unroll 8
      for (int cc = 0; cc < DK; ++cc) {
        const float s = sS[cc * DVS + j];
        u = fmaf(-sW[i * LK + cc], s, u);
        o = fmaf(sQe[i * LK + cc], s, o);
      }
      sU[idx] = u;
      if (a.out && i < len) a.out[((size_t)(t0 + i) * H + h) * DV + j0 + j] = from_f32<IO>(a.scale * o);
    }
    __syncthreads();
    for (int idx = tid; idx < DK * DVS; idx += kWalkSimtThreads) {
      const int cc = idx / DVS, j = idx % DVS;
      float s = sgl[cc] * sS[idx];
      for (int i = 0; i < len; ++i) s = fmaf(sKb[i * LK + cc], sU[i * DVS + j], s);
      sS[idx] = s;
    }
  }
  __syncthreads();
  if (a.hT) {
    for (int idx = tid; idx < DK * DVS; idx += kWalkSimtThreads) {
      const int cc = idx / DVS, j = idx % DVS;
      a.hT[state_base + (size_t)cc * DV + j0 + j] = sS[idx];
    }
  }
}

}  // namespace gdn2
