// segscan.cuh -- the two-level chunk scan: segment bookkeeping and the scan
// of the segments' affine state maps.
//
// Long sequences walk their chunks one after the other, so the state walk of
// one (sequence, head) is a serial chain of T/64 steps.  The two-level form
// splits each sequence into segments of L chunks (virtual sequences), and
//   1. walks every segment from [I | 0] in parallel (walk_tc map mode),
//      giving its affine map S_end = Phi_s S_start + Psi_s;
//   2. scans the maps of each sequence in order from h0 (this file, fp32 on
//      the CUDA cores): S_{s+1} = Phi_s S_s + Psi_s, giving every segment its
//      true start state and the sequence its final state;
//   3. walks every segment again, with outputs, from its start state.
// The recurrence is affine in the state over any range of tokens (page
// "Gated DeltaNet-2：将擦除与写入分开", section "在两个维度上独立控制"), so
// this is the same computation reordered; the pages' chunking is 64 tokens
// (section "词元路径与并行训练").  Segments start on chunk boundaries, so the
// chunk factors of the prep are shared by all three steps.
#pragma once

#include "common.cuh"

namespace gdn2 {

constexpr int kSegPlanThreads = 1024;

// Virtual segments of L chunks.  chunk_off [N + 1] comes from plan_kernel (in
// the same stream); a malformed cu_seqlens left it all zero, so every sequence
// has no segment.  Writes seg_cu [ns_max + 1] (token bounds of each segment,
// a refinement of the sequences' bounds), seg_chunk [ns_max + 1] (global
// index of each segment's first chunk) and seq_seg [N + 1] (first segment of
// each sequence); entries past the last segment describe empty segments.
__global__ void __launch_bounds__(kSegPlanThreads)
segplan_kernel(const int32_t* __restrict__ cu, int N, int T_dense, int T_total, const int32_t* __restrict__ chunk_off,
               int L, int ns_max, int32_t* __restrict__ seg_cu, int32_t* __restrict__ seg_chunk,
               int32_t* __restrict__ seq_seg) {
  __shared__ int s_scan[kSegPlanThreads];
  const int tid = threadIdx.x;
  const int per = (N + kSegPlanThreads - 1) / kSegPlanThreads;
  const int n0 = min(N, tid * per), n1 = min(N, n0 + per);
  int count = 0;
  for (int n = n0; n < n1; ++n) count += (chunk_off[n + 1] - chunk_off[n] + L - 1) / L;
  s_scan[tid] = count;
  __syncthreads();
  for (int o = 1; o < kSegPlanThreads; o <<= 1) {
    const int add = tid >= o ? s_scan[tid - o] : 0;
    __syncthreads();
    s_scan[tid] += add;
    __syncthreads();
  }
  const int total = s_scan[kSegPlanThreads - 1];
  int s = s_scan[tid] - count;
  for (int n = n0; n < n1; ++n) {
    seq_seg[n] = s;
    const int b = cu ? cu[n] : n * T_dense;
    const int nch = chunk_off[n + 1] - chunk_off[n];
    for (int j = 0; j * L < nch; ++j, ++s) {
      seg_cu[s] = b + j * L * kChunk;
      seg_chunk[s] = chunk_off[n] + j * L;
    }
  }
  if (tid == 0) seq_seg[N] = total;
  // the end of the last segment, and empty segments up to ns_max
  for (int i = total + tid; i <= ns_max; i += kSegPlanThreads) {
    seg_cu[i] = T_total;
    seg_chunk[i] = chunk_off[N];
  }
}

constexpr int kScanThreads = 256;
constexpr int kScanCols = 32;   // value columns per block

// Step 2: per (sequence, head, 32 value columns), in segment order,
//   seg_h0[s] = S;  S <- Phi_s S + Psi_s,
// starting from h0 (or zero); the final S goes to hT (if given).  fp32
// throughout: the state never passes through bf16 here.  Thread t owns key
// row t / 2 and 16 of the block's columns; S lives in shared memory, Phi
// rows are read from global memory.
template <int DK, int DV>
__global__ void __launch_bounds__(kScanThreads)
segscan_kernel(const float* __restrict__ phi, const float* __restrict__ psi, const int32_t* __restrict__ seq_seg,
               int H, const float* __restrict__ h0, float* __restrict__ seg_h0, float* __restrict__ hT) {
  static_assert(DK * kScanCols == kScanThreads * 16, "one row x 16 columns per thread");
  __shared__ __align__(16) float sS[DK][kScanCols];
  constexpr int CB = DV / kScanCols;
  const int blk = blockIdx.x;
  const int cb = blk % CB, h = (blk / CB) % H, n = blk / (CB * H);
  const int t = threadIdx.x, i = t >> 1, c0 = (t & 1) * 16;
  const int col = cb * kScanCols + c0;
  float S[16];
  {
    const float* src = h0 ? h0 + (((size_t)n * H + h) * DK + i) * DV + col : nullptr;
#pragma unroll
    for (int e = 0; e < 16; e += 4) {
      const float4 v = src ? *reinterpret_cast<const float4*>(src + e) : make_float4(0.f, 0.f, 0.f, 0.f);
      S[e] = v.x; S[e + 1] = v.y; S[e + 2] = v.z; S[e + 3] = v.w;
    }
  }
  const int s0 = seq_seg[n], s1 = seq_seg[n + 1];
  for (int s = s0; s < s1; ++s) {
    float* dst = seg_h0 + (((size_t)s * H + h) * DK + i) * DV + col;
#pragma unroll
    for (int e = 0; e < 16; e += 4) {
      *reinterpret_cast<float4*>(dst + e) = make_float4(S[e], S[e + 1], S[e + 2], S[e + 3]);
      *reinterpret_cast<float4*>(&sS[i][c0 + e]) = make_float4(S[e], S[e + 1], S[e + 2], S[e + 3]);
    }
    __syncthreads();
    const float* prow = phi + (((size_t)s * H + h) * DK + i) * DK;
    const float* qrow = psi + (((size_t)s * H + h) * DK + i) * DV + col;
    float acc[16];
#pragma unroll
    for (int e = 0; e < 16; e += 4) {
      const float4 v = *reinterpret_cast<const float4*>(qrow + e);
      acc[e] = v.x; acc[e + 1] = v.y; acc[e + 2] = v.z; acc[e + 3] = v.w;
    }
    for (int j0 = 0; j0 < DK; j0 += 4) {
      const float4 p4 = *reinterpret_cast<const float4*>(prow + j0);
      const float pj[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
          const float4 sv = *reinterpret_cast<const float4*>(&sS[j0 + jj][c0 + e]);
          acc[e] = fmaf(pj[jj], sv.x, acc[e]);
          acc[e + 1] = fmaf(pj[jj], sv.y, acc[e + 1]);
          acc[e + 2] = fmaf(pj[jj], sv.z, acc[e + 2]);
          acc[e + 3] = fmaf(pj[jj], sv.w, acc[e + 3]);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 16; ++e) S[e] = acc[e];
    __syncthreads();
  }
  if (hT) {
    float* dst = hT + (((size_t)n * H + h) * DK + i) * DV + col;
#pragma unroll
    for (int e = 0; e < 16; e += 4)
      *reinterpret_cast<float4*>(dst + e) = make_float4(S[e], S[e + 1], S[e + 2], S[e + 3]);
  }
}

}  // namespace gdn2
