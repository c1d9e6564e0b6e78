// plan.cuh -- chunk bookkeeping on the device.
//
// cu_seqlens lives in device memory, so the chunk offsets of each sequence are
// computed on the device (no host round trip, no stream synchronisation).  One
// block of 1024 threads: each thread owns a contiguous run of sequences,
// checks them, counts their 64-token chunks, and a block-wide exclusive scan
// turns the counts into chunk_off[0..N].  A malformed cu_seqlens (first entry
// not 0, a decreasing pair, or a last entry other than the total token count)
// stores GDN2_ERR_SEQLENS in the status word and zero chunks for every
// sequence, so no later kernel touches the token arrays.  It also clears the
// handed-back list and the flags the fused prep + walk synchronise on.
#pragma once

#include "common.cuh"

namespace gdn2 {

constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(const int32_t* __restrict__ cu, int N, int T_dense, int T_total,
            int32_t* __restrict__ chunk_off, int32_t* __restrict__ status, int err_code,
            int32_t* __restrict__ fix_count, int32_t* __restrict__ sync, int n_sync) {
  __shared__ int s_scan[kPlanThreads];
  __shared__ int s_bad;
  const int tid = threadIdx.x;
  if (tid == 0) s_bad = 0;
  __syncthreads();
  const int per = (N + kPlanThreads - 1) / kPlanThreads;
  const int n0 = min(N, tid * per), n1 = min(N, n0 + per);
  int count = 0;
  bool bad = false;
  for (int n = n0; n < n1; ++n) {
    const int b = cu ? cu[n] : n * T_dense;
    const int e = cu ? cu[n + 1] : (n + 1) * T_dense;
    if (e < b) bad = true;
    else count += (e - b + kChunk - 1) / kChunk;
  }
  if (cu && tid == 0 && (cu[0] != 0 || cu[N] != T_total)) bad = true;
  if (bad) atomicOr(&s_bad, 1);
  s_scan[tid] = count;
  __syncthreads();
  // Hillis-Steele inclusive scan over the per-thread counts.
  for (int o = 1; o < kPlanThreads; o <<= 1) {
    const int add = tid >= o ? s_scan[tid - o] : 0;
    __syncthreads();
    s_scan[tid] += add;
    __syncthreads();
  }
  const bool any_bad = s_bad != 0;
  int run = any_bad ? 0 : s_scan[tid] - count;
  for (int n = n0; n < n1; ++n) {
    chunk_off[n] = run;
    if (!any_bad) {
      const int b = cu ? cu[n] : n * T_dense;
      const int e = cu ? cu[n + 1] : (n + 1) * T_dense;
      run += (e - b + kChunk - 1) / kChunk;
    }
  }
  if (tid == kPlanThreads - 1) chunk_off[N] = any_bad ? 0 : s_scan[tid];
  if (tid == 0) {
    *status = any_bad ? err_code : 0;
    if (fix_count) *fix_count = 0;
  }
  // task counter, redo flag and ready flags of the fused prep + walk
  for (int i = tid; i < n_sync; i += kPlanThreads) sync[i] = 0;
}

}  // namespace gdn2
