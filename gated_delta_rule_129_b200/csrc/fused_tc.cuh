// fused_tc.cuh -- the tensor-core prep and walk in one launch.
//
// On a long sequence with few heads the walk runs on a few dozen SMs while
// the prep could use all of them, and run back to back the two add up.  Here
// one persistent grid of one CTA per SM holds both: the last n_walk CTAs walk
// (one per sequence, head and 64-column value slice), the others take prep
// tasks in chunk-major order from a shared counter.  The walk CTAs take prep
// tasks too until the counter reaches stop_at, chosen on the host so that
// the walk, started then, ends about when the prep does.  A prep CTA publishes a
// chunk's ready flag once its factors are in global memory (where they are
// still in L2 when the walk reads them); the walk's TMA warps wait for the
// flag before loading.  Only the walk waits, and only for work that the prep
// CTAs take without waiting on anyone, so the wait always ends; every wait is
// bounded all the same.
#pragma once

#include "prep_tc.cuh"
#include "walk_tc.cuh"

namespace gdn2 {

template <int DV>
struct FusedTcCfg {
  // the walk leaves the prep's extra (store) warp idle
  static constexpr int THREADS = PrepTcCfg<DV>::THREADS;
  static_assert(THREADS >= WalkTcCfg<DV>::THREADS, "one block shape for both roles");
  static constexpr int SMEM =
      PrepTcCfg<DV>::SMEM > WalkTcCfg<DV>::SMEM ? PrepTcCfg<DV>::SMEM : WalkTcCfg<DV>::SMEM;
  static constexpr int MIN_PREP_CTAS = 32;
};

template <int DV>
__global__ void __launch_bounds__(FusedTcCfg<DV>::THREADS, 1)
fused_tc_kernel(const __grid_constant__ PrepTcArgs pa, const __grid_constant__ WalkTcArgs wa, int n_prep) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = tc::smem_u32(smem_raw);
  uint8_t* sm = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  if ((int)blockIdx.x < n_prep) {
    prep_tc_cta<DV>(pa, sm, blockIdx.x, n_prep);
  } else {
    // early on, the walk would only wait for the prep wavefront: take prep
    // tasks until the counter reaches pa.stop_at, then walk
    if (pa.stop_at > 0) prep_tc_cta<DV>(pa, sm, blockIdx.x, gridDim.x, true);
    walk_tc_cta<DV>(wa, sm, (int)blockIdx.x - n_prep);
  }
}

}  // namespace gdn2
