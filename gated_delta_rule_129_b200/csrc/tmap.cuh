// tmap.cuh -- host-side creation of TMA tensor maps (cuTensorMapEncodeTiled),
// reached through the runtime's driver entry point so the library does not
// link libcuda directly.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

namespace gdn2 {

inline PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// A 2-D (or 3-D) row-major tensor map.  dims[0] is the innermost extent in
// elements, strides are in bytes for dims 1.. (multiples of 16), box sizes in
// elements.  Returns false if the driver rejects the description.
inline bool make_tmap(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int rank, const uint64_t* dims,
                      const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapSwizzle swz) {
  auto enc = tmap_encoder();
  if (!enc) return false;
  uint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUresult r = enc(m, dt, (cuuint32_t)rank, const_cast<void*>(base), (const cuuint64_t*)dims,
                         (const cuuint64_t*)strides_bytes, (const cuuint32_t*)box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace gdn2
