// tc_probe.cu -- test-only kernels that check the sm_100a building blocks in
// gated_delta_rule_129_b200/csrc/tc.cuh on their own: one UMMA (tcgen05.mma
// kind::f16) per operand layout the kernels use, and the byte image a TMA
// SWIZZLE_128B load leaves in shared memory.  Every shared-memory address is
// inside the 64 KiB operand area; waits are bounded and report a status.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tc.cuh"
#include "tmap.cuh"

using namespace gdn2::tc;

namespace {

enum Lay { KSW = 0, MNSW = 1, MNIL = 2 };
struct Mode {
  int M, N, K, la, lb;
};
__host__ __device__ inline Mode mode_of(int m) {
  switch (m) {
    case 0: return {128, 16, 128, KSW, KSW};
    case 1: return {128, 128, 128, KSW, MNSW};
    case 2: return {128, 128, 64, MNSW, MNSW};
    case 3: return {64, 128, 128, KSW, MNSW};
    case 4: return {128, 16, 128, KSW, MNIL};
    case 5: return {64, 128, 64, KSW, MNSW};
    case 6: return {128, 32, 128, KSW, KSW};
    case 7: return {128, 64, 64, MNSW, MNIL};
    default: return {0, 0, 0, 0, 0};
  }
}

// byte offset of operand element (row r of R rows, k) for a K-major operand,
// or (k, mn) of an MN-major operand with `MNext` columns and `K` rows.
__device__ inline uint32_t off_k_sw(int R, int r, int k) { return (k / 64) * R * 128 + sw128_off(r, k % 64); }
__device__ inline uint32_t off_mn_sw(int K, int k, int mn) { return (mn / 64) * K * 128 + sw128_off(k, mn % 64); }
__device__ inline uint32_t il_lbo(int MNext) { return (MNext / 8) * 128; }

__device__ inline uint64_t desc_for(int lay, uint32_t base, int rows_or_k, int mn_ext, int K, int s) {
  if (lay == KSW) {
    const int k0 = s * 16;
    return sdesc(base + (k0 / 64) * rows_or_k * 128 + (k0 % 64) * 2, 16, 1024, kLayoutSW128);
  } else if (lay == MNSW) {
    return sdesc(base + s * 16 * 128, K * 128, 1024, kLayoutSW128);
  } else {
    const uint32_t lbo = il_lbo(mn_ext);
    return sdesc(base + s * 2 * lbo, lbo, 128, kLayoutNone);
  }
}

__global__ void __launch_bounds__(128) umma_probe_kernel(int mode, const __nv_bfloat16* A,
                                                         const __nv_bfloat16* B, float* D, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const Mode md = mode_of(mode);
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  uint8_t* sA = smem_raw + pad;
  uint8_t* sB = sA + 32768;
  uint64_t* bar = reinterpret_cast<uint64_t*>(sB + 32768);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bar + 1);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int i = tid; i < md.M * md.K; i += 128) {
    const int r = i / md.K, k = i % md.K;  // A is M x K row-major in global
    const uint32_t off = md.la == KSW ? off_k_sw(md.M, r, k) : off_mn_sw(md.K, k, r);
    *reinterpret_cast<__nv_bfloat16*>(sA + off) = A[i];
  }
  for (int i = tid; i < md.K * md.N; i += 128) {
    const int k = i / md.N, n = i % md.N;  // B is K x N row-major in global
    uint32_t off;
    if (md.lb == KSW) off = off_k_sw(md.N, n, k);
    else if (md.lb == MNSW) off = off_mn_sw(md.K, k, n);
    else off = il_mn_off(k, n, il_lbo(md.N), 128);
    *reinterpret_cast<__nv_bfloat16*>(sB + off) = B[i];
  }
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tslot, 128);
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  if (tid == 0) {
    const uint32_t idesc = idesc_bf16(md.M, md.N, md.la != KSW, md.lb != KSW);
    for (int s = 0; s < md.K / 16; ++s) {
      const uint64_t ad = desc_for(md.la, smem_u32(sA), md.M, md.M, md.K, s);
      const uint64_t bd = desc_for(md.lb, smem_u32(sB), md.N, md.N, md.K, s);
      umma_f16(tbase, ad, bd, idesc, s > 0);
    }
    umma_commit(bar);
  }
  const bool ok = mbar_wait(bar, 0);
  if (!ok && lane == 0) atomicExch(status, 1);
  tc_fence_after();
  if (ok) {
    for (int c0 = 0; c0 < md.N; c0 += 16) {
      float v[16];
      tmem_ld16(tmem_addr(tbase, 32 * warp, c0), v);
      tmem_wait_ld();
      int row = -1;
      if (md.M == 128) row = 32 * warp + lane;
      else if (lane < 16) row = 16 * warp + lane;
      if (row >= 0)
        for (int i = 0; i < 16; ++i) D[row * md.N + c0 + i] = v[i];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 128);
    tmem_relinquish();
  }
}

__global__ void tma_probe_kernel(const __grid_constant__ CUtensorMap tmap, int c0, int c1, int rows,
                                 uint8_t* out, int* status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* s = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(s + 16384);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar, rows * 128);
    tma_load_2d(s, &tmap, bar, c0, c1);
  }
  const bool ok = mbar_wait(bar, 0);
  if (!ok && threadIdx.x == 0) atomicExch(status, 1);
  if (ok)
    for (int i = threadIdx.x; i < rows * 128; i += blockDim.x) out[i] = s[i];
}

}  // namespace

extern "C" {

int probe_mode_shape(int mode, int* M, int* N, int* K) {
  const Mode m = mode_of(mode);
  *M = m.M;
  *N = m.N;
  *K = m.K;
  return m.M ? 0 : 1;
}

int probe_umma(int mode, const void* A, const void* B, float* D, int* status) {
  if (mode_of(mode).M == 0) return 1;
  const int smem = 65536 + 1024 + 64;
  if (cudaFuncSetAttribute(umma_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 2;
  umma_probe_kernel<<<1, 128, smem>>>(mode, (const __nv_bfloat16*)A, (const __nv_bfloat16*)B, D, status);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

// Load the box {64 columns, rows} at (c0, c1) of a [height, width] bf16
// row-major tensor with SWIZZLE_128B; copy the raw shared-memory image out.
int probe_tma(const void* src, int width, int height, int c0, int c1, int rows, void* out, int* status) {
  if (rows < 1 || rows > 128 || width % 8 != 0) return 1;
  CUtensorMap m;
  const uint64_t dims[2] = {(uint64_t)width, (uint64_t)height};
  const uint64_t strides[1] = {(uint64_t)width * 2};
  const uint32_t box[2] = {64, (uint32_t)rows};
  if (!gdn2::make_tmap(&m, src, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dims, strides, box,
                       CU_TENSOR_MAP_SWIZZLE_128B))
    return 2;
  const int smem = 16384 + 1024 + 64;
  tma_probe_kernel<<<1, 128, smem>>>(m, c0, c1, rows, (uint8_t*)out, status);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

}  // extern "C"
