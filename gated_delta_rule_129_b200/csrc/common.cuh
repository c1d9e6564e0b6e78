// common.cuh -- small device helpers shared by the Gated DeltaNet-2 kernels.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn2 {

// Chunk length of the WY form (page "Gated DeltaNet-2：将擦除与写入分开",
// section "词元路径与并行训练": training uses 64-token chunks).
constexpr int kChunk = 64;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// acc + (a, a) * b on a pair of fp32 values as one packed FMA (sm_100's
// f32x2 FMA; each component is rounded exactly like fmaf, so a loop that
// keeps each output's order of terms gives the same bits as with fmaf).
__device__ __forceinline__ float2 fma2s(float a, float2 b, float2 acc) {
  return __ffma2_rn(make_float2(a, a), b, acc);
}

// The two bf16 values packed in a 32-bit word, as fp32 (exact).
__device__ __forceinline__ float bf16_lo_f(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Asynchronous 16-byte global -> shared copies (cp.async, completion per
// thread by commit groups; a barrier after the wait makes them visible).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }
__device__ __forceinline__ void cp_async_wait_all() {
  cp_async_commit();
  cp_async_wait<0>();
}

// Rows [0, rows) of a row-major global array (row stride gstride bytes) into
// shared memory (row stride sstride bytes), BYTES per row (a multiple of 16,
// both addresses 16-byte aligned), by threads tid of nthr; rows >= valid are
// written as zeros instead of read.
template <int BYTES>
__device__ __forceinline__ void stage_rows(void* dst, int sstride, const void* src, size_t gstride, int rows,
                                           int valid, int tid, int nthr) {
  static_assert(BYTES % 16 == 0, "16-byte pieces");
  constexpr int PER = BYTES / 16;
  for (int idx = tid; idx < rows * PER; idx += nthr) {
    const int r = idx / PER, u = idx % PER;
    char* d = static_cast<char*>(dst) + r * sstride + u * 16;
    if (r < valid) cp_async16(d, static_cast<const char*>(src) + r * gstride + u * 16);
    else *reinterpret_cast<uint4*>(d) = make_uint4(0u, 0u, 0u, 0u);
  }
}

// N consecutive elements (N = 2 or 4, the address a multiple of their size)
// of a shared-memory row of fp32 or bf16, as fp32.
template <int N>
__device__ __forceinline__ void load_vec(const float* p, float (&o)[N]) {
  if constexpr (N == 4) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
  } else {
    static_assert(N == 2, "2 or 4");
    const float2 v = *reinterpret_cast<const float2*>(p);
    o[0] = v.x; o[1] = v.y;
  }
}
template <int N>
__device__ __forceinline__ void load_vec(const __nv_bfloat16* p, float (&o)[N]) {
  if constexpr (N == 4) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    o[0] = bf16_lo_f(v.x); o[1] = bf16_hi_f(v.x); o[2] = bf16_lo_f(v.y); o[3] = bf16_hi_f(v.y);
  } else {
    static_assert(N == 2, "2 or 4");
    const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
    o[0] = bf16_lo_f(v); o[1] = bf16_hi_f(v);
  }
}

// N consecutive fp32 or bf16 elements of global memory (16-byte aligned, N a
// multiple of 16 bytes' worth) as fp32, by 16-byte loads.
template <int N>
__device__ __forceinline__ void ldg_vec(const float* p, float (&o)[N]) {
  static_assert(N % 4 == 0, "16-byte pieces");
#pragma unroll
  for (int j = 0; j < N / 4; ++j) {
    const float4 v = *reinterpret_cast<const float4*>(p + 4 * j);
    o[4 * j] = v.x; o[4 * j + 1] = v.y; o[4 * j + 2] = v.z; o[4 * j + 3] = v.w;
  }
}
template <int N>
__device__ __forceinline__ void ldg_vec(const __nv_bfloat16* p, float (&o)[N]) {
  static_assert(N % 8 == 0, "16-byte pieces");
#pragma unroll
  for (int j = 0; j < N / 8; ++j) {
    const uint4 v = *reinterpret_cast<const uint4*>(p + 8 * j);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      o[8 * j + 2 * e] = bf16_lo_f(w[e]);
      o[8 * j + 2 * e + 1] = bf16_hi_f(w[e]);
    }
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Sequence bookkeeping shared by every chunked kernel.  Sequence n covers
// tokens [seq_begin(n), seq_end(n)); its chunks are global indices
// [chunk_off[n], chunk_off[n+1]) and chunk j of it starts at token
// seq_begin(n) + 64 j.
struct SeqMap {
  const int32_t* cu;        // packed boundaries or nullptr (dense)
  const int32_t* chunk_off; // [N + 1], written by the plan kernel
  int N;                    // sequences
  int T;                    // dense tokens per sequence (unused when packed)

  __device__ __forceinline__ int seq_begin(int n) const { return cu ? cu[n] : n * T; }
  __device__ __forceinline__ int seq_end(int n) const { return cu ? cu[n + 1] : (n + 1) * T; }

  // The sequence owning global chunk c (c < chunk_off[N]): the largest n with
  // chunk_off[n] <= c; empty sequences (equal offsets) are skipped over.
  __device__ __forceinline__ int seq_of_chunk(int c) const {
    int lo = 0, hi = N - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (chunk_off[mid] <= c) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
};

// Where one chunk sits in the token stream.
struct ChunkPos {
  int seq, t0, len;
};

__device__ __forceinline__ ChunkPos chunk_pos(const SeqMap& m, int c) {
  ChunkPos p;
  p.seq = m.seq_of_chunk(c);
  const int j = c - m.chunk_off[p.seq];
  p.t0 = m.seq_begin(p.seq) + j * kChunk;
  p.len = min(kChunk, m.seq_end(p.seq) - p.t0);
  return p;
}

}  // namespace gdn2
