// gdn2_api.cu -- the C ABI declared in include/gdn2.h.
//
// Host side only: argument checks (no CUDA call happens before they pass),
// workspace carving, and dispatch of the kernels for (dk, dv, io dtype).
// Nothing here allocates device memory or synchronises a stream.
#include "gdn2.h"

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <type_traits>

#include "bwd_chunk.cuh"
#include "common.cuh"
#include "decode.cuh"
#include "plan.cuh"
#include "prep_simt.cuh"
#include "prep_tc.cuh"
#include "fused_tc.cuh"
#include "segscan.cuh"
#include "token_path.cuh"
#include "tmap.cuh"
#include "walk_simt.cuh"
#include "walk_tc.cuh"

namespace {

using bf16 = __nv_bfloat16;
using gdn2::kChunk;

constexpr size_t kAlign = 256;
int sm_count();
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gdn2_status check_dims(const gdn2_desc* d, bool packed) {
  if (!d) return GDN2_ERR_NULL;
  if (d->io != GDN2_IO_F32 && d->io != GDN2_IO_BF16) return GDN2_ERR_DTYPE;
  if ((d->dk != 64 && d->dk != 128) || (d->dv != 64 && d->dv != 128)) return GDN2_ERR_SHAPE;
  if (d->H < 1 || d->B < 1 || d->T < 0) return GDN2_ERR_SHAPE;
  // packed calls describe num_seqs >= 1 sequences in one row; dense calls
  // leave num_seqs at 0 (this keeps gdn2_workspace_size consistent)
  if (packed && (d->B != 1 || d->num_seqs < 1)) return GDN2_ERR_SHAPE;
  if (!packed && d->num_seqs != 0) return GDN2_ERR_SHAPE;
  // all token-level indices are computed in 64-bit, but token and chunk
  // counts themselves must fit in int32
  const long long tokens = (long long)d->B * d->T;
  if (tokens > INT32_MAX / 2) return GDN2_ERR_SHAPE;
  return GDN2_OK;
}

struct Layout {
  gdn2_ws_layout l;
  int N;
};

// The bf16 path with dk = 128 stores each chunk's affine state map and walks
// with one tensor-core product per chunk; every other case stores the WY
// factors and walks on CUDA cores.
bool uses_affine(const gdn2_desc* d) { return d->io == GDN2_IO_BF16 && d->dk == 128; }

gdn2_status make_layout(const gdn2_desc* d, bool packed, Layout* out) {
  gdn2_status st = check_dims(d, packed);
  if (st != GDN2_OK) return st;
  const int N = packed ? d->num_seqs : d->B;
  const long long tokens = (long long)d->B * d->T;
  const long long max_chunks =
      packed ? tokens / kChunk + N : (long long)d->B * ((d->T + kChunk - 1) / kChunk);
  if (max_chunks > INT32_MAX / 2) return GDN2_ERR_SHAPE;
  gdn2_ws_layout& L = out->l;
  std::memset(&L, 0, sizeof(L));
  L.max_chunks = (int)max_chunks;
  L.factor_elem_bytes = d->io == GDN2_IO_F32 ? 4 : 2;
  L.factor_set = uses_affine(d) ? 1 : 0;
  const bool wy = L.factor_set == 0;
  const size_t tiles = (size_t)max_chunks * d->H * kChunk;
  const size_t mats = (size_t)max_chunks * d->H * d->dk;
  const size_t eb = (size_t)L.factor_elem_bytes;
  size_t off = 0;
  L.off_W = off;          off = align_up(off + (wy ? tiles * d->dk * eb : 0));
  L.off_Ut = off;         off = align_up(off + (wy ? tiles * d->dv * eb : 0));
  L.off_Kbar = off;       off = align_up(off + (wy ? tiles * d->dk * eb : 0));
  L.off_Qeff = off;       off = align_up(off + tiles * d->dk * eb);
  L.off_Opart = off;      off = align_up(off + tiles * d->dv * eb);
  L.off_gamma_last = off; off = align_up(off + (size_t)max_chunks * d->H * d->dk * sizeof(float));
  L.off_Mp = off;         off = align_up(off + (wy ? 0 : mats * d->dk * eb));
  L.off_Nc = off;         off = align_up(off + (wy ? 0 : mats * d->dv * eb));
  L.off_chunk_offsets = off; off = align_up(off + (size_t)(N + 1) * sizeof(int32_t));
  L.off_status = off;     off = align_up(off + sizeof(int32_t));
  L.off_fix = off;        off = align_up(off + (wy ? 0 : (size_t)(1 + (size_t)max_chunks * d->H) * sizeof(int32_t)));
  L.off_sync = off;       off = align_up(off + (wy ? 0 : (size_t)(2 + (size_t)max_chunks * d->H) * sizeof(int32_t)));
  L.off_colscale = off;   off = align_up(off + (wy ? 0 : (size_t)max_chunks * d->H * d->dk * sizeof(float)));
  L.total_bytes = off;
  out->N = N;
  return GDN2_OK;
}

gdn2_status check_workspace(const gdn2_desc* d, const Layout& L) {
  if (!d->workspace) return GDN2_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(d->workspace) & (kAlign - 1)) != 0) return GDN2_ERR_ALIGN;
  if (d->workspace_bytes < L.l.total_bytes) return GDN2_ERR_WORKSPACE;
  return GDN2_OK;
}

gdn2_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? GDN2_OK : GDN2_ERR_CUDA;
}

template <typename T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

gdn2::SeqMap seq_map(const gdn2_desc* d, const Layout& L, const int32_t* cu) {
  gdn2::SeqMap m;
  m.cu = cu;
  m.chunk_off = at<const int32_t>(d->workspace, L.l.off_chunk_offsets);
  m.N = L.N;
  m.T = d->T;
  return m;
}

gdn2_status launch_plan(const gdn2_desc* d, const Layout& L, const int32_t* cu, cudaStream_t s) {
  const bool affine = L.l.factor_set == 1;
  gdn2::plan_kernel<<<1, gdn2::kPlanThreads, 0, s>>>(
      cu, L.N, d->T, d->B * d->T, at<int32_t>(d->workspace, L.l.off_chunk_offsets),
      at<int32_t>(d->workspace, L.l.off_status), (int)GDN2_ERR_SEQLENS,
      affine ? at<int32_t>(d->workspace, L.l.off_fix) : nullptr,
      affine ? at<int32_t>(d->workspace, L.l.off_sync) : nullptr, affine ? 2 + L.l.max_chunks * d->H : 0);
  return launch_status();
}

// ------------------------------------------------------- prep (tensor) ----
// bf16 I/O with dk = 128: gate prep, intra-chunk WY and the affine state map
// on the tensor cores.
template <int DV>
gdn2_status fill_prep_tc(const gdn2_desc* d, const Layout& L, const void* q, const void* k, const void* v,
                         const float* la, const float* b, const float* w, const int32_t* cu, gdn2::PrepTcArgs& a) {
  using C = gdn2::PrepTcCfg<DV>;
  std::memset(&a, 0, sizeof(a));
  const uint64_t T_total = (uint64_t)d->B * d->T;
  const uint64_t dk[3] = {128, (uint64_t)d->H, T_total}, dv[3] = {(uint64_t)DV, (uint64_t)d->H, T_total};
  const uint64_t sk2[2] = {128 * 2, (uint64_t)d->H * 128 * 2}, sk4[2] = {128 * 4, (uint64_t)d->H * 128 * 4};
  const uint64_t sv2[2] = {(uint64_t)DV * 2, (uint64_t)d->H * DV * 2}, sv4[2] = {(uint64_t)DV * 4, (uint64_t)d->H * DV * 4};
  const uint32_t bk[3] = {32, 1, 64}, bv[3] = {(uint32_t)C::VS, 1, 64};
  const CUtensorMapDataType BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, F32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const CUtensorMapSwizzle NS = CU_TENSOR_MAP_SWIZZLE_NONE;
  if (!gdn2::make_tmap(&a.tm_q, q, BF, 3, dk, sk2, bk, NS) || !gdn2::make_tmap(&a.tm_k, k, BF, 3, dk, sk2, bk, NS) ||
      !gdn2::make_tmap(&a.tm_v, v, BF, 3, dv, sv2, bv, NS) ||
      !gdn2::make_tmap(&a.tm_la, la, F32, 3, dk, sk4, bk, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !gdn2::make_tmap(&a.tm_b, b, F32, 3, dk, sk4, bk, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !gdn2::make_tmap(&a.tm_w, w, F32, 3, dv, sv4, bv, C::W_SWIZZLED ? CU_TENSOR_MAP_SWIZZLE_128B : NS))
    return GDN2_ERR_CUDA;
  {
    const long long rows_k = (long long)std::max(L.l.max_chunks, 1) * d->H * 128;
    if (rows_k >= (1ll << 31)) return GDN2_ERR_SHAPE;  // TMA coordinates are int32
    const uint64_t d_mp[2] = {128, (uint64_t)rows_k}, d_nc[2] = {(uint64_t)DV, (uint64_t)rows_k};
    const uint64_t d_qe[2] = {128, (uint64_t)rows_k / 2}, d_op[2] = {(uint64_t)DV, (uint64_t)rows_k / 2};
    const uint64_t st_k[1] = {256}, st_v[1] = {(uint64_t)DV * 2};
    const uint32_t b_k[2] = {64, 128}, b_t[2] = {64, 64};
    const CUtensorMapSwizzle SW = CU_TENSOR_MAP_SWIZZLE_128B;
    if (!gdn2::make_tmap(&a.tm_Mp, at<void>(d->workspace, L.l.off_Mp), BF, 2, d_mp, st_k, b_k, SW) ||
        !gdn2::make_tmap(&a.tm_Nc, at<void>(d->workspace, L.l.off_Nc), BF, 2, d_nc, st_v, b_k, SW) ||
        !gdn2::make_tmap(&a.tm_Qe, at<void>(d->workspace, L.l.off_Qeff), BF, 2, d_qe, st_k, b_t, SW) ||
        !gdn2::make_tmap(&a.tm_Op, at<void>(d->workspace, L.l.off_Opart), BF, 2, d_op, st_v, b_t, SW))
      return GDN2_ERR_CUDA;
  }
  a.map = seq_map(d, L, cu);
  a.H = d->H;
  a.Qeff = at<bf16>(d->workspace, L.l.off_Qeff);
  a.Opart = at<bf16>(d->workspace, L.l.off_Opart);
  a.Mp = at<bf16>(d->workspace, L.l.off_Mp);
  a.Nc = at<bf16>(d->workspace, L.l.off_Nc);
  a.gamma_last = at<float>(d->workspace, L.l.off_gamma_last);
  a.colscale = at<float>(d->workspace, L.l.off_colscale);
  a.fix_list = at<int32_t>(d->workspace, L.l.off_fix);
  a.status = at<int32_t>(d->workspace, L.l.off_status);
  a.ready = nullptr;
  a.task_counter = nullptr;
  a.l2_prefetch = 1;
  return GDN2_OK;
}

template <int DV>
gdn2_status launch_prep_tc(const gdn2_desc* d, const Layout& L, const void* q, const void* k, const void* v,
                           const float* la, const float* b, const float* w, const int32_t* cu, cudaStream_t s) {
  using C = gdn2::PrepTcCfg<DV>;
  if ((uint64_t)d->B * d->T == 0) return GDN2_OK;
  gdn2::PrepTcArgs a;
  gdn2_status st = fill_prep_tc<DV>(d, L, q, k, v, la, b, w, cu, a);
  if (st != GDN2_OK) return st;
  auto kern = gdn2::prep_tc_kernel<DV>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
    return GDN2_ERR_CUDA;
  // persistent: one CTA per SM (shared memory and TMEM allow no more)
  const long long tasks = (long long)L.l.max_chunks * d->H;
  const int grid = (int)std::min<long long>(tasks, sm_count());
  if (grid <= 0) return GDN2_OK;
  kern<<<grid, C::THREADS, C::SMEM, s>>>(a);
  return launch_status();
}

// ---------------------------------------------------------------- prep ----
template <int DK, int DV, typename IO, typename FT>
gdn2::PrepArgs<IO, FT> prep_args(const gdn2_desc* d, const Layout& L, const void* q, const void* k,
                                 const void* v, const float* la, const float* b, const float* w,
                                 const int32_t* cu) {
  gdn2::PrepArgs<IO, FT> a;
  a.q = static_cast<const IO*>(q);
  a.k = static_cast<const IO*>(k);
  a.v = static_cast<const IO*>(v);
  a.la = la;
  a.b = b;
  a.w = w;
  a.map = seq_map(d, L, cu);
  a.H = d->H;
  a.W = at<FT>(d->workspace, L.l.off_W);
  a.Ut = at<FT>(d->workspace, L.l.off_Ut);
  a.Kbar = at<FT>(d->workspace, L.l.off_Kbar);
  a.Qeff = at<FT>(d->workspace, L.l.off_Qeff);
  a.Opart = at<FT>(d->workspace, L.l.off_Opart);
  a.gamma_last = at<float>(d->workspace, L.l.off_gamma_last);
  a.Mp = at<FT>(d->workspace, L.l.off_Mp);
  a.Nc = at<FT>(d->workspace, L.l.off_Nc);
  a.colscale = L.l.factor_set == 1 ? at<float>(d->workspace, L.l.off_colscale) : nullptr;
  a.Tm = nullptr;
  a.Pm = nullptr;
  return a;
}

// Exact redo of the chunks the tensor-core prep handed back (the kernel
// reads the list's length on the device; an empty list costs one launch).
template <int DK, int DV, typename IO, typename FT>
gdn2_status launch_fixup(const gdn2_desc* d, const Layout& L, const void* q, const void* k, const void* v,
                         const float* la, const float* b, const float* w, const int32_t* cu, cudaStream_t s) {
  const auto a = prep_args<DK, DV, IO, FT>(d, L, q, k, v, la, b, w, cu);
  constexpr size_t smem = gdn2::prep_simt_smem_bytes<DK, DV>();
  auto fix = gdn2::prep_fixup_kernel<DK, DV, IO, FT>;
  if (cudaFuncSetAttribute(fix, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return GDN2_ERR_CUDA;
  const int grid = std::min(L.l.max_chunks * d->H, sm_count());
  fix<<<grid, gdn2::kPrepSimtThreads, smem, s>>>(a, at<const int32_t>(d->workspace, L.l.off_fix));
  return launch_status();
}

template <int DK, int DV, typename IO, typename FT>
gdn2_status launch_prep_t(const gdn2_desc* d, const Layout& L, const void* q, const void* k,
                          const void* v, const float* la, const float* b, const float* w,
                          const int32_t* cu, cudaStream_t s) {
  const auto a = prep_args<DK, DV, IO, FT>(d, L, q, k, v, la, b, w, cu);
  if (L.l.max_chunks == 0) return GDN2_OK;
  constexpr size_t smem = gdn2::prep_simt_smem_bytes<DK, DV>();
  if constexpr (DK == 128 && std::is_same<IO, bf16>::value) {
    if (L.l.factor_set == 1) {
      const gdn2_status st = launch_prep_tc<DV>(d, L, q, k, v, la, b, w, cu, s);
      if (st != GDN2_OK) return st;
      return launch_fixup<DK, DV, IO, FT>(d, L, q, k, v, la, b, w, cu, s);
    }
  }
  auto kern = L.l.factor_set == 1 ? gdn2::prep_simt_kernel<DK, DV, IO, FT, true>
                                  : gdn2::prep_simt_kernel<DK, DV, IO, FT, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return GDN2_ERR_CUDA;
  dim3 grid(L.l.max_chunks, d->H);
  kern<<<grid, gdn2::kPrepSimtThreads, smem, s>>>(a);
  return launch_status();
}

// ------------------------------------------------------- walk (tensor) ----
// bf16 I/O with dk = 128: the affine walk on the tensor cores.
template <int DV>
gdn2_status fill_walk_tc(const gdn2_desc* d, const Layout& L, float scale, const float* h0, const int32_t* cu,
                         void* out, float* hT, float* chunk_states, gdn2::WalkTcArgs& a) {
  using C = gdn2::WalkTcCfg<DV>;
  std::memset(&a, 0, sizeof(a));
  const long long rows_mp = (long long)std::max(L.l.max_chunks, 1) * d->H * 128;
  if (rows_mp >= (1ll << 31)) return GDN2_ERR_SHAPE;  // TMA coordinates are int32
  const uint64_t rows_k = (uint64_t)rows_mp, rows_t = rows_k / 2, rows_g = rows_k / 128;
  const CUtensorMapDataType BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint64_t d_mp[2] = {128, rows_k}, d_qe[2] = {128, rows_t};
  const uint64_t d_nc[2] = {(uint64_t)DV, rows_k}, d_op[2] = {(uint64_t)DV, rows_t}, d_g[2] = {128, rows_g};
  const uint64_t st_k[1] = {256}, st_v[1] = {(uint64_t)DV * 2}, st_g[1] = {512};
  const uint32_t b_mp[2] = {64, 128}, b_qe[2] = {64, 64}, b_nc[2] = {(uint32_t)C::NSL, 128},
                 b_op[2] = {(uint32_t)C::NSL, 64}, b_g[2] = {128, 1};
  const CUtensorMapSwizzle SW = CU_TENSOR_MAP_SWIZZLE_128B;
  if (!gdn2::make_tmap(&a.tm_Mp, at<void>(d->workspace, L.l.off_Mp), BF, 2, d_mp, st_k, b_mp, SW) ||
      !gdn2::make_tmap(&a.tm_Qe, at<void>(d->workspace, L.l.off_Qeff), BF, 2, d_qe, st_k, b_qe, SW) ||
      !gdn2::make_tmap(&a.tm_Nc, at<void>(d->workspace, L.l.off_Nc), BF, 2, d_nc, st_v, b_nc, SW) ||
      !gdn2::make_tmap(&a.tm_Op, at<void>(d->workspace, L.l.off_Opart), BF, 2, d_op, st_v, b_op, SW) ||
      !gdn2::make_tmap(&a.tm_g, at<void>(d->workspace, L.l.off_gamma_last), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, d_g, st_g,
                       b_g, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !gdn2::make_tmap(&a.tm_cs, at<void>(d->workspace, L.l.off_colscale), CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, d_g,
                       st_g, b_g, CU_TENSOR_MAP_SWIZZLE_NONE))
    return GDN2_ERR_CUDA;
  a.map = seq_map(d, L, cu);
  a.H = d->H;
  a.scale = scale;
  a.h0 = h0;
  a.out = static_cast<bf16*>(out);
  a.hT = hT;
  a.chunk_states = chunk_states;
  a.status = at<int32_t>(d->workspace, L.l.off_status);
  return GDN2_OK;
}

template <int DV>
gdn2_status launch_walk_tc(const gdn2_desc* d, const Layout& L, float scale, const float* h0,
                           const int32_t* cu, void* out, float* hT, float* chunk_states, cudaStream_t s,
                           const int* gate = nullptr, bool flagged = false, unsigned long long wait_ns = 0) {
  using C = gdn2::WalkTcCfg<DV>;
  if (L.N == 0) return GDN2_OK;
  gdn2::WalkTcArgs a;
  gdn2_status st = fill_walk_tc<DV>(d, L, scale, h0, cu, out, hT, chunk_states, a);
  if (st != GDN2_OK) return st;
  a.gate = gate;
  if (flagged) {
    int* sync = at<int>(d->workspace, L.l.off_sync);
    a.ready = sync + 2;
    a.redo = sync + 1;
  }
  a.wait_ns = wait_ns;
  auto kern = gdn2::walk_tc_kernel<DV>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
    return GDN2_ERR_CUDA;
  const long long blocks = (long long)L.N * d->H * C::SLICES;
  if (blocks > INT32_MAX) return GDN2_ERR_SHAPE;
  kern<<<(unsigned)blocks, C::THREADS, C::SMEM, s>>>(a);
  return launch_status();
}

// The walk over other ranges than the call's sequences (the segments of the
// two-level scan), in map mode (MAP: [Phi | Psi] from [I | 0]) or with
// outputs from per-range start states.
template <int DV, bool MAP>
gdn2_status launch_walk_ranges(const gdn2_desc* d, const Layout& L, float scale, const gdn2::SeqMap& ranges,
                               const float* h0, void* out, float* phi, float* psi, cudaStream_t s) {
  using C = gdn2::WalkTcCfg<DV>;
  if (ranges.N == 0) return GDN2_OK;
  gdn2::WalkTcArgs a;
  gdn2_status st = fill_walk_tc<DV>(d, L, scale, h0, nullptr, out, nullptr, nullptr, a);
  if (st != GDN2_OK) return st;
  a.map = ranges;
  a.phi = phi;
  a.psi = psi;
  auto kern = gdn2::walk_tc_kernel<DV, MAP>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess)
    return GDN2_ERR_CUDA;
  const long long slices = MAP ? (128 + DV) / C::NSL : C::SLICES;
  const long long blocks = (long long)ranges.N * d->H * slices;
  if (blocks > INT32_MAX) return GDN2_ERR_SHAPE;
  kern<<<(unsigned)blocks, C::THREADS, C::SMEM, s>>>(a);
  return launch_status();
}

// ---------------------------------------------------------------- walk ----
template <int DK, int DV, typename IO, typename FT>
gdn2_status launch_walk_t(const gdn2_desc* d, const Layout& L, float scale, const float* h0,
                          const int32_t* cu, void* out, float* hT, float* chunk_states,
                          cudaStream_t s) {
  gdn2::WalkArgs<IO, FT> a;
  a.W = at<const FT>(d->workspace, L.l.off_W);
  a.Ut = at<const FT>(d->workspace, L.l.off_Ut);
  a.Kbar = at<const FT>(d->workspace, L.l.off_Kbar);
  a.Qeff = at<const FT>(d->workspace, L.l.off_Qeff);
  a.Opart = at<const FT>(d->workspace, L.l.off_Opart);
  a.gamma_last = at<const float>(d->workspace, L.l.off_gamma_last);
  a.map = seq_map(d, L, cu);
  a.H = d->H;
  a.scale = scale;
  a.h0 = h0;
  a.out = static_cast<IO*>(out);
  a.hT = hT;
  a.chunk_states = chunk_states;
  a.U_out = nullptr;
  if constexpr (DK == 128 && std::is_same<IO, bf16>::value) {
    if (L.l.factor_set == 1) return launch_walk_tc<DV>(d, L, scale, h0, cu, out, hT, chunk_states, s);
  }
  if (L.N == 0) return GDN2_OK;
  constexpr size_t smem = gdn2::walk_simt_smem_bytes<DK, gdn2::kWalkSimtDVS>();
  auto kern = gdn2::walk_simt_kernel<DK, DV, IO, FT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return GDN2_ERR_CUDA;
  const long long blocks = (long long)L.N * d->H * (DV / gdn2::kWalkSimtDVS);
  if (blocks > INT32_MAX) return GDN2_ERR_SHAPE;
  kern<<<(unsigned)blocks, gdn2::walk_simt_threads(gdn2::kWalkSimtDVS), smem, s>>>(a);
  return launch_status();
}

// ------------------------------------------------------------- fused ----
// Prep and walk in one launch when the walk needs few CTAs (long sequences,
// few heads); then the fixup of handed-back chunks and, only if one of them
// cut the walk short, the walk again.
template <int DV>
bool fused_fits(const gdn2_desc* d, const Layout& L) {
  const long long n_walk = (long long)L.N * d->H * gdn2::WalkTcCfg<DV>::SLICES;
  return L.l.factor_set == 1 && L.N > 0 && (long long)d->B * d->T > 0 &&
         n_walk + gdn2::FusedTcCfg<DV>::MIN_PREP_CTAS <= sm_count();
}

template <int DV>
gdn2_status launch_fused_tc(const gdn2_desc* d, const Layout& L, const void* q, const void* k, const void* v,
                            const float* la, const float* b, const float* w, const int32_t* cu, float scale,
                            const float* h0, void* out, float* hT, cudaStream_t s) {
  using F = gdn2::FusedTcCfg<DV>;
  gdn2::PrepTcArgs pa;
  gdn2::WalkTcArgs wa;
  gdn2_status st = fill_prep_tc<DV>(d, L, q, k, v, la, b, w, cu, pa);
  if (st != GDN2_OK) return st;
  if ((st = fill_walk_tc<DV>(d, L, scale, h0, cu, out, hT, nullptr, wa)) != GDN2_OK) return st;
  int* sync = at<int>(d->workspace, L.l.off_sync);
  pa.task_counter = sync;
  pa.ready = sync + 2;
  pa.l2_prefetch = 0;
  wa.ready = sync + 2;
  wa.redo = sync + 1;
  const int n_sm = sm_count();
  const int n_walk = L.N * d->H * gdn2::WalkTcCfg<DV>::SLICES;
  // When the walk CTAs stop taking prep tasks: a walk of nch chunks started
  // when nch * (n_sm - n_walk) / 7 tasks are left ends about with the prep
  // (beside the prep, a walk step costs about a seventh of a prep task on
  // one SM).  With the prep's stores off its critical path this leaves the
  // walk CTAs no prep work on the workloads measured (a sweep of the switch
  // point at 16K x 1 has its optimum at 0), and then they skip the prep role.
  {
    const long long tasks = (long long)L.l.max_chunks * d->H;
    const long long nch = ((long long)d->B * d->T + (long long)kChunk * L.N - 1) / ((long long)kChunk * L.N);
    const long long left = nch * (n_sm - n_walk) / 7;
    pa.stop_at = (int)std::max(0ll, tasks - left);
  }
  auto kern = gdn2::fused_tc_kernel<DV>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, F::SMEM) != cudaSuccess)
    return GDN2_ERR_CUDA;
  // The walk CTAs wait on flags the prep CTAs raise, so every CTA must be
  // resident at once: a cooperative launch guarantees it or fails (fewer SMs
  // available than the device reports, e.g. under MPS or in a green context),
  // and then the caller runs the two stage kernels instead.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(n_sm);
  cfg.blockDim = dim3(F::THREADS);
  cfg.dynamicSmemBytes = F::SMEM;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, pa, wa, n_sm - n_walk);
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();
    return GDN2_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? launch_status() : GDN2_ERR_CUDA;
}

template <int DV>
gdn2_status launch_fused_full(const gdn2_desc* d, const Layout& L, const void* q, const void* k, const void* v,
                              const float* la, const float* b, const float* w, const int32_t* cu, float scale,
                              const float* h0, void* out, float* hT, cudaStream_t s) {
  gdn2_status st = launch_fused_tc<DV>(d, L, q, k, v, la, b, w, cu, scale, h0, out, hT, s);
  if (st == GDN2_ERR_UNSUPPORTED) {
    // not all CTAs could be resident at once: the two stage kernels
    if ((st = launch_prep_t<128, DV, bf16, bf16>(d, L, q, k, v, la, b, w, cu, s)) != GDN2_OK) return st;
    return launch_walk_tc<DV>(d, L, scale, h0, cu, out, hT, nullptr, s);
  }
  if (st != GDN2_OK) return st;
  if ((st = launch_fixup<128, DV, bf16, bf16>(d, L, q, k, v, la, b, w, cu, s)) != GDN2_OK) return st;
  return launch_walk_tc<DV>(d, L, scale, h0, cu, out, hT, nullptr, s, at<int>(d->workspace, L.l.off_sync) + 1);
}

// ----------------------------------------------------------- dispatch ----
template <template <int, int, typename, typename> class F, typename... Args>
gdn2_status dispatch(const gdn2_desc* d, Args... args) {
  const bool f32 = d->io == GDN2_IO_F32;
#define GDN2_CASE(DK_, DV_)                                                        \
  if (d->dk == DK_ && d->dv == DV_)                                                \
    return f32 ? F<DK_, DV_, float, float>::run(d, args...)                        \
               : F<DK_, DV_, bf16, bf16>::run(d, args...);
  GDN2_CASE(64, 64)
  GDN2_CASE(64, 128)
  GDN2_CASE(128, 64)
  GDN2_CASE(128, 128)
#undef GDN2_CASE
  return GDN2_ERR_SHAPE;
}

template <int DK, int DV, typename IO, typename FT>
struct PrepOp {
  template <typename... A>
  static gdn2_status run(const gdn2_desc* d, A... a) { return launch_prep_t<DK, DV, IO, FT>(d, a...); }
};
template <int DK, int DV, typename IO, typename FT>
struct WalkOp {
  template <typename... A>
  static gdn2_status run(const gdn2_desc* d, A... a) { return launch_walk_t<DK, DV, IO, FT>(d, a...); }
};

template <int DK, int DV, typename IO, typename FT>
struct DecodeOp {
  static gdn2_status run(const gdn2_desc* d, const void* q, const void* k, const void* v,
                         const float* la, const float* b, const float* w, float scale,
                         float* state, void* out, cudaStream_t s) {
    gdn2::DecodeArgs<IO> a;
    a.q = static_cast<const IO*>(q);
    a.k = static_cast<const IO*>(k);
    a.v = static_cast<const IO*>(v);
    a.la = la;
    a.b = b;
    a.w = w;
    a.state = state;
    a.out = static_cast<IO*>(out);
    a.H = d->H;
    a.scale = scale;
    constexpr int cols = DV < 32 ? DV : 32;
    const long long blocks = (long long)d->B * d->H * (DV / cols);
    if (blocks == 0) return GDN2_OK;
    if (blocks > INT32_MAX) return GDN2_ERR_SHAPE;
    gdn2::decode_kernel<DK, DV, IO><<<(unsigned)blocks, gdn2::kDecodeThreads, 0, s>>>(a);
    return launch_status();
  }
};

// ------------------------------------------------------------- backward ----
// Workspace of gdn2_chunk_bwd: the status word; the forward's fp32 WY factor
// set (the layout gdn2_chunk_fwd uses for fp32 I/O, whatever the I/O type of
// the call), with its chunk map; T and P of every (chunk, head); the state at
// every chunk start (S0); the gradient reaching every chunk's end (dS1); from
// the two walks, U = U~ - W S0 and Kbar dS1 of every chunk; and the outputs'
// share of the state gradient, G = scale Q_eff^T dO, of every chunk.
struct BwdLayout {
  Layout f;            // the factor set, relative to the workspace + kAlign
  size_t off_T, off_P, off_S0, off_dS1, off_U, off_X, off_G, total;   // from the workspace start
};

gdn2_desc bwd_factor_desc(const gdn2_desc* d) {
  gdn2_desc f = *d;
  f.io = GDN2_IO_F32;
  f.workspace = d->workspace ? static_cast<char*>(d->workspace) + kAlign : nullptr;
  f.workspace_bytes = d->workspace_bytes > kAlign ? d->workspace_bytes - kAlign : 0;
  return f;
}

gdn2_status bwd_layout(const gdn2_desc* d, bool packed, BwdLayout* B) {
  const gdn2_desc f = bwd_factor_desc(d);
  gdn2_status st = make_layout(&f, packed, &B->f);
  if (st != GDN2_OK) return st;
  const size_t chunks_h = (size_t)B->f.l.max_chunks * d->H;
  size_t off = kAlign + B->f.l.total_bytes;
  B->off_T = off;   off = align_up(off + chunks_h * kChunk * kChunk * sizeof(float));
  B->off_P = off;   off = align_up(off + chunks_h * kChunk * kChunk * sizeof(float));
  B->off_S0 = off;  off = align_up(off + chunks_h * d->dk * d->dv * sizeof(float));
  B->off_dS1 = off; off = align_up(off + chunks_h * d->dk * d->dv * sizeof(float));
  B->off_U = off;   off = align_up(off + chunks_h * kChunk * d->dv * sizeof(float));
  B->off_X = off;   off = align_up(off + chunks_h * kChunk * d->dv * sizeof(float));
  B->off_G = off;   off = align_up(off + chunks_h * d->dk * d->dv * sizeof(float));
  B->total = off;
  return GDN2_OK;
}

template <int DK, int DV, typename IO, typename FT>
struct BwdOp {
  static gdn2_status run(const gdn2_desc* d, const BwdLayout& B, const void* q, const void* k, const void* v,
                         const float* la, const float* b, const float* w, float scale, const float* h0,
                         const int32_t* cu, const void* dO, const float* dhT, float* dq, float* dk, float* dv,
                         float* dla, float* db, float* dw, float* dh0, cudaStream_t s) {
    const gdn2_desc f = bwd_factor_desc(d);
    const Layout& L = B.f;
    int32_t* status = at<int32_t>(d->workspace, 0);
    // chunk map (and the check of cu_seqlens, into the status word)
    gdn2::plan_kernel<<<1, gdn2::kPlanThreads, 0, s>>>(cu, L.N, d->T, d->B * d->T,
                                                        at<int32_t>(f.workspace, L.l.off_chunk_offsets), status,
                                                        (int)GDN2_ERR_SEQLENS, nullptr, nullptr, 0);
    gdn2_status st = launch_status();
    if (st != GDN2_OK) return st;
    const gdn2::SeqMap map = seq_map(&f, L, cu);
    // 1. factors, T and P in fp32
    if (L.l.max_chunks > 0) {
      auto pa = prep_args<DK, DV, IO, float>(&f, L, q, k, v, la, b, w, cu);
      pa.Tm = at<float>(d->workspace, B.off_T);
      pa.Pm = at<float>(d->workspace, B.off_P);
      constexpr size_t smem = gdn2::prep_simt_smem_bytes<DK, DV>();
      auto kern = gdn2::prep_simt_kernel<DK, DV, IO, float, false>;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return GDN2_ERR_CUDA;
      kern<<<dim3(L.l.max_chunks, d->H), gdn2::kPrepSimtThreads, smem, s>>>(pa);
      if ((st = launch_status()) != GDN2_OK) return st;
    }
    if (L.N == 0) return GDN2_OK;
    // G = scale Q_eff^T dO of every chunk, for the reverse walk
    if (L.l.max_chunks > 0) {
      constexpr size_t smem = gdn2::bwd_g_smem_bytes<DK, DV, IO>();
      auto kern = gdn2::bwd_g_kernel<DK, DV, IO>;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return GDN2_ERR_CUDA;
      kern<<<dim3(L.l.max_chunks, d->H), gdn2::kBwdGThreads, smem, s>>>(
          at<const float>(f.workspace, L.l.off_Qeff), dO, map, d->H, scale, at<float>(d->workspace, B.off_G));
      if ((st = launch_status()) != GDN2_OK) return st;
    }
    // 2. the state at every chunk start and 3. the gradient reaching every
    // chunk's end state (and dh0), in one launch
    {
      gdn2::WalkArgs<IO, float> wa;
      wa.W = at<const float>(f.workspace, L.l.off_W);
      wa.Ut = at<const float>(f.workspace, L.l.off_Ut);
      wa.Kbar = at<const float>(f.workspace, L.l.off_Kbar);
      wa.Qeff = at<const float>(f.workspace, L.l.off_Qeff);
      wa.Opart = at<const float>(f.workspace, L.l.off_Opart);
      wa.gamma_last = at<const float>(f.workspace, L.l.off_gamma_last);
      wa.map = map;
      wa.H = d->H;
      wa.scale = scale;
      wa.h0 = h0;
      wa.out = nullptr;
      wa.hT = nullptr;
      wa.chunk_states = at<float>(d->workspace, B.off_S0);
      wa.U_out = at<float>(d->workspace, B.off_U);
      gdn2::BwdStateArgs ra;
      ra.W = wa.W;
      ra.Kbar = wa.Kbar;
      ra.gamma_last = wa.gamma_last;
      ra.G = at<const float>(d->workspace, B.off_G);
      ra.map = map;
      ra.H = d->H;
      ra.dhT = dhT;
      ra.dS1 = at<float>(d->workspace, B.off_dS1);
      ra.X = at<float>(d->workspace, B.off_X);
      ra.dh0 = dh0;
      ra.status = status;
      constexpr size_t smem =
          std::max(gdn2::walk_simt_smem_bytes<DK, gdn2::kBwdWalkCols>(), gdn2::bwd_dstate_smem_bytes<DK>());
      auto kern = gdn2::bwd_walks_kernel<DK, DV, IO>;
      if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return GDN2_ERR_CUDA;
      const long long n_fwd = (long long)L.N * d->H * (DV / gdn2::kBwdWalkCols);
      const long long n_rev = (long long)L.N * d->H * (DV / gdn2::kBwdWalkCols);
      if (n_fwd + n_rev > INT32_MAX) return GDN2_ERR_SHAPE;
      kern<<<(unsigned)(n_fwd + n_rev), gdn2::kBwdWalkThreads, smem, s>>>(wa, ra, (int)n_fwd);
      if ((st = launch_status()) != GDN2_OK) return st;
    }
    // 4. every (chunk, head): the gradients of its tokens
    if (L.l.max_chunks == 0) return GDN2_OK;
    gdn2::BwdChunkArgs ca;
    ca.q = q; ca.k = k; ca.v = v; ca.dO = dO;
    ca.la = la; ca.b = b; ca.w = w;
    ca.Tm = at<const float>(d->workspace, B.off_T);
    ca.Pm = at<const float>(d->workspace, B.off_P);
    ca.S0 = at<const float>(d->workspace, B.off_S0);
    ca.dS1 = at<const float>(d->workspace, B.off_dS1);
    ca.U = at<const float>(d->workspace, B.off_U);
    ca.X = at<const float>(d->workspace, B.off_X);
    ca.map = map;
    ca.H = d->H;
    ca.scale = scale;
    ca.dq = dq; ca.dk = dk; ca.dla = dla; ca.db = db; ca.dv = dv; ca.dw = dw;
    constexpr size_t smem = gdn2::BwdCfg<DK, DV, IO>::SMEM;
    auto kern = gdn2::bwd_chunk_kernel<DK, DV, IO>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return GDN2_ERR_CUDA;
    kern<<<dim3(L.l.max_chunks, d->H), gdn2::kBwdThreads, smem, s>>>(ca);
    return launch_status();
  }
};

// ------------------------------------------------- two-level chunk scan ----
// Extra workspace of gdn2_chunk_fwd_segmented, after the usual layout: the
// virtual segments, their maps (Phi, Psi, fp32) and start states (fp32).
struct SegLayout {
  int L = 0, ns_max = 0;
  size_t off_seg_cu = 0, off_seg_chunk = 0, off_seq_seg = 0, off_phi = 0, off_psi = 0, off_seg_h0 = 0, total = 0;
};

gdn2_status seg_layout(const gdn2_desc* d, const Layout& L, int segment_chunks, SegLayout* g) {
  if (segment_chunks < 0) return GDN2_ERR_SHAPE;
  const long long tokens = (long long)d->B * d->T;
  // chunks per sequence (on average, for a packed row)
  const long long nch = L.N > 0 ? (tokens / L.N + kChunk - 1) / kChunk : 0;
  const long long Lc = segment_chunks > 0 ? segment_chunks : std::max(8ll, (nch + 3) / 4);
  const bool packed = d->num_seqs > 0;
  const long long ns = packed ? L.l.max_chunks / Lc + L.N
                              : (long long)d->B * ((((long long)d->T + kChunk - 1) / kChunk + Lc - 1) / Lc);
  if (ns > INT32_MAX / 4 || Lc > INT32_MAX / 4) return GDN2_ERR_SHAPE;
  g->L = (int)Lc;
  g->ns_max = (int)ns;
  size_t off = align_up(L.l.total_bytes);
  g->off_seg_cu = off;    off = align_up(off + (size_t)(ns + 1) * sizeof(int32_t));
  g->off_seg_chunk = off; off = align_up(off + (size_t)(ns + 1) * sizeof(int32_t));
  g->off_seq_seg = off;   off = align_up(off + (size_t)(L.N + 1) * sizeof(int32_t));
  g->off_phi = off;       off = align_up(off + (size_t)ns * d->H * d->dk * d->dk * sizeof(float));
  g->off_psi = off;       off = align_up(off + (size_t)ns * d->H * d->dk * d->dv * sizeof(float));
  g->off_seg_h0 = off;    off = align_up(off + (size_t)ns * d->H * d->dk * d->dv * sizeof(float));
  g->total = off;
  return GDN2_OK;
}

template <int DV>
gdn2_status launch_segmented(const gdn2_desc* d, const Layout& L, const SegLayout& g, const void* q, const void* k,
                             const void* v, const float* la, const float* b, const float* w, const int32_t* cu,
                             float scale, const float* h0, void* out, float* hT, cudaStream_t s) {
  gdn2_status st;
  if ((st = launch_prep_t<128, DV, bf16, bf16>(d, L, q, k, v, la, b, w, cu, s)) != GDN2_OK) return st;
  int32_t* seg_cu = at<int32_t>(d->workspace, g.off_seg_cu);
  int32_t* seg_chunk = at<int32_t>(d->workspace, g.off_seg_chunk);
  int32_t* seq_seg = at<int32_t>(d->workspace, g.off_seq_seg);
  float* phi = at<float>(d->workspace, g.off_phi);
  float* psi = at<float>(d->workspace, g.off_psi);
  float* seg_h0 = at<float>(d->workspace, g.off_seg_h0);
  gdn2::segplan_kernel<<<1, gdn2::kSegPlanThreads, 0, s>>>(cu, L.N, d->T, d->B * d->T,
                                                           at<const int32_t>(d->workspace, L.l.off_chunk_offsets),
                                                           g.L, g.ns_max, seg_cu, seg_chunk, seq_seg);
  if ((st = launch_status()) != GDN2_OK) return st;
  gdn2::SeqMap segs;
  segs.cu = seg_cu;
  segs.chunk_off = seg_chunk;
  segs.N = g.ns_max;
  segs.T = d->T;
  // 1. every segment's affine map
  if ((st = launch_walk_ranges<DV, true>(d, L, scale, segs, nullptr, nullptr, phi, psi, s)) != GDN2_OK) return st;
  // 2. the scan of the maps: start states of the segments, final states
  const long long blocks = (long long)L.N * d->H * (DV / gdn2::kScanCols);
  if (blocks > INT32_MAX) return GDN2_ERR_SHAPE;
  if (blocks > 0) {
    gdn2::segscan_kernel<128, DV><<<(unsigned)blocks, gdn2::kScanThreads, 0, s>>>(phi, psi, seq_seg, d->H, h0,
                                                                                  seg_h0, hT);
    if ((st = launch_status()) != GDN2_OK) return st;
  }
  // 3. the segments again, with outputs, from their start states
  return launch_walk_ranges<DV, false>(d, L, scale, segs, seg_h0, out, nullptr, nullptr, s);
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 1;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return 1;
  return n;
}

bool device_ok() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  int major = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10;
}

// Token arrays may be NULL only when there are no tokens (an empty tensor has
// no storage); non-NULL pointers must always be 16-byte aligned.
gdn2_status check_inputs(const void* q, const void* k, const void* v, const float* la,
                         const float* b, const float* w, long long tokens = 1) {
  if (tokens > 0 && (!q || !k || !v || !la || !b || !w)) return GDN2_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(la) || !aligned16(b) ||
      !aligned16(w))
    return GDN2_ERR_ALIGN;
  return GDN2_OK;
}

}  // namespace

// one prologue launch with the width d and the tap count W as template
// arguments (d in {64, 128}, 1 <= W <= 8, both checked by the caller)
template <typename IO, int D>
static void launch_prologue_d(int W, const gdn2::TokProArgs& a, dim3 grid, cudaStream_t stream) {
  switch (W) {
#define GDN2_PRO_W(W_) \
  case W_: gdn2::token_prologue_kernel<IO, D, W_><<<grid, gdn2::kTokThreads, 0, stream>>>(a); break;
    GDN2_PRO_W(1) GDN2_PRO_W(2) GDN2_PRO_W(3) GDN2_PRO_W(4)
    GDN2_PRO_W(5) GDN2_PRO_W(6) GDN2_PRO_W(7) GDN2_PRO_W(8)
#undef GDN2_PRO_W
    default: break;
  }
}

template <typename IO>
static void launch_prologue(int d, int W, const gdn2::TokProArgs& a, dim3 grid, cudaStream_t stream) {
  if (d == 64) launch_prologue_d<IO, 64>(W, a, grid, stream);
  else launch_prologue_d<IO, 128>(W, a, grid, stream);
}

extern "C" {

size_t gdn2_workspace_size(const gdn2_desc* desc) {
  if (!desc) return 0;
  Layout L;
  const bool packed = desc->num_seqs > 0;
  if (make_layout(desc, packed, &L) != GDN2_OK) return 0;
  return L.l.total_bytes;
}

gdn2_status gdn2_workspace_layout(const gdn2_desc* desc, gdn2_ws_layout* layout) {
  if (!desc || !layout) return GDN2_ERR_NULL;
  Layout L;
  const bool packed = desc->num_seqs > 0;
  const gdn2_status st = make_layout(desc, packed, &L);
  if (st != GDN2_OK) return st;
  *layout = L.l;
  return GDN2_OK;
}

gdn2_status gdn2_chunk_prep(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                            const float* log_alpha, const float* b, const float* w,
                            const int32_t* cu_seqlens, cudaStream_t stream) {
  Layout L;
  gdn2_status st = make_layout(desc, cu_seqlens != nullptr, &L);
  if (st != GDN2_OK) return st;
  if ((st = check_workspace(desc, L)) != GDN2_OK) return st;
  if ((st = check_inputs(q, k, v, log_alpha, b, w, (long long)desc->B * desc->T)) != GDN2_OK) return st;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  if ((st = launch_plan(desc, L, cu_seqlens, stream)) != GDN2_OK) return st;
  return dispatch<PrepOp>(desc, L, q, k, v, log_alpha, b, w, cu_seqlens, stream);
}

gdn2_status gdn2_chunk_walk(const gdn2_desc* desc, float scale, const float* h0,
                            const int32_t* cu_seqlens, void* out, float* hT, float* chunk_states,
                            cudaStream_t stream) {
  Layout L;
  gdn2_status st = make_layout(desc, cu_seqlens != nullptr, &L);
  if (st != GDN2_OK) return st;
  if ((st = check_workspace(desc, L)) != GDN2_OK) return st;
  if (!out && (long long)desc->B * desc->T > 0) return GDN2_ERR_NULL;
  if (!aligned16(out) || (h0 && !aligned16(h0)) || (hT && !aligned16(hT)) ||
      (chunk_states && !aligned16(chunk_states)))
    return GDN2_ERR_ALIGN;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  return dispatch<WalkOp>(desc, L, scale, h0, cu_seqlens, out, hT, chunk_states, stream);
}

gdn2_status gdn2_chunk_fwd(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                           const float* log_alpha, const float* b, const float* w, float scale,
                           const float* h0, const int32_t* cu_seqlens, void* out, float* hT,
                           cudaStream_t stream) {
  Layout L;
  gdn2_status st = make_layout(desc, cu_seqlens != nullptr, &L);
  if (st != GDN2_OK) return st;
  if ((st = check_workspace(desc, L)) != GDN2_OK) return st;
  const long long tokens = (long long)desc->B * desc->T;
  if ((st = check_inputs(q, k, v, log_alpha, b, w, tokens)) != GDN2_OK) return st;
  if (!out && tokens > 0) return GDN2_ERR_NULL;
  if (!aligned16(out) || (h0 && !aligned16(h0)) || (hT && !aligned16(hT))) return GDN2_ERR_ALIGN;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  if ((st = launch_plan(desc, L, cu_seqlens, stream)) != GDN2_OK) return st;
  if (desc->io == GDN2_IO_BF16 && desc->dk == 128) {
    if (desc->dv == 128 && fused_fits<128>(desc, L))
      return launch_fused_full<128>(desc, L, q, k, v, log_alpha, b, w, cu_seqlens, scale, h0, out, hT, stream);
    if (desc->dv == 64 && fused_fits<64>(desc, L))
      return launch_fused_full<64>(desc, L, q, k, v, log_alpha, b, w, cu_seqlens, scale, h0, out, hT, stream);
  }
  if ((st = dispatch<PrepOp>(desc, L, q, k, v, log_alpha, b, w, cu_seqlens, stream)) != GDN2_OK)
    return st;
  return dispatch<WalkOp>(desc, L, scale, h0, cu_seqlens, out, hT, (float*)nullptr, stream);
}

gdn2_status gdn2_chunk_plan(const gdn2_desc* desc, const int32_t* cu_seqlens, cudaStream_t stream) {
  Layout L;
  gdn2_status st = make_layout(desc, cu_seqlens != nullptr, &L);
  if (st != GDN2_OK) return st;
  if ((st = check_workspace(desc, L)) != GDN2_OK) return st;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  return launch_plan(desc, L, cu_seqlens, stream);
}

gdn2_status gdn2_chunk_fused(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                             const float* log_alpha, const float* b, const float* w, float scale,
                             const float* h0, const int32_t* cu_seqlens, void* out, float* hT,
                             cudaStream_t stream) {
  Layout L;
  gdn2_status st = make_layout(desc, cu_seqlens != nullptr, &L);
  if (st != GDN2_OK) return st;
  if ((st = check_workspace(desc, L)) != GDN2_OK) return st;
  const long long tokens = (long long)desc->B * desc->T;
  if ((st = check_inputs(q, k, v, log_alpha, b, w, tokens)) != GDN2_OK) return st;
  if (!out && tokens > 0) return GDN2_ERR_NULL;
  if (!aligned16(out) || (h0 && !aligned16(h0)) || (hT && !aligned16(hT))) return GDN2_ERR_ALIGN;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  if (desc->io == GDN2_IO_BF16 && desc->dk == 128) {
    if (desc->dv == 128 && fused_fits<128>(desc, L))
      return launch_fused_tc<128>(desc, L, q, k, v, log_alpha, b, w, cu_seqlens, scale, h0, out, hT, stream);
    if (desc->dv == 64 && fused_fits<64>(desc, L))
      return launch_fused_tc<64>(desc, L, q, k, v, log_alpha, b, w, cu_seqlens, scale, h0, out, hT, stream);
  }
  return GDN2_ERR_UNSUPPORTED;
}

size_t gdn2_segmented_workspace_size(const gdn2_desc* desc, int segment_chunks) {
  if (!desc) return 0;
  Layout L;
  if (make_layout(desc, desc->num_seqs > 0, &L) != GDN2_OK || L.l.factor_set != 1) return 0;
  SegLayout g;
  if (seg_layout(desc, L, segment_chunks, &g) != GDN2_OK) return 0;
  return g.total;
}

gdn2_status gdn2_chunk_fwd_segmented(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                                     const float* log_alpha, const float* b, const float* w, float scale,
                                     const float* h0, const int32_t* cu_seqlens, void* out, float* hT,
                                     int segment_chunks, cudaStream_t stream) {
  Layout L;
  gdn2_status st = make_layout(desc, cu_seqlens != nullptr, &L);
  if (st != GDN2_OK) return st;
  if (L.l.factor_set != 1) return GDN2_ERR_UNSUPPORTED;
  SegLayout g;
  if ((st = seg_layout(desc, L, segment_chunks, &g)) != GDN2_OK) return st;
  if (!desc->workspace) return GDN2_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(desc->workspace) & (kAlign - 1)) != 0) return GDN2_ERR_ALIGN;
  if (desc->workspace_bytes < g.total) return GDN2_ERR_WORKSPACE;
  const long long tokens = (long long)desc->B * desc->T;
  if ((st = check_inputs(q, k, v, log_alpha, b, w, tokens)) != GDN2_OK) return st;
  if (!out && tokens > 0) return GDN2_ERR_NULL;
  if (!aligned16(out) || (h0 && !aligned16(h0)) || (hT && !aligned16(hT))) return GDN2_ERR_ALIGN;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  if ((st = launch_plan(desc, L, cu_seqlens, stream)) != GDN2_OK) return st;
  if (desc->dv == 128)
    return launch_segmented<128>(desc, L, g, q, k, v, log_alpha, b, w, cu_seqlens, scale, h0, out, hT, stream);
  return launch_segmented<64>(desc, L, g, q, k, v, log_alpha, b, w, cu_seqlens, scale, h0, out, hT, stream);
}

gdn2_status gdn2_state_map(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                           const float* log_alpha, const float* b, const float* w, const int32_t* cu_seqlens,
                           float* phi, float* psi, cudaStream_t stream) {
  Layout L;
  gdn2_status st = make_layout(desc, cu_seqlens != nullptr, &L);
  if (st != GDN2_OK) return st;
  if (L.l.factor_set != 1) return GDN2_ERR_UNSUPPORTED;
  if ((st = check_workspace(desc, L)) != GDN2_OK) return st;
  if ((st = check_inputs(q, k, v, log_alpha, b, w, (long long)desc->B * desc->T)) != GDN2_OK) return st;
  if (!phi || !psi) return GDN2_ERR_NULL;
  if (!aligned16(phi) || !aligned16(psi)) return GDN2_ERR_ALIGN;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  if ((st = launch_plan(desc, L, cu_seqlens, stream)) != GDN2_OK) return st;
  gdn2::SeqMap seqs = seq_map(desc, L, cu_seqlens);
  if (desc->dv == 128) {
    if ((st = launch_prep_t<128, 128, bf16, bf16>(desc, L, q, k, v, log_alpha, b, w, cu_seqlens, stream)) != GDN2_OK)
      return st;
    return launch_walk_ranges<128, true>(desc, L, 1.f, seqs, nullptr, nullptr, phi, psi, stream);
  }
  if ((st = launch_prep_t<128, 64, bf16, bf16>(desc, L, q, k, v, log_alpha, b, w, cu_seqlens, stream)) != GDN2_OK)
    return st;
  return launch_walk_ranges<64, true>(desc, L, 1.f, seqs, nullptr, nullptr, phi, psi, stream);
}

gdn2_status gdn2_chunk_walk_flagged(const gdn2_desc* desc, float scale, const float* h0,
                                    const int32_t* cu_seqlens, void* out, float* hT,
                                    unsigned long long wait_budget_ns, cudaStream_t stream) {
  Layout L;
  gdn2_status st = make_layout(desc, cu_seqlens != nullptr, &L);
  if (st != GDN2_OK) return st;
  if ((st = check_workspace(desc, L)) != GDN2_OK) return st;
  if (!out && (long long)desc->B * desc->T > 0) return GDN2_ERR_NULL;
  if (!aligned16(out) || (h0 && !aligned16(h0)) || (hT && !aligned16(hT))) return GDN2_ERR_ALIGN;
  if (L.l.factor_set != 1) return GDN2_ERR_UNSUPPORTED;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  if (desc->dv == 128)
    return launch_walk_tc<128>(desc, L, scale, h0, cu_seqlens, out, hT, nullptr, stream, nullptr, true,
                               wait_budget_ns);
  return launch_walk_tc<64>(desc, L, scale, h0, cu_seqlens, out, hT, nullptr, stream, nullptr, true,
                            wait_budget_ns);
}

gdn2_status gdn2_token_prologue(const gdn2_desc* desc, const void* q_raw, const void* k_raw, const void* v_raw,
                                const float* conv_q, const float* conv_k, const float* conv_v, int conv_width,
                                const int32_t* cu_seqlens, void* q, void* k, void* v, cudaStream_t stream) {
  if (!desc) return GDN2_ERR_NULL;
  const bool packed = cu_seqlens != nullptr;
  gdn2_status st = check_dims(desc, packed);
  if (st != GDN2_OK) return st;
  if (conv_width < 1 || conv_width > gdn2::kMaxConvWidth) return GDN2_ERR_SHAPE;
  const long long tokens = (long long)desc->B * desc->T;
  if (tokens > 0 && (!q_raw || !k_raw || !v_raw || !conv_q || !conv_k || !conv_v || !q || !k || !v))
    return GDN2_ERR_NULL;
  if (!aligned16(q_raw) || !aligned16(k_raw) || !aligned16(v_raw) || !aligned16(q) || !aligned16(k) ||
      !aligned16(v) || !aligned16(conv_q) || !aligned16(conv_k) || !aligned16(conv_v))
    return GDN2_ERR_ALIGN;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  if (tokens == 0) return GDN2_OK;
  gdn2::TokProArgs a{};
  a.cu = cu_seqlens;
  a.N = packed ? desc->num_seqs : desc->B;
  a.T = desc->T;
  a.T_total = (int)tokens;
  a.H = desc->H;
  const int tile = desc->io == GDN2_IO_F32 ? gdn2::tok_tile<float>() : gdn2::tok_tile<bf16>();
  const long long tiles = (tokens + tile - 1) / tile;
  if (tiles > INT32_MAX || desc->H > 65535) return GDN2_ERR_SHAPE;
  // q and k (and v when dv == dk) in one launch, v in a second one otherwise
  a.x[0] = q_raw; a.wt[0] = conv_q; a.y[0] = q; a.l2[0] = 1;
  a.x[1] = k_raw; a.wt[1] = conv_k; a.y[1] = k; a.l2[1] = 1;
  gdn2::TokProArgs av = a;
  av.x[0] = v_raw; av.wt[0] = conv_v; av.y[0] = v; av.l2[0] = 0;
  const bool one = desc->dk == desc->dv;
  if (one) { a.x[2] = v_raw; a.wt[2] = conv_v; a.y[2] = v; a.l2[2] = 0; }
  const dim3 grid_qk((unsigned)tiles, (unsigned)desc->H, one ? 3 : 2), grid_v((unsigned)tiles, (unsigned)desc->H, 1);
  const bool f32 = desc->io == GDN2_IO_F32;
  if (f32) {
    launch_prologue<float>(desc->dk, conv_width, a, grid_qk, stream);
    if (!one) launch_prologue<float>(desc->dv, conv_width, av, grid_v, stream);
  } else {
    launch_prologue<bf16>(desc->dk, conv_width, a, grid_qk, stream);
    if (!one) launch_prologue<bf16>(desc->dv, conv_width, av, grid_v, stream);
  }
  return launch_status();
}

gdn2_status gdn2_token_epilogue(const gdn2_desc* desc, const void* o, const void* gate, const float* norm_weight,
                                void* out, cudaStream_t stream) {
  if (!desc) return GDN2_ERR_NULL;
  if (desc->io != GDN2_IO_F32 && desc->io != GDN2_IO_BF16) return GDN2_ERR_DTYPE;
  if ((desc->dk != 64 && desc->dk != 128) || (desc->dv != 64 && desc->dv != 128)) return GDN2_ERR_SHAPE;
  if (desc->H < 1 || desc->B < 1 || desc->T < 0) return GDN2_ERR_SHAPE;
  const long long tokens = (long long)desc->B * desc->T;
  if (tokens > INT32_MAX / 2) return GDN2_ERR_SHAPE;
  if (tokens > 0 && (!o || !gate || !norm_weight || !out)) return GDN2_ERR_NULL;
  if (!aligned16(o) || !aligned16(gate) || !aligned16(norm_weight) || !aligned16(out)) return GDN2_ERR_ALIGN;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  if (tokens == 0) return GDN2_OK;
  gdn2::TokEpiArgs a;
  a.o = o; a.g = gate; a.weight = norm_weight;
  a.rows = tokens * desc->H;
  a.out = out;
  const long long per_block = gdn2::kTokThreads / 16 * gdn2::kEpiRows;   // kEpiRows rows per half-warp
  const long long blocks = (a.rows + per_block - 1) / per_block;
  if (blocks > INT32_MAX) return GDN2_ERR_SHAPE;
  const bool f32 = desc->io == GDN2_IO_F32;
  if (desc->dv == 128) {
    if (f32) gdn2::token_epilogue_kernel<float, 128><<<(unsigned)blocks, gdn2::kTokThreads, 0, stream>>>(a);
    else gdn2::token_epilogue_kernel<bf16, 128><<<(unsigned)blocks, gdn2::kTokThreads, 0, stream>>>(a);
  } else {
    if (f32) gdn2::token_epilogue_kernel<float, 64><<<(unsigned)blocks, gdn2::kTokThreads, 0, stream>>>(a);
    else gdn2::token_epilogue_kernel<bf16, 64><<<(unsigned)blocks, gdn2::kTokThreads, 0, stream>>>(a);
  }
  return launch_status();
}

gdn2_status gdn2_recurrent_step(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* b, const float* w, float scale,
                                float* state, void* out, cudaStream_t stream) {
  if (!desc) return GDN2_ERR_NULL;
  if (desc->io != GDN2_IO_F32 && desc->io != GDN2_IO_BF16) return GDN2_ERR_DTYPE;
  if ((desc->dk != 64 && desc->dk != 128) || (desc->dv != 64 && desc->dv != 128)) return GDN2_ERR_SHAPE;
  if (desc->B < 0 || desc->H < 1) return GDN2_ERR_SHAPE;
  gdn2_status st = check_inputs(q, k, v, log_alpha, b, w, desc->B);
  if (st != GDN2_OK) return st;
  if (desc->B > 0 && (!state || !out)) return GDN2_ERR_NULL;
  if (!aligned16(state) || !aligned16(out)) return GDN2_ERR_ALIGN;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  return dispatch<DecodeOp>(desc, q, k, v, log_alpha, b, w, scale, state, out, stream);
}

const char* gdn2_status_string(gdn2_status s) {
  switch (s) {
    case GDN2_OK: return "ok";
    case GDN2_ERR_NULL: return "a required pointer is NULL";
    case GDN2_ERR_SHAPE: return "unsupported or inconsistent sizes";
    case GDN2_ERR_DTYPE: return "unknown io dtype";
    case GDN2_ERR_ALIGN: return "a pointer is not 16-byte aligned (workspace: 256-byte)";
    case GDN2_ERR_SEQLENS: return "cu_seqlens is malformed";
    case GDN2_ERR_WORKSPACE: return "workspace missing or too small";
    case GDN2_ERR_CUDA: return "a CUDA call or kernel launch failed";
    case GDN2_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait gave up";
    case GDN2_ERR_UNSUPPORTED: return "the current device is not sm_100 (B200 class)";
  }
  return "unknown status";
}

int gdn2_version(void) { return 100; }

size_t gdn2_backward_workspace_size(const gdn2_desc* desc) {
  if (!desc) return 0;
  BwdLayout B;
  if (bwd_layout(desc, desc->num_seqs > 0, &B) != GDN2_OK) return 0;
  return B.total;
}

gdn2_status gdn2_chunk_bwd(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                           const float* log_alpha, const float* b, const float* w, float scale, const float* h0,
                           const int32_t* cu_seqlens, const void* dO, const float* dhT, float* dq, float* dk,
                           float* dv, float* dlog_alpha, float* db, float* dw, float* dh0, cudaStream_t stream) {
  if (!desc) return GDN2_ERR_NULL;
  const bool packed = cu_seqlens != nullptr;
  BwdLayout B;
  gdn2_status st = bwd_layout(desc, packed, &B);
  if (st != GDN2_OK) return st;
  if (!desc->workspace) return GDN2_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(desc->workspace) & (kAlign - 1)) != 0) return GDN2_ERR_ALIGN;
  if (desc->workspace_bytes < B.total) return GDN2_ERR_WORKSPACE;
  const long long tokens = (long long)desc->B * desc->T;
  if ((st = check_inputs(q, k, v, log_alpha, b, w, tokens)) != GDN2_OK) return st;
  if (tokens > 0 && (!dO || !dq || !dk || !dv || !dlog_alpha || !db || !dw)) return GDN2_ERR_NULL;
  if (!dh0) return GDN2_ERR_NULL;
  if (!aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dlog_alpha) ||
      !aligned16(db) || !aligned16(dw) || !aligned16(dh0) || (h0 && !aligned16(h0)) || (dhT && !aligned16(dhT)))
    return GDN2_ERR_ALIGN;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  int* status = at<int32_t>(desc->workspace, 0);
  if (cudaMemsetAsync(status, 0, sizeof(int32_t), stream) != cudaSuccess) return GDN2_ERR_CUDA;
  if (packed && tokens > 0) {
    // every token of a well-formed packing belongs to one chunk, which writes
    // all of its gradients; a malformed one leaves the chunk map empty, and
    // the gradients must then read as zero
    const size_t kbytes = (size_t)tokens * desc->H * desc->dk * sizeof(float);
    const size_t vbytes = (size_t)tokens * desc->H * desc->dv * sizeof(float);
    for (float* p : {dq, dk, dlog_alpha, db})
      if (cudaMemsetAsync(p, 0, kbytes, stream) != cudaSuccess) return GDN2_ERR_CUDA;
    for (float* p : {dv, dw})
      if (cudaMemsetAsync(p, 0, vbytes, stream) != cudaSuccess) return GDN2_ERR_CUDA;
  }
  return dispatch<BwdOp>(desc, B, q, k, v, log_alpha, b, w, scale, h0, cu_seqlens, dO, dhT, dq, dk, dv, dlog_alpha,
                         db, dw, dh0, stream);
}

}  // extern "C"

// ------------------------------------------------------- no-alloc variant ----
// The scratch of gdn2_chunk_fwd_noalloc: part of the library's device image,
// one copy per device, shared by every call.  In host code the symbol is only
// a stand-in; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GDN2_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of the scratch on the current device.  It is looked up on
// every call (a host-side query once the module is loaded), so a module that
// was reloaded at another address (after cudaDeviceReset, or under another
// context) is never reached through a stale pointer.
gdn2_status noalloc_scratch(void** addr) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GDN2_ERR_CUDA;
  *addr = p;
  return GDN2_OK;
}
}  // namespace

extern "C" {

gdn2_status gdn2_chunk_fwd_noalloc(const gdn2_desc* desc, const void* q, const void* k, const void* v,
                                   const float* log_alpha, const float* b, const float* w, float scale,
                                   const float* h0, const int32_t* cu_seqlens, void* out, float* hT,
                                   cudaStream_t stream) {
  if (!desc) return GDN2_ERR_NULL;
  gdn2_desc d = *desc;
  d.workspace = nullptr;
  d.workspace_bytes = 0;
  Layout L;
  gdn2_status st = make_layout(&d, cu_seqlens != nullptr, &L);
  if (st != GDN2_OK) return st;
  if (L.l.total_bytes > (size_t)GDN2_NOALLOC_SCRATCH_BYTES) return GDN2_ERR_WORKSPACE;
  const long long tokens = (long long)d.B * d.T;
  if ((st = check_inputs(q, k, v, log_alpha, b, w, tokens)) != GDN2_OK) return st;
  if (!out && tokens > 0) return GDN2_ERR_NULL;
  if (!aligned16(out) || (h0 && !aligned16(h0)) || (hT && !aligned16(hT))) return GDN2_ERR_ALIGN;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != GDN2_OK) return st;
  d.workspace = scratch;
  d.workspace_bytes = (size_t)GDN2_NOALLOC_SCRATCH_BYTES;
  return gdn2_chunk_fwd(&d, q, k, v, log_alpha, b, w, scale, h0, cu_seqlens, out, hT, stream);
}

}  // extern "C"

extern "C" {

gdn2_status gdn2_noalloc_status(const gdn2_desc* desc, int32_t* status, cudaStream_t stream) {
  if (!desc || !status) return GDN2_ERR_NULL;
  if (!aligned16(status)) return GDN2_ERR_ALIGN;
  gdn2_desc d = *desc;
  d.workspace = nullptr;
  d.workspace_bytes = 0;
  Layout L;
  gdn2_status st = make_layout(&d, d.num_seqs > 0, &L);
  if (st != GDN2_OK) return st;
  if (L.l.total_bytes > (size_t)GDN2_NOALLOC_SCRATCH_BYTES) return GDN2_ERR_WORKSPACE;
  if (!device_ok()) return GDN2_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != GDN2_OK) return st;
  if (cudaMemcpyAsync(status, static_cast<char*>(scratch) + L.l.off_status, sizeof(int32_t),
                      cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
    return GDN2_ERR_CUDA;
  return GDN2_OK;
}

}  // extern "C"
