// decode.cuh -- one decode token of the Gated Delta Rule-2 recurrence on a
// batch of states, updated in place (constant-memory decoding).
//
// The step is a single pass over each dk x dv fp32 state: it is bound by HBM
// (read and write every state value once).  One CTA per (batch, head) and
// value-column group: thread (r, j) owns column j for the key rows
// r, r + RG, r + 2 RG, ..., so every warp loads and stores whole 128-byte
// row segments.  Two reductions over the key axis (r = Sbar^T e and
// o = S^T q) go through shared memory.
//   Sbar = diag(exp(log_alpha)) S,  r = Sbar^T (b * k),  u = w * v - r,
//   S    = Sbar + k u^T,            o = scale * S^T q
#pragma once

#include "common.cuh"

namespace gdn2 {

template <typename IO>
struct DecodeArgs {
  const IO* q;
  const IO* k;
  const IO* v;
  const float* la;
  const float* b;
  const float* w;
  float* state;
  IO* out;
  int H;
  float scale;
};

constexpr int kDecodeThreads = 256;

template <int DK, int DV, typename IO>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(const DecodeArgs<IO> a) {
  constexpr int COLS = DV < 32 ? DV : 32;             // columns per CTA
  constexpr int RG = kDecodeThreads / COLS;            // row groups
  constexpr int RPT = DK / RG;                         // rows per thread
  static_assert(DK % RG == 0, "rows divide evenly");
  const int groups = DV / COLS;
  const int bh = blockIdx.x / groups;
  const int j0 = (blockIdx.x % groups) * COLS;
  const int h = bh % a.H;
  const int tid = threadIdx.x;
  const int j = tid % COLS, r = tid / COLS;

  __shared__ float s_alpha[DK], s_e[DK], s_k[DK], s_q[DK];
  __shared__ float s_part[RG][COLS];
  __shared__ float s_u[COLS];
  const size_t vk = (size_t)bh * DK;
  for (int c = tid; c < DK; c += kDecodeThreads) {
    const float kc = to_f32(a.k[vk + c]);
    s_k[c] = kc;
    s_e[c] = a.b[vk + c] * kc;
    s_q[c] = to_f32(a.q[vk + c]);
    s_alpha[c] = expf(a.la[vk + c]);
  }
  __syncthreads();
  float* S = a.state + (size_t)bh * DK * DV + j0 + j;
  float s[RPT];
  float racc = 0.f;
#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    const int c = r + m * RG;
    s[m] = S[(size_t)c * DV] * s_alpha[c];
    racc = fmaf(s[m], s_e[c], racc);
  }
  s_part[r][j] = racc;
  __syncthreads();
  if (r == 0) {
    float rr = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) rr += s_part[g][j];
    const size_t vo = (size_t)bh * DV + j0 + j;
    s_u[j] = a.w[vo] * to_f32(a.v[vo]) - rr;
  }
  __syncthreads();
  const float u = s_u[j];
  float oacc = 0.f;
#pragma unroll
  for (int m = 0; m < RPT; ++m) {
    const int c = r + m * RG;
    s[m] = fmaf(s_k[c], u, s[m]);
    S[(size_t)c * DV] = s[m];
    oacc = fmaf(s[m], s_q[c], oacc);
  }
  __syncthreads();  // everyone has read s_part for r
  s_part[r][j] = oacc;
  __syncthreads();
  if (r == 0) {
    float oo = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) oo += s_part[g][j];
    a.out[(size_t)bh * DV + j0 + j] = from_f32<IO>(a.scale * oo);
  }
}

}  // namespace gdn2
