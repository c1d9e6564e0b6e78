// bwd_simt.cuh -- gradients of the forward operator on the CUDA cores (fp32
// arithmetic, fp32 or bf16 inputs, dk and dv in {64, 128}).
//
// Reverse mode through the token recurrence (page "Gated DeltaNet-2：将擦除与写入分开",
// section "在两个维度上独立控制": e = b k, z = w v, Sbar = diag(alpha) S,
// r = Sbar^T e, S = Sbar + k (z - r)^T, o = scale S^T q; the pages train with
// it, section "词元路径与并行训练").  The value columns of the state evolve
// independently, so one CTA takes kBwdCols columns of one (sequence, head),
// a thread per key row:
//
//   1. forward over the sequence, storing the state at the start of every
//      64-token chunk (checkpoints in the workspace);
//   2. the chunks in reverse order: the chunk's token states are recomputed
//      from its checkpoint into shared memory, then the tokens in reverse,
//      with dS (the gradient reaching the state) in registers:
//        dS += scale q dO^T;  dq = scale S_t dO
//        u = z - r;  dk = dS u;  du = dS^T k;  dr = -du
//        dSbar = dS + e dr^T;  de = Sbar dr;  db = de k;  dk += de b
//        dw = du v;  dv = du w
//        dlog_alpha = alpha * rowsum(dSbar * S_{t-1});  dS = diag(alpha) dSbar
//   3. dh0 = dS after the first token.
//
// The key-side gradients (dq, dk, db, dlog_alpha) sum over the value columns
// of every CTA of the head: they are added with atomics into outputs the host
// zeroes first.  The value-side ones (dv, dw) and dh0 belong to one CTA.
#pragma once

#include "common.cuh"

namespace gdn2 {

constexpr int kBwdCols = 2;  // value columns per CTA

template <typename IO>
struct BwdArgs {
  const IO *q, *k, *v, *dO;       // [T_total, H, d]
  const float *la, *b, *w;        // [T_total, H, d]
  const float *h0, *dhT;          // [N, H, dk, dv] or nullptr (zero)
  const int32_t* cu;              // packed boundaries or nullptr (dense)
  int N, T, T_total, H;
  float scale;
  float* ckpt;                    // [slots, H, dk, dv]: slot of chunk m of sequence n = seq_begin(n) / 64 + m + n
  float *dq, *dk, *dla, *db;      // [T_total, H, dk], zeroed by the host, added to
  float *dv, *dw;                 // [T_total, H, dv]
  float* dh0;                     // [N, H, dk, dv]
  int* status;
  int seqlens_err;
};

template <int NW, int CB>
__device__ __forceinline__ void bwd_block_sum(float (&x)[CB], float* red, int& parity) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
  for (int j = 0; j < CB; ++j) x[j] = warp_sum(x[j]);
  float* rb = red + parity * NW * CB;
  if (lane == 0)
#pragma unroll
    for (int j = 0; j < CB; ++j) rb[wid * CB + j] = x[j];
  __syncthreads();
#pragma unroll
  for (int j = 0; j < CB; ++j) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) s += rb[w * CB + j];
    x[j] = s;
  }
  // two buffers: the next sum writes the other one, and the one after that
  // comes after the next sum's barrier, when every thread has read this one
  parity ^= 1;
}

template <int DK, int DV>
constexpr int bwd_smem_floats() {
  return (kChunk + 1) * DK * kBwdCols + kChunk * kBwdCols + 2 * (DK / 32) * kBwdCols;
}

template <int DK, int DV, typename IO>
__global__ void __launch_bounds__(DK) bwd_simt_kernel(const BwdArgs<IO> a) {
  constexpr int CB = kBwdCols, NCB = DV / CB, NW = DK / 32;
  extern __shared__ float bwd_smem[];
  float* Ssm = bwd_smem;                            // [kChunk + 1][DK][CB] states of one chunk
  float* rsm = Ssm + (kChunk + 1) * DK * CB;        // [kChunk][CB] r of each token
  float* red = rsm + kChunk * CB;                   // [2][NW][CB]
  const int c = threadIdx.x;
  const int cb = blockIdx.x % NCB, h = (blockIdx.x / NCB) % a.H, n = blockIdx.x / (NCB * a.H);
  const int col0 = cb * CB;
  int s0, s1;
  if (a.cu) {
    s0 = a.cu[n];
    s1 = a.cu[n + 1];
    // every access below stays inside [s0, s1), so a range inside the tokens
    // is all this CTA needs; a bad one is reported and nothing is touched
    if (s0 < 0 || s1 < s0 || s1 > a.T_total) {
      if (c == 0) atomicExch(a.status, a.seqlens_err);
      return;
    }
  } else {
    s0 = n * a.T;
    s1 = s0 + a.T;
  }
  const size_t st_row = (((size_t)n * a.H + h) * DK + c) * DV + col0;  // this thread's row of h0 / hT / dh0
  auto ck_row = [&](int slot) { return a.ckpt + (((size_t)slot * a.H + h) * DK + c) * DV + col0; };
  const int slot0 = s0 / kChunk + n;
  int parity = 0;

  // one token of the forward: S <- diag(alpha) S + k (z - Sbar^T e)^T; r out
  auto fwd_step = [&](int t, float (&S)[CB], float (&r)[CB]) {
    const size_t tk = ((size_t)t * a.H + h) * DK + c, tv = ((size_t)t * a.H + h) * DV + col0;
    const float alpha = expf(a.la[tk]), kc = to_f32(a.k[tk]), ec = a.b[tk] * kc;
    float sb[CB];
#pragma unroll
    for (int j = 0; j < CB; ++j) {
      sb[j] = alpha * S[j];
      r[j] = sb[j] * ec;
    }
    bwd_block_sum<NW, CB>(r, red, parity);
#pragma unroll
    for (int j = 0; j < CB; ++j) S[j] = sb[j] + kc * (a.w[tv + j] * to_f32(a.v[tv + j]) - r[j]);
  };

  // 1. forward with a checkpoint at every chunk start
  {
    float S[CB], r[CB];
#pragma unroll
    for (int j = 0; j < CB; ++j) S[j] = a.h0 ? a.h0[st_row + j] : 0.f;
    for (int t0 = s0, m = 0; t0 < s1; t0 += kChunk, ++m) {
      float* ck = ck_row(slot0 + m);
#pragma unroll
      for (int j = 0; j < CB; ++j) ck[j] = S[j];
      const int t1 = min(t0 + kChunk, s1);
      for (int t = t0; t < t1; ++t) fwd_step(t, S, r);
    }
  }

  // 2. the chunks in reverse
  float dS[CB];
#pragma unroll
  for (int j = 0; j < CB; ++j) dS[j] = a.dhT ? a.dhT[st_row + j] : 0.f;
  const int nch = (s1 - s0 + kChunk - 1) / kChunk;
  for (int m = nch - 1; m >= 0; --m) {
    const int t0 = s0 + m * kChunk, nt = min(kChunk, s1 - t0);
    {
      float S[CB], r[CB];
      const float* ck = ck_row(slot0 + m);
#pragma unroll
      for (int j = 0; j < CB; ++j) {
        S[j] = ck[j];
        Ssm[c * CB + j] = S[j];
      }
      for (int i = 0; i < nt; ++i) {
        fwd_step(t0 + i, S, r);
#pragma unroll
        for (int j = 0; j < CB; ++j) Ssm[((i + 1) * DK + c) * CB + j] = S[j];
        if (c == 0)
#pragma unroll
          for (int j = 0; j < CB; ++j) rsm[i * CB + j] = r[j];
      }
    }
    __syncthreads();  // r of every token visible to all threads
    for (int i = nt - 1; i >= 0; --i) {
      const int t = t0 + i;
      const size_t tk = ((size_t)t * a.H + h) * DK + c, tv = ((size_t)t * a.H + h) * DV + col0;
      const float alpha = expf(a.la[tk]), kc = to_f32(a.k[tk]), bc = a.b[tk], ec = bc * kc;
      const float qc = to_f32(a.q[tk]);
      float Sp[CB], vj[CB], wj[CB], u[CB], du[CB];
      float dq_part = 0.f, dk_part = 0.f;
#pragma unroll
      for (int j = 0; j < CB; ++j) {
        Sp[j] = Ssm[(i * DK + c) * CB + j];
        const float Sc = Ssm[((i + 1) * DK + c) * CB + j];
        const float dOj = to_f32(a.dO[tv + j]);
        vj[j] = to_f32(a.v[tv + j]);
        wj[j] = a.w[tv + j];
        u[j] = wj[j] * vj[j] - rsm[i * CB + j];
        dS[j] += a.scale * qc * dOj;      // o_t reads S_t
        dq_part += Sc * dOj;
      }
#pragma unroll
      for (int j = 0; j < CB; ++j) {
        dk_part += dS[j] * u[j];          // S_t = Sbar + k u^T
        du[j] = dS[j] * kc;
      }
      bwd_block_sum<NW, CB>(du, red, parity);
      float de = 0.f, dal = 0.f;
#pragma unroll
      for (int j = 0; j < CB; ++j) {
        const float dr = -du[j];
        const float dsb = dS[j] + ec * dr;  // direct term, and r = Sbar^T e
        de += alpha * Sp[j] * dr;
        dal += dsb * Sp[j];
        dS[j] = alpha * dsb;                // into S_{t-1}
      }
      atomicAdd(a.dq + tk, a.scale * dq_part);
      atomicAdd(a.dk + tk, dk_part + de * bc);
      atomicAdd(a.db + tk, de * kc);
      atomicAdd(a.dla + tk, dal * alpha);
#pragma unroll
      for (int j = 0; j < CB; ++j)
        if (c == j) {
          a.dw[tv + j] = du[j] * vj[j];
          a.dv[tv + j] = du[j] * wj[j];
        }
    }
    __syncthreads();  // every thread is done with rsm before the next chunk rewrites it
  }

  // 3. what reaches the initial state
#pragma unroll
  for (int j = 0; j < CB; ++j) a.dh0[st_row + j] = dS[j];
}

}  // namespace gdn2
