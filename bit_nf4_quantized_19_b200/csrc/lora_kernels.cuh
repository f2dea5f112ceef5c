// Rank-r adapter products of the QLoRA linear layer ("QLoRA", ozercemkelahmet.com,
// How it works, Steps 4-6): XA = X A and G = dY B^T (projections to rank r), and
// the adapter gradients dA = s X^T G, dB = s XA^T dY.  fp32 accumulation in a
// fixed order (deterministic).  The projections also emit s*P split into bf16
// hi/lo halves, the operand of the LoRA K-steps of the fused GEMM.
#pragma once
#include "common.cuh"

namespace qlora {

constexpr int kProjTM = 32;     // tokens per CTA
constexpr int kProjKC = 64;     // contraction chunk
constexpr int kProjThreads = 128;

// out[m][j] = sum_c P[m][c] * Q(c, j), Q(c, j) = Q[c*r + j] (q_rows_are_c) or Q[j*C + c].
// P bf16 [M, C]; Q bf16; out fp32 [M, r]; hl bf16 [M, 2r] = hi/lo of s*out.
// Thread t: token m = t/4, column quads jq = (t%4) + 4i.
__global__ void __launch_bounds__(kProjThreads) lora_project_kernel(
    const uint16_t *__restrict__ P, int M, int C, const uint16_t *__restrict__ Q,
    int q_rows_are_c, int r, float s, float *__restrict__ out, uint16_t *__restrict__ hl) {
  extern __shared__ float psm[];
  float *Ps = psm;                          // [kProjTM][kProjKC + 1]
  float *Qs = Ps + kProjTM * (kProjKC + 1); // [kProjKC][r]
  const int tid = threadIdx.x;
  const int m_base = blockIdx.x * kProjTM;
  const int ml = tid >> 2;
  const int jg = tid & 3;
  const int nquads = r / 4;
  float acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = 0.f;

  for (int c0 = 0; c0 < C; c0 += kProjKC) {
    for (int i = tid; i < kProjTM * kProjKC; i += kProjThreads) {
      const int mm = i / kProjKC, cc = i % kProjKC;
      const int m = m_base + mm;
      float v = 0.f;
      if (m < M) v = __uint_as_float(static_cast<uint32_t>(P[static_cast<int64_t>(m) * C + c0 + cc]) << 16);
      Ps[mm * (kProjKC + 1) + cc] = v;
    }
    for (int i = tid; i < kProjKC * r; i += kProjThreads) {
      const int cc = i / r, j = i % r;
      const uint16_t q = q_rows_are_c ? Q[static_cast<int64_t>(c0 + cc) * r + j]
                                      : Q[static_cast<int64_t>(j) * C + c0 + cc];
      Qs[cc * r + j] = __uint_as_float(static_cast<uint32_t>(q) << 16);
    }
    __syncthreads();
    for (int cc = 0; cc < kProjKC; ++cc) {
      const float x = Ps[ml * (kProjKC + 1) + cc];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int jq = jg + 4 * i;
        if (jq < nquads) {
          const float4 q4 = *reinterpret_cast<const float4 *>(&Qs[cc * r + 4 * jq]);
          acc[4 * i + 0] = fmaf(x, q4.x, acc[4 * i + 0]);
          acc[4 * i + 1] = fmaf(x, q4.y, acc[4 * i + 1]);
          acc[4 * i + 2] = fmaf(x, q4.z, acc[4 * i + 2]);
          acc[4 * i + 3] = fmaf(x, q4.w, acc[4 * i + 3]);
        }
      }
    }
    __syncthreads();
  }
  const int m = m_base + ml;
  if (m >= M) return;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int jq = jg + 4 * i;
    if (jq >= nquads) continue;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * jq + e;
      const float v = acc[4 * i + e];
      out[static_cast<int64_t>(m) * r + j] = v;
      const float sv = s * v;
      const __nv_bfloat16 h = __float2bfloat16_rn(sv);
      const __nv_bfloat16 l = __float2bfloat16_rn(sv - __bfloat162float(h));
      hl[static_cast<int64_t>(m) * 2 * r + j] = *reinterpret_cast<const uint16_t *>(&h);
      hl[static_cast<int64_t>(m) * 2 * r + r + j] = *reinterpret_cast<const uint16_t *>(&l);
    }
  }
}

constexpr int kGradCT = 64;     // output columns c per CTA
constexpr int kGradTM = 32;     // tokens per chunk
constexpr int kGradThreads = 128;

// Partial adapter gradient over one token split:
//   part[split][c][j] = sum_{m in split} P[m][c] * F[m][j]
// P bf16 [M, C] (X or dY), F fp32 [M, r] (G or XA).  Thread t: column c = t % 64,
// j = (t / 64) + 2i.
__global__ void __launch_bounds__(kGradThreads) lora_grad_partial_kernel(
    const uint16_t *__restrict__ P, const float *__restrict__ F, int M, int C, int r,
    int tokens_per_split, float *__restrict__ part) {
  extern __shared__ float gsm[];
  float *Ps = gsm;                          // [kGradTM][kGradCT]
  float *Fs = Ps + kGradTM * kGradCT;       // [kGradTM][r]
  const int tid = threadIdx.x;
  const int c0 = blockIdx.x * kGradCT;
  const int split = blockIdx.y;
  const int m_lo = split * tokens_per_split;
  const int m_hi = min(M, m_lo + tokens_per_split);
  const int cl = tid & 63;
  const int jh = tid >> 6;
  float acc[64];
#pragma unroll
  for (int i = 0; i < 64; ++i) acc[i] = 0.f;
  for (int mb = m_lo; mb < m_hi; mb += kGradTM) {
    for (int i = tid; i < kGradTM * kGradCT; i += kGradThreads) {
      const int mm = i / kGradCT, cc = i % kGradCT;
      const int m = mb + mm;
      float v = 0.f;
      if (m < m_hi && c0 + cc < C)
        v = __uint_as_float(static_cast<uint32_t>(P[static_cast<int64_t>(m) * C + c0 + cc]) << 16);
      Ps[i] = v;
    }
    for (int i = tid; i < kGradTM * r; i += kGradThreads) {
      const int mm = i / r, j = i % r;
      const int m = mb + mm;
      Fs[i] = (m < m_hi) ? F[static_cast<int64_t>(m) * r + j] : 0.f;
    }
    __syncthreads();
    for (int mm = 0; mm < kGradTM; ++mm) {
      const float x = Ps[mm * kGradCT + cl];
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const int j = jh + 2 * i;
        if (j < r) acc[i] = fmaf(x, Fs[mm * r + j], acc[i]);
      }
    }
    __syncthreads();
  }
  if (c0 + cl >= C) return;
  float *dst = part + (static_cast<int64_t>(split) * C + c0 + cl) * r;
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const int j = jh + 2 * i;
    if (j < r) dst[j] = acc[i];
  }
}

// out = s * sum over splits (in split order) of part[split][c][j];
// layout 0: out[c][j] (dA [K, r]); layout 1: out[j][c] (dB [r, N]).
__global__ void __launch_bounds__(256) lora_grad_reduce_kernel(const float *__restrict__ part,
                                                               int splits, int C, int r, float s,
                                                               int layout, float *__restrict__ out) {
  const int64_t total = static_cast<int64_t>(C) * r;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float v = 0.f;
    for (int sp = 0; sp < splits; ++sp) v += part[static_cast<int64_t>(sp) * total + i];
    const int64_t c = i / r, j = i % r;
    if (layout == 0) out[i] = s * v;
    else out[j * C + c] = s * v;
  }
}

}  // namespace qlora
