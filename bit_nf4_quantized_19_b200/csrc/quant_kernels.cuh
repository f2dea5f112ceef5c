// Blockwise NF4 quantization with double quantization, and standalone dequant.
// Sources: "QLoRA" (ozercemkelahmet.com/tools/qlora), How it works, Steps 1-3 and
// "A worked example"; "QLoRA: Efficient Finetuning of Quantized LLMs"
// (crackai.dev), How It Works 1-2.
#pragma once
#include "common.cuh"
#include "nf4_table.hpp"

namespace qlora {

constexpr int kBlock = 64;                 // values per first-level block
constexpr int kGroup = 256;                // blocks per second-level constant
constexpr int kGroupElems = kBlock * kGroup;

struct QuantTables {
  QuantBin bins[kQuantBins];   // indexed by round(32 * xn) mod 128
  float rcp[128];              // RN32(1 / (1 + k/128)): reciprocals of the bf16 mantissas
};
struct Levels {
  float v[16];
};

// One CTA per group of 256 blocks (16384 values); 256 threads; 8 threads per
// block, each owning 8 consecutive values (one 16-byte load), 32 blocks per pass,
// 8 passes.  All eight 16-byte loads are issued before any arithmetic.
//   absmax: max |w| within the thread, then an xor-shuffle over the 8 lanes;
//   xn:     RN32(w / a_b).  For 2^-64 <= a_b <= 2^64 (every realistic block) the
//           division is Markstein's FMA correction of w * RN32(1/a_b), where
//           RN32(1/a_b) is an exact power-of-two scaling of a table entry because
//           a_b is a bf16 value; outside that range, IEEE division.  An exhaustive
//           host check over all bf16 pairs of the fast range shows both give the
//           same code for every input (tests/csrc/division_check.c);
//   code:   bin j = round(32 xn) (exact, from the sum 32 xn + 1.5*2^23), then
//           code = bins[j].c + (xn > bins[j].t): the number of decision thresholds
//           below xn, i.e. the nearest level with ties to the lower index;
//   pack:   8 codes -> one 32-bit word (element 2j in the low nibble of byte j);
//   double quant (after all passes): c_g = max a_b over the group,
//           step = RN32(c_g / 255), q8 = min(255, rint(RN32(a_b / step))).
__global__ void __launch_bounds__(256, 3) nf4_quantize_kernel(
    const uint16_t *__restrict__ W, int64_t n, uint8_t *__restrict__ codes,
    uint8_t *__restrict__ q8, float *__restrict__ step, const __grid_constant__ QuantTables tab) {
  __shared__ QuantBin bins[kQuantBins];
  __shared__ float rcp[128];
  __shared__ float amax[kGroup];
  __shared__ float wmax[8];
  const int tid = threadIdx.x;
  if (tid < kQuantBins) bins[tid] = tab.bins[tid];
  if (tid < 128) rcp[tid] = tab.rcp[tid];

  const int64_t g = blockIdx.x;
  const int64_t gbase = g * kGroupElems;
  const int sub = tid & 7;
  const int bl = tid >> 3;

  uint4 v[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int64_t e = gbase + static_cast<int64_t>(p * 32 + bl) * kBlock + sub * 8;
    if (e + 8 <= n) {
      v[p] = ld_global_nc_v4(W + e);
    } else {
      uint32_t t[4] = {0, 0, 0, 0};
      for (int j = 0; j < 8; ++j)
        if (e + j < n) t[j >> 1] |= static_cast<uint32_t>(W[e + j]) << (16 * (j & 1));
      v[p] = make_uint4(t[0], t[1], t[2], t[3]);
    }
  }
  __syncthreads();

  bool nonfinite = false;
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int64_t e = gbase + static_cast<int64_t>(p * 32 + bl) * kBlock + sub * 8;
    const uint32_t wd[4] = {v[p].x, v[p].y, v[p].z, v[p].w};
    float w[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      w[2 * j] = bf16_lo(wd[j]);
      w[2 * j + 1] = bf16_hi(wd[j]);
    }
    float am = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) am = fmaxf(am, fabsf(w[j]));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 4));
    if (!(am <= 3.402823466e38f)) nonfinite = true;
    const bool fast = (am >= 0x1p-64f) && (am <= 0x1p64f);
    // RN32(1/am) = RN32(1/m) * 2^-e for am = m * 2^e (m has 7 fraction bits)
    const uint32_t ab = __float_as_uint(am);
    const int ex = static_cast<int>((ab >> 23) & 0xFFu) - 127;
    const float y = __uint_as_float(__float_as_uint(rcp[(ab >> 16) & 127u]) - (static_cast<uint32_t>(ex) << 23));
    uint32_t word = 0;
    if (__all_sync(0xffffffffu, fast)) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float q0 = __fmul_rn(w[j], y);
        const float r = __fmaf_rn(-q0, am, w[j]);
        const float xn = __fmaf_rn(r, y, q0);
        const float f = __fmaf_rn(xn, 32.0f, 12582912.0f);
        const QuantBin b = bins[__float_as_uint(f) & (kQuantBins - 1)];
        word |= static_cast<uint32_t>(b.c + (xn > b.t ? 1 : 0)) << (4 * j);
      }
    } else {
      const float a = (am > 0.f) ? am : 1.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        float xn;
        if (fast) {
          const float q0 = __fmul_rn(w[j], y);
          const float r = __fmaf_rn(-q0, am, w[j]);
          xn = __fmaf_rn(r, y, q0);
        } else {
          xn = __fdiv_rn(w[j], a);
        }
        const float f = __fmaf_rn(xn, 32.0f, 12582912.0f);
        const QuantBin b = bins[__float_as_uint(f) & (kQuantBins - 1)];
        word |= static_cast<uint32_t>(b.c + (xn > b.t ? 1 : 0)) << (4 * j);
      }
    }
    if (e + 8 <= n) {
      *reinterpret_cast<uint32_t *>(codes + (e >> 1)) = word;
    } else if (e < n) {
      const int valid = static_cast<int>(n - e);           // 1..7
      const uint32_t keep = (1u << (4 * valid)) - 1u;      // zero the nibbles past n
      word &= keep;
      const int nbytes = (valid + 1) >> 1;
      for (int j = 0; j < nbytes; ++j) codes[(e >> 1) + j] = static_cast<uint8_t>(word >> (8 * j));
    }
    if (sub == 0) amax[p * 32 + bl] = am;
  }
  if (nonfinite && sub == 0) atomicOr(&g_device_status, kStatNonFinite);
  __syncthreads();

  // second level: one constant per group
  const int64_t nblocks = (n + kBlock - 1) / kBlock;
  const int64_t b = g * kGroup + tid;
  const float a = (b < nblocks) ? amax[tid] : 0.f;
  float m = a;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((tid & 31) == 0) wmax[tid >> 5] = m;
  __syncthreads();
  float c = wmax[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) c = fmaxf(c, wmax[i]);
  const float st = (c > 0.f) ? __fdiv_rn(c, 255.0f) : 0.f;
  if (b < nblocks) {
    int q = 0;
    if (c > 0.f) q = min(255, __float2int_rn(__fdiv_rn(a, st)));
    q8[b] = static_cast<uint8_t>(q);
  }
  if (tid == 0) step[g] = st;
}

// Standalone dequant: 16 values per thread per iteration (8 bytes of codes in,
// 32 bytes of bf16 out), grid-stride.  w = bf16_RN(RN32(L[code] * RN32(q8*step))).
__global__ void __launch_bounds__(256) nf4_dequant_kernel(
    const uint8_t *__restrict__ codes, const uint8_t *__restrict__ q8,
    const float *__restrict__ step, int64_t n, uint16_t *__restrict__ out,
    const __grid_constant__ Levels lv) {
  __shared__ float L[16];
  if (threadIdx.x < 16) L[threadIdx.x] = lv.v[threadIdx.x];
  __syncthreads();
  const int64_t units = n >> 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < units;
       u += stride) {
    const int64_t e = u << 4;
    const uint2 c = *reinterpret_cast<const uint2 *>(codes + (e >> 1));
    const int64_t b = e >> 6;
    const float sc = __fmul_rn(static_cast<float>(q8[b]), step[b >> 8]);
    uint32_t o[8];
    const uint32_t cw[2] = {c.x, c.y};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t byte = (cw[h] >> (8 * j)) & 0xFFu;
        o[h * 4 + j] = pack_bf16x2(__fmul_rn(L[byte & 15u], sc), __fmul_rn(L[byte >> 4], sc));
      }
    }
    uint4 *dst = reinterpret_cast<uint4 *>(out + e);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
  // tail (n % 16 values), one thread
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    for (int64_t e = units << 4; e < n; ++e) {
      const uint8_t byte = codes[e >> 1];
      const uint32_t code = (e & 1) ? (byte >> 4) : (byte & 15u);
      const int64_t b = e >> 6;
      const float sc = __fmul_rn(static_cast<float>(q8[b]), step[b >> 8]);
      const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(L[code], sc));
      out[e] = *reinterpret_cast<const uint16_t *>(&h);
    }
  }
}

// Per-block constants expanded for the fused GEMM, stored transposed:
// S[kb][n] = RN32(q8[n*KB + kb] * step[(n*KB + kb) / 256]),  KB = K / 64.
__global__ void __launch_bounds__(256) nf4_expand_scales_kernel(
    const uint8_t *__restrict__ q8, const float *__restrict__ step, int N, int KB,
    float *__restrict__ S) {
  const int64_t total = static_cast<int64_t>(N) * KB;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int kb = static_cast<int>(i / N);
    const int nrow = static_cast<int>(i - static_cast<int64_t>(kb) * N);
    const int64_t b = static_cast<int64_t>(nrow) * KB + kb;
    S[i] = __fmul_rn(static_cast<float>(q8[b]), step[b >> 8]);
  }
}

}  // namespace qlora
