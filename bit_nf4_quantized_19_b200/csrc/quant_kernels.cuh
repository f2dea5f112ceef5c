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

// Bin table of the quantize kernel, indexed by the low byte of 32 xn + 32 + 1.5*2^23:
// entries 0..64 are the bins round(32 xn) = -32..32; the rest are reachable only from
// a non-finite block and hold an inert bin (t = 2, c = 0).
constexpr int kQuantBins256 = 256;
struct QuantTables {
  QuantBin bins[kQuantBins256];
  float rcp[128];              // RN32(1 / (1 + k/128)): reciprocals of the bf16 mantissas
};
struct Levels {
  float v[16];
};

// Persistent CTAs (one per SM), each looping over groups of 256 blocks (16384
// values); 512 threads; 8 threads per block, each owning 8 consecutive values (one
// 16-byte piece), 64 blocks per pass, 4 passes; the groups arrive through a ring of
// bulk copies (see the kernel).
//   absmax: max |w| within the thread, then an xor-shuffle over the 8 lanes;
//   xn:     RN32(w / a_b).  For 2^-64 <= a_b <= 2^64 (every realistic block) the
//           division is Markstein's FMA correction of w * RN32(1/a_b), where
//           RN32(1/a_b) is an exact power-of-two scaling of a table entry because
//           a_b is a bf16 value; outside that range, IEEE division.  An exhaustive
//           host check over all bf16 pairs of the fast range shows both give the
//           same code for every input (tests/csrc/division_check.c);
//   code:   bin j = round(32 xn) (exact, the low byte of 32 xn + 32 + 1.5*2^23 is
//           j + 32), then code = bins[j].c + (xn > bins[j].t): the number of decision
//           thresholds below xn, i.e. the nearest level with ties to the lower index.
//           Every lane of a half-warp reads its own copy of the bin table (entry i
//           of copy c = lane mod 16 at byte 128 i + 8 c), so the data-dependent
//           lookups never conflict on a bank;
//   pack:   8 codes -> one 32-bit word (element 2j in the low nibble of byte j),
//           accumulated as word = 16 word + code from the last element down;
//   double quant (after all passes): c_g = max a_b over the group,
//           step = RN32(c_g / 255), q8 = min(255, rint(RN32(a_b / step))).
// Markstein's quotient (P. Markstein, "IA-64 and Elementary Functions", 2000) for
// two values at once with the packed fp32 FMA of sm_100 (each lane an IEEE fp32
// operation with a single rounding, subnormals kept): q0 = w*y, r = fma(q0, -a, w),
// xn = fma(r, y, q0); also f = fma(xn, 32, 1.5*2^23 + 32), whose low byte is
// round(32 xn) + 32 for |xn| <= 1.
QDEV void quotient_x2(float w0, float w1, float y, float neg_a, float &xn0, float &xn1, float &f0,
                      float &f1) {
  asm("{\n\t.reg .b64 w, yy, na, q, r, x, k, m, f;\n\t"
      "mov.b64 w, {%4, %5};\n\t"
      "mov.b64 yy, {%6, %6};\n\t"
      "mov.b64 na, {%7, %7};\n\t"
      "mov.b64 k, {%8, %8};\n\t"
      "mov.b64 m, {%9, %9};\n\t"
      "mul.rn.f32x2 q, w, yy;\n\t"
      "fma.rn.f32x2 r, q, na, w;\n\t"
      "fma.rn.f32x2 x, r, yy, q;\n\t"
      "fma.rn.f32x2 f, x, k, m;\n\t"
      "mov.b64 {%0, %1}, x;\n\t"
      "mov.b64 {%2, %3}, f;\n\t}"
      : "=f"(xn0), "=f"(xn1), "=f"(f0), "=f"(f1)
      : "f"(w0), "f"(w1), "f"(y), "f"(neg_a), "f"(32.0f), "f"(12582944.0f));
}

// Byte offset of bin entry i = (low byte of f) for this lane's table copy: entries
// are 128-byte rows of 16 copies, copy (lane mod 16) at 8 (lane mod 16) = lane8.
// A 64-bit shared load is served in two half-warp phases, so 16 copies keep every
// data-dependent lookup conflict-free.
QDEV uint32_t bin_offset(float f, uint32_t lane8) { return ((__float_as_uint(f) * 128u) & 0x7F80u) | lane8; }

// max of two bf16x2 words, lane by lane, NaN-propagating
QDEV uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The NP 16-byte loads of one thread for one group straight from global memory
// (pass p: block (256/NP) p + bl, values 8 sub .. 8 sub + 7), with bounds checks:
// the path of the one group that may end inside the tensor.
template <int NP>
QDEV void quant_load_tail(const uint16_t *__restrict__ W, int64_t n, int64_t gbase, int bl, int sub, uint4 (&v)[NP]) {
  constexpr int BPP = kGroup / NP;
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int64_t e = gbase + static_cast<int64_t>(p * BPP + bl) * kBlock + sub * 8;
    if (e + 8 <= n) {
      v[p] = ld_global_nc_v4(W + e);
    } else {
      uint32_t t[4] = {0, 0, 0, 0};
      for (int j = 0; j < 8; ++j)
        if (e + j < n) t[j >> 1] |= static_cast<uint32_t>(W[e + j]) << (16 * (j & 1));
      v[p] = make_uint4(t[0], t[1], t[2], t[3]);
    }
  }
}

// Codes of one group.  The eight block absmaxes come first, on the packed bf16
// words (|w| is w with the sign bits cleared; NaN propagates), two passes per
// shuffle; one warp vote then picks the path for the whole group.
template <bool WHOLE, int NP>
QDEV void quant_compute(const uint4 (&v)[NP], int64_t n, int64_t gbase, int bl, int sub, const float *rcp,
                        const uint8_t *bins_bytes, uint32_t lane8, uint8_t *__restrict__ codes,
                        float *amax, bool &nonfinite) {
  constexpr int BPP = kGroup / NP;
  float am[NP];
#pragma unroll
  for (int p = 0; p < NP; p += 2) {
    uint32_t m0 = bmax2(bmax2(v[p].x & 0x7FFF7FFFu, v[p].y & 0x7FFF7FFFu), bmax2(v[p].z & 0x7FFF7FFFu, v[p].w & 0x7FFF7FFFu));
    uint32_t m1 = bmax2(bmax2(v[p + 1].x & 0x7FFF7FFFu, v[p + 1].y & 0x7FFF7FFFu),
                        bmax2(v[p + 1].z & 0x7FFF7FFFu, v[p + 1].w & 0x7FFF7FFFu));
    // low half: pass p, high half: pass p + 1
    uint32_t mm = bmax2(prmt(m0, m1, 0x5410u), prmt(m0, m1, 0x7632u));
    mm = bmax2(mm, __shfl_xor_sync(0xffffffffu, mm, 1));
    mm = bmax2(mm, __shfl_xor_sync(0xffffffffu, mm, 2));
    mm = bmax2(mm, __shfl_xor_sync(0xffffffffu, mm, 4));
    am[p] = __uint_as_float(mm << 16);
    am[p + 1] = __uint_as_float(mm & 0xFFFF0000u);
  }
  bool fast = true;
#pragma unroll
  for (int p = 0; p < NP; ++p) fast = fast && (am[p] >= 0x1p-64f) && (am[p] <= 0x1p64f);
  const bool group_fast = __all_sync(0xffffffffu, fast);
  uint8_t *cbase = codes + ((gbase + bl * kBlock + sub * 8) >> 1);
#pragma unroll
  for (int p = 0; p < NP; ++p) {
    const int64_t e = gbase + static_cast<int64_t>(p * BPP + bl) * kBlock + sub * 8;
    const uint32_t wd[4] = {v[p].x, v[p].y, v[p].z, v[p].w};
    float w[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      w[2 * j] = __uint_as_float(wd[j] * 65536u);
      w[2 * j + 1] = bf16_hi(wd[j]);
    }
    const float a_b = am[p];
    // RN32(1/a_b) = RN32(1/m) * 2^-e for a_b = m * 2^e (m has 7 fraction bits)
    const uint32_t ab = __float_as_uint(a_b);
    const int ex = static_cast<int>((ab >> 23) & 0xFFu) - 127;
    const float y = __uint_as_float(__float_as_uint(rcp[(ab >> 16) & 127u]) - (static_cast<uint32_t>(ex) << 23));
    uint32_t word = 0;
    if (group_fast) {
#pragma unroll
      for (int j = 6; j >= 0; j -= 2) {
        float xa, xb, fa, fb;
        quotient_x2(w[j], w[j + 1], y, -a_b, xa, xb, fa, fb);
        const uint2 tb = *reinterpret_cast<const uint2 *>(bins_bytes + bin_offset(fb, lane8));
        const uint2 ta = *reinterpret_cast<const uint2 *>(bins_bytes + bin_offset(fa, lane8));
        // xn > t exactly when t - xn is negative (both finite; no threshold is zero,
        // so the difference is never a negative zero): its sign bit is the increment
        word = word * 16u + tb.y + (__float_as_uint(__fsub_rn(__uint_as_float(tb.x), xb)) >> 31);
        word = word * 16u + ta.y + (__float_as_uint(__fsub_rn(__uint_as_float(ta.x), xa)) >> 31);
      }
    } else {
      const bool fast_b = (a_b >= 0x1p-64f) && (a_b <= 0x1p64f);
      if (!(a_b <= 3.402823466e38f)) nonfinite = true;     // inf or NaN somewhere in the block
      const float a = (a_b > 0.f) ? a_b : 1.0f;
#pragma unroll
      for (int j = 7; j >= 0; --j) {
        float xn;
        if (fast_b) {
          const float q0 = __fmul_rn(w[j], y);
          const float r = __fmaf_rn(-q0, a_b, w[j]);
          xn = __fmaf_rn(r, y, q0);
        } else {
          xn = __fdiv_rn(w[j], a);
        }
        const float f = __fmaf_rn(xn, 32.0f, 12582944.0f);
        const uint2 t = *reinterpret_cast<const uint2 *>(bins_bytes + bin_offset(f, lane8));
        word = word * 16u + t.y + (xn > __uint_as_float(t.x) ? 1u : 0u);
      }
    }
    if (WHOLE || e + 8 <= n) {
      *reinterpret_cast<uint32_t *>(cbase + p * BPP * kBlock / 2) = word;
    } else if (e < n) {
      const int valid = static_cast<int>(n - e);           // 1..7
      const uint32_t keep = (1u << (4 * valid)) - 1u;      // zero the nibbles past n
      word &= keep;
      const int nbytes = (valid + 1) >> 1;
      for (int j = 0; j < nbytes; ++j) codes[(e >> 1) + j] = static_cast<uint8_t>(word >> (8 * j));
    }
    if (sub == 0) amax[p * BPP + bl] = a_b;
  }
}

// Two persistent CTAs of 512 threads per SM (at most 64 registers per thread).  The
// groups a CTA owns stream through a ring of kQuantStages 32 KB buffers, each filled
// by one bulk copy on its own mbarrier (kept kQuantStages groups ahead), so the SM
// always has about 128 KB of loads in flight whatever the compute is doing; the
// compute reads its 16-byte pieces from shared memory (consecutive threads,
// consecutive pieces).  The one group that may end inside the tensor takes
// bounds-checked global loads.
constexpr int kQuantThreads = 512;
constexpr int kQuantStages = 2;
constexpr int kQuantCtasPerSm = 2;
constexpr int kQuantCopies = 16;                                  // bin-table copies
constexpr int kQuantPasses = kGroupElems / (kQuantThreads * 8);   // 4
constexpr int kQuantStageBytes = kGroupElems * 2;                 // 32 KB
constexpr int kQuantSmemBytes = kQuantStages * kQuantStageBytes + kQuantBins256 * kQuantCopies * 8 +
                                (128 + kGroup + 16) * 4 + kQuantStages * 8 + 16;

__global__ void __launch_bounds__(kQuantThreads, kQuantCtasPerSm) nf4_quantize_kernel(
    const uint16_t *__restrict__ W, int64_t n, uint8_t *__restrict__ codes,
    uint8_t *__restrict__ q8, float *__restrict__ step, const __grid_constant__ QuantTables tab,
    uint64_t limit_ns) {
  extern __shared__ __align__(128) uint8_t qsm[];
  uint8_t *ring = qsm;                                                             // [stages][32 KB]
  uint8_t *bins_bytes = qsm + kQuantStages * kQuantStageBytes;
  uint2 *bins = reinterpret_cast<uint2 *>(bins_bytes);                             // [256 entries][16 copies]
  float *rcp = reinterpret_cast<float *>(bins_bytes + kQuantBins256 * kQuantCopies * 8);   // [128]
  float *amax = rcp + 128;                                                         // [256]
  float *wmax = amax + kGroup;                                                     // [16]
  uint64_t *full = reinterpret_cast<uint64_t *>(wmax + 16);                        // [stages]
  volatile int *abort_flag = reinterpret_cast<volatile int *>(full + kQuantStages);
  const int tid = threadIdx.x, lane = tid & 31;
  const int64_t ngroups = (n + kGroupElems - 1) / kGroupElems;
  const int64_t nblocks = (n + kBlock - 1) / kBlock;
  const int64_t G = gridDim.x;
  auto whole = [&](int64_t g) { return (g + 1) * kGroupElems <= n; };

  for (int i = tid; i < kQuantBins256 * kQuantCopies; i += kQuantThreads) {
    const QuantBin e = tab.bins[i / kQuantCopies];
    bins[i] = make_uint2(__float_as_uint(e.t), static_cast<uint32_t>(e.c));
  }
  if (tid < 128) rcp[tid] = tab.rcp[tid];
  if (tid == 0) {
    *abort_flag = 0;
    for (int k = 0; k < kQuantStages; ++k) mbar_init(&full[k], 1);
    fence_mbar_init();
    for (int k = 0; k < kQuantStages; ++k) {
      const int64_t g = blockIdx.x + k * G;
      if (g < ngroups && whole(g)) {
        mbar_arrive_expect_tx(&full[k], kQuantStageBytes);
        bulk_load(ring + k * kQuantStageBytes, W + g * kGroupElems, kQuantStageBytes, &full[k]);
      }
    }
  }
  const Waiter waiter{abort_flag, limit_ns};
  const uint32_t lane8 = 8u * static_cast<uint32_t>(lane % kQuantCopies);
  const int sub = tid & 7;
  const int bl = tid >> 3;                     // block within a pass (0..63)
  bool nonfinite = false;

  int it = 0;
  for (int64_t g = blockIdx.x; g < ngroups; g += G, ++it) {
    const int s = it % kQuantStages;
    const uint32_t ph = static_cast<uint32_t>(it / kQuantStages) & 1u;
    const int64_t gbase = g * kGroupElems;
    __syncthreads();   // tables and barriers ready; the previous group's amax and wmax consumed
    uint4 v[kQuantPasses];
    if (whole(g)) {
      if (!__syncthreads_and(wait_bar(&full[s], ph, waiter))) break;
      const uint32_t src = smem_u32(ring + s * kQuantStageBytes) + static_cast<uint32_t>((bl * kBlock + sub * 8) * 2);
#pragma unroll
      for (int p = 0; p < kQuantPasses; ++p)
        v[p] = ld_shared_v4(src + static_cast<uint32_t>(p * (kGroup / kQuantPasses) * kBlock * 2));
      quant_compute<true, kQuantPasses>(v, n, gbase, bl, sub, rcp, bins_bytes, lane8, codes, amax, nonfinite);
    } else {
      quant_load_tail<kQuantPasses>(W, n, gbase, bl, sub, v);
      quant_compute<false, kQuantPasses>(v, n, gbase, bl, sub, rcp, bins_bytes, lane8, codes, amax, nonfinite);
    }
    __syncthreads();   // stage s consumed, the group's block absmaxes complete
    if (tid == 0) {
      const int64_t gn = g + kQuantStages * G;
      if (gn < ngroups && whole(gn)) {
        mbar_arrive_expect_tx(&full[s], kQuantStageBytes);
        bulk_load(ring + s * kQuantStageBytes, W + gn * kGroupElems, kQuantStageBytes, &full[s]);
      }
    }

    // second level: one constant per group (threads 0..255, one block each); with
    // single-level constants (q8 null) the block absmax itself is stored in fp32
    const int64_t b = g * kGroup + tid;
    const float a = (tid < kGroup && b < nblocks) ? amax[tid] : 0.f;
    if (q8 == nullptr) {
      if (tid < kGroup && b < nblocks) step[b] = a;
      continue;
    }
    float m = a;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0 && tid < kGroup) wmax[tid >> 5] = m;
    __syncthreads();
    if (tid < kGroup) {
      float c = wmax[0];
#pragma unroll
      for (int i = 1; i < kGroup / 32; ++i) c = fmaxf(c, wmax[i]);
      const float st = (c > 0.f) ? __fdiv_rn(c, 255.0f) : 0.f;
      if (b < nblocks) {
        int q = 0;
        if (c > 0.f) q = min(255, __float2int_rn(__fdiv_rn(a, st)));
        q8[b] = static_cast<uint8_t>(q);
      }
      if (tid == 0) step[g] = st;
    }
  }
  if (nonfinite && sub == 0) atomicOr(&g_device_status, kStatNonFinite);
}

// Standalone dequant: 16 values per thread per iteration (8 bytes of codes in,
// 32 bytes of bf16 out), grid-stride.  w = bf16_RN(RN32(L[code] * RN32(q8*step))),
// or bf16_RN(RN32(L[code] * step[b])) with single-level constants (q8 null).
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
    const float sc = q8 ? __fmul_rn(static_cast<float>(q8[b]), step[b >> 8]) : step[b];
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
      const float sc = q8 ? __fmul_rn(static_cast<float>(q8[b]), step[b >> 8]) : step[b];
      const __nv_bfloat16 h = __float2bfloat16_rn(__fmul_rn(L[code], sc));
      out[e] = *reinterpret_cast<const uint16_t *>(&h);
    }
  }
}

}  // namespace qlora
