// The adapter folded into a 16-bit weight for serving ("QLoRA",
// ozercemkelahmet.com, How it works, Step 8 and section "Merging after QLoRA"):
//   out[n][k] = bf16_RN( base[n][k] + s * sum_j B[j][n] A[k][j] )
// with base the bf16 original W16 [N, K], or the dequantized NF4 weight
// bf16(RN32(L[c] RN32(q8 step))) (the same element as the standalone dequant).
//
// (A B)^T is a dense contraction over r into every weight element, so it runs on
// tcgen05.  One CTA computes a 128 (n) x 256 (k) tile:
//   MMA A = B^T tile, MN-major from B [r, N]: two TMA boxes {64 n, 64 j};
//   MMA B = A tile, K-major from A [K, r]: one TMA box {64 j, 256 k}.
// Rows j >= r of either box lie outside the tensor and are zero-filled by TMA,
// so one stage covers r <= 64 and two cover r <= 128.  The accumulator is 256
// TMEM columns.  Epilogue warps 4..7 own one row n each: they read 16 columns at
// a time from TMEM, form the base (16 bf16 of W16, or 8 code bytes and the block
// constant), add s * acc with one fp32 FMA, round to bf16 and store 32 bytes.
// Warps: 0 TMA producer, 1 TMEM allocator + MMA issuer, 4..7 epilogue.
#pragma once
#include "common.cuh"

namespace qlora {

constexpr int kMgThreads = 256;
constexpr int kMgRows = 128;                   // n per tile
constexpr int kMgCols = 256;                   // k per tile (MMA N)
constexpr int kMgABytes = kMgRows * 128;       // B^T tile: 128 n x 64 j bf16
constexpr int kMgBBytes = kMgCols * 128;       // A tile: 256 k x 64 j bf16

struct MergeParams {
  const uint8_t *codes;   // NF4 base (when w16 is null): packed codes, q8, step
  const uint8_t *q8;      // null: single-level constants (step[block] = absmax)
  const float *step;
  const uint16_t *w16;    // bf16 base [N, K], or null
  uint16_t *out;          // bf16 [N, K]
  int N, K;
  int stages;             // ceil(r / 64)
  float s;
  float levels[16];
  uint64_t limit_ns;
};

// At least 80 KB, so at most two CTAs share an SM and their 256 TMEM columns each
// always fit in the SM's 512.
inline int merge_smem_bytes(int stages) {
  const int b = 1024 + stages * (kMgABytes + kMgBBytes) + 128;
  return b < 80 * 1024 ? 80 * 1024 : b;
}

__global__ void __launch_bounds__(kMgThreads, 1)
    nf4_merge_kernel(const __grid_constant__ CUtensorMap tm_bt, const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ MergeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sA = smem;
  uint8_t *sB = sA + p.stages * kMgABytes;
  uint64_t *full = reinterpret_cast<uint64_t *>(sB + p.stages * kMgBBytes);
  uint64_t *done = full + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k0 = blockIdx.x * kMgCols;
  const int n0 = blockIdx.y * kMgRows;

  if (tid == 0) {
    for (int i = 0; i < p.stages; ++i) mbar_init(&full[i], 1);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kMgCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Waiter wt{abort_flag, p.limit_ns};

  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_bt);
    prefetch_tmap(&tm_a);
    for (int st = 0; st < p.stages; ++st) {
      mbar_arrive_expect_tx(&full[st], kMgABytes + kMgBBytes);
      tma_load_2d(sA + st * kMgABytes, &tm_bt, &full[st], n0, st * 64);
      tma_load_2d(sA + st * kMgABytes + 8192, &tm_bt, &full[st], n0 + 64, st * 64);
      tma_load_2d(sB + st * kMgBBytes, &tm_a, &full[st], st * 64, k0);
    }
    // no copy may still be in flight when the block exits
    volatile int no_abort = 0;
    const Waiter fw{&no_abort, p.limit_ns};
    for (int st = 0; st < p.stages; ++st) wait_bar(&full[st], 0, fw);
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = make_idesc_bf16(kMgRows, kMgCols, true, false);
    for (int st = 0; st < p.stages; ++st) {
      if (!wait_bar(&full[st], 0, wt)) break;
      tc_fence_after();
      const uint32_t a = smem_u32(sA + st * kMgABytes);
      const uint32_t b = smem_u32(sB + st * kMgBBytes);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_bf16_ss(tmem_base, sw128_desc(a + kk * 2048, 8192, 1024), sw128_desc(b + kk * 32, 16, 1024), idesc,
                    (st > 0 || kk > 0) ? 1u : 0u);
    }
    mma_commit(done);   // also drains every issued MMA before TMEM is released
  } else if (warp >= 4) {
    const int q = warp & 3;
    const int n = n0 + q * 32 + lane;
    volatile int no_abort = 0;
    const Waiter dw{&no_abort, p.limit_ns};
    const bool got = __all_sync(0xffffffffu, wait_bar(done, 0, dw) ? 1 : 0) && *abort_flag == 0;
    tc_fence_after();
    float L[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) L[i] = p.levels[i];
    for (int c = 0; c < kMgCols / 16; ++c) {
      uint32_t v[16];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
          "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
            "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
            "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
          : "r"(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(c * 16)));
      tmem_wait_ld();
      const int col = k0 + c * 16;
      if (!got || n >= p.N || col >= p.K) continue;
      const int64_t e0 = static_cast<int64_t>(n) * p.K + col;    // first element, a multiple of 16
      float base[16];
      if (p.w16) {
        const uint4 w0 = *reinterpret_cast<const uint4 *>(p.w16 + e0);
        const uint4 w1 = *reinterpret_cast<const uint4 *>(p.w16 + e0 + 8);
        const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          base[2 * i] = bf16_lo(w[i]);
          base[2 * i + 1] = bf16_hi(w[i]);
        }
      } else {
        // the block's 16 dequantized values as a register table (the same
        // bf16(RN32(L[c] RN32(q8 step))) elements as the standalone dequant)
        const uint2 cw = *reinterpret_cast<const uint2 *>(p.codes + (e0 >> 1));
        const int64_t blk = e0 >> 6;
        Nf4Lut t;
        const float sc = p.q8 ? __fmul_rn(static_cast<float>(p.q8[blk]), p.step[blk >> 8]) : p.step[blk];
        nf4_build_lut(L, sc, t);
        uint32_t d0[4], d1[4];
        nf4_decode8(cw.x, t, d0);
        nf4_decode8(cw.y, t, d1);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          base[2 * i] = bf16_lo(d0[i]);
          base[2 * i + 1] = bf16_hi(d0[i]);
          base[8 + 2 * i] = bf16_lo(d1[i]);
          base[8 + 2 * i + 1] = bf16_hi(d1[i]);
        }
      }
      uint32_t o[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        o[i] = pack_bf16x2(__fmaf_rn(p.s, __uint_as_float(v[2 * i]), base[2 * i]),
                           __fmaf_rn(p.s, __uint_as_float(v[2 * i + 1]), base[2 * i + 1]));
      *reinterpret_cast<uint4 *>(p.out + e0) = make_uint4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<uint4 *>(p.out + e0 + 8) = make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kMgCols);
  }
}

}  // namespace qlora
