// The adapter folded into a 16-bit weight for serving ("QLoRA",
// ozercemkelahmet.com, How it works, Step 8 and section "Merging after QLoRA"):
//   out[n][k] = bf16_RN( base[n][k] + s * sum_j B[j][n] A[k][j] )
// with base the bf16 original W16 [N, K], or the dequantized NF4 weight
// bf16(RN32(L[c] RN32(q8 step))) (the same element as the standalone dequant).
//
// (A B)^T is a dense contraction over r into every weight element, so it runs on
// tcgen05; the rest is a stream of the base in and the merged weight out, which
// moves by TMA.  One CTA computes a 128 (n) x 256 (k) tile:
//   MMA A = B^T tile, MN-major from B [r, N]: two TMA boxes {64 n, 64 j};
//   MMA B = A tile, K-major from A [K, r]: one TMA box {64 j, 256 k}.
// Rows j >= r of either box lie outside the tensor and are zero-filled by TMA,
// so one stage covers r <= 64 and two cover r <= 128.  The accumulator is 256
// TMEM columns.  The base tile is requested at once beside the operands: four
// 128B-swizzled boxes {64 k, 128 n} of W16, or one box {128 bytes, 128 n} of
// packed codes.  Each epilogue thread owns one row n and half the columns: it reads 16 at a
// time from TMEM, take the base from shared memory (16 bf16, or 8 code bytes
// decoded through the block's table, one table per 64 values), add s * acc with one
// fp32 FMA, round to bf16 and write the result into the output tile in shared
// memory (in place of the bf16 base; in the operand buffers, free once the MMAs are
// done, for the NF4 base), which one thread then stores by TMA.
// Warps: 0 TMA producer, 1 TMEM allocator + MMA issuer, then all eight the epilogue.
#pragma once
#include "common.cuh"

namespace qlora {

constexpr int kMgThreads = 256;
constexpr int kMgRows = 128;                   // n per tile
constexpr int kMgCols = 256;                   // k per tile (MMA N)
constexpr int kMgABytes = kMgRows * 128;       // B^T tile: 128 n x 64 j bf16
constexpr int kMgBBytes = kMgCols * 128;       // A tile: 256 k x 64 j bf16
constexpr int kMgBoxBytes = kMgRows * 128;     // one output / bf16 base box: 128 n x 64 k
constexpr int kMgCodeBytes = kMgRows * 128;    // packed codes of a tile: 128 n x 256 k

struct MergeParams {
  const uint8_t *q8;      // NF4 base (codes by tensor map): null for single-level constants
  const float *step;
  int nf4;                // 1: NF4 base (codes map), 0: bf16 base (W16 map)
  int N, K;
  int stages;             // ceil(r / 64)
  float s;
  float levels[16];
  uint64_t limit_ns;
};

// Shared memory: the operand stages, then (bf16 base) the base tile that becomes the
// output tile, or (NF4 base) the codes tile plus one output box beyond the three
// that fit in a single operand stage.
__host__ __device__ inline int merge_base_bytes(int stages, bool nf4) {
  if (!nf4) return 4 * kMgBoxBytes;
  const int ops = stages * (kMgABytes + kMgBBytes);
  return kMgCodeBytes + (ops >= 4 * kMgBoxBytes ? 0 : 4 * kMgBoxBytes - ops);
}
// At least 80 KB, so at most two CTAs share an SM and their 256 TMEM columns each
// always fit in the SM's 512.  The dynamic shared memory is declared 1024-byte
// aligned and no slack is reserved for aligning it (the bf16-base plan then fits two
// CTAs per SM; with slack it missed by 256 bytes); the kernel checks the alignment.
inline int merge_smem_bytes(int stages, bool nf4) {
  const int b = stages * (kMgABytes + kMgBBytes) + merge_base_bytes(stages, nf4) + 128;
  return b < 80 * 1024 ? 80 * 1024 : b;
}
inline int merge_smem_max() {
  const int a = merge_smem_bytes(2, false), b = merge_smem_bytes(2, true);
  return a > b ? a : b;
}

QDEV void tma_store_2d(const CUtensorMap *map, const void *src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}

__global__ void __launch_bounds__(kMgThreads, 1)
    nf4_merge_kernel(const __grid_constant__ CUtensorMap tm_bt, const __grid_constant__ CUtensorMap tm_a,
                     const __grid_constant__ CUtensorMap tm_base, const __grid_constant__ CUtensorMap tm_out,
                     const __grid_constant__ MergeParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // the 128B-swizzled boxes need 1024-byte alignment, which the declaration asks for
  // and the plan counts on: a misplaced buffer is reported and nothing is touched
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) atomicOr(&g_device_status, kStatLayout);
    return;
  }
  uint8_t *smem = smem_raw;
  const int ops_bytes = p.stages * (kMgABytes + kMgBBytes);
  uint8_t *sA = smem;
  uint8_t *sB = sA + p.stages * kMgABytes;
  uint8_t *sBase = smem + ops_bytes;                 // W16 boxes, or the codes tile
  uint64_t *full = reinterpret_cast<uint64_t *>(sBase + merge_base_bytes(p.stages, p.nf4 != 0));
  uint64_t *done = full + 2;
  uint64_t *base_full = done + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(base_full + 1);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  // output box i: in place of the bf16 base; for the NF4 base, in the operand buffers
  // (boxes 0..2, or all four with two stages) and after the codes tile
  auto out_box = [&](int i) -> uint8_t * {
    if (!p.nf4) return sBase + i * kMgBoxBytes;
    return (i * kMgBoxBytes < ops_bytes) ? smem + i * kMgBoxBytes : sBase + kMgCodeBytes + (i * kMgBoxBytes - ops_bytes);
  };

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k0 = blockIdx.x * kMgCols;
  const int n0 = blockIdx.y * kMgRows;
  const int nbox = min(4, (p.K - k0) / 64);          // 64-column boxes inside the tensor

  if (tid == 0) {
    for (int i = 0; i < p.stages; ++i) mbar_init(&full[i], 1);
    mbar_init(done, 1);
    mbar_init(base_full, 1);
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
    prefetch_tmap(&tm_base);
    prefetch_tmap(&tm_out);
    for (int st = 0; st < p.stages; ++st) {
      mbar_arrive_expect_tx(&full[st], kMgABytes + kMgBBytes);
      tma_load_2d(sA + st * kMgABytes, &tm_bt, &full[st], n0, st * 64);
      tma_load_2d(sA + st * kMgABytes + 8192, &tm_bt, &full[st], n0 + 64, st * 64);
      tma_load_2d(sB + st * kMgBBytes, &tm_a, &full[st], st * 64, k0);
    }
    if (p.nf4) {
      mbar_arrive_expect_tx(base_full, kMgCodeBytes);
      tma_load_2d(sBase, &tm_base, base_full, k0 / 2, n0);
    } else {
      mbar_arrive_expect_tx(base_full, 4 * kMgBoxBytes);
      for (int i = 0; i < 4; ++i) tma_load_2d(sBase + i * kMgBoxBytes, &tm_base, base_full, k0 + 64 * i, n0);
    }
    // no copy may still be in flight when the block exits
    volatile int no_abort = 0;
    const Waiter fw{&no_abort, p.limit_ns};
    for (int st = 0; st < p.stages; ++st) wait_bar(&full[st], 0, fw);
    wait_bar(base_full, 0, fw);
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
  }
  __syncwarp();
  {
    // epilogue: all eight warps, warps 4..7 on columns 0..127 and warps 0..3 (their
    // producer and MMA lanes done) on columns 128..255; TMEM lane quadrant warp & 3
    const int q = warp & 3;
    const int c_begin = (warp >= 4) ? 0 : kMgCols / 32, c_end = c_begin + kMgCols / 32;
    const int row = q * 32 + lane;                   // row within the tile (TMEM lane)
    const int n = n0 + row;
    const uint32_t sw = static_cast<uint32_t>(row & 7);   // 128B swizzle of this row
    // the row's block constants, requested before any wait
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
    if (p.nf4 && n < p.N) {
      const int64_t b0 = static_cast<int64_t>(n) * (p.K / 64) + k0 / 64;
#pragma unroll
      for (int b = 0; b < 4; ++b)
        if (b < nbox) sc[b] = p.q8 ? __fmul_rn(static_cast<float>(__ldg(p.q8 + b0 + b)), __ldg(p.step + ((b0 + b) >> 8)))
                                   : __ldg(p.step + b0 + b);
    }
    float L[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) L[i] = p.levels[i];
    volatile int no_abort = 0;
    const Waiter dw{&no_abort, p.limit_ns};
    const bool got = __all_sync(0xffffffffu, (wait_bar(done, 0, dw) && wait_bar(base_full, 0, dw)) ? 1 : 0) &&
                     *abort_flag == 0;
    tc_fence_after();
    Nf4Lut t{};
    for (int c = c_begin; c < c_end; ++c) {
      uint32_t v[16];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
          "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
            "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
            "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
          : "r"(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(c * 16)));
      tmem_wait_ld();
      const int box = c >> 2;                         // 64-column box of these 16 columns
      if (!got || box >= nbox) continue;
      // the 16 columns are 16-byte chunks 2 (c & 3) and 2 (c & 3) + 1 of the row in its box
      const uint32_t j0 = static_cast<uint32_t>(2 * (c & 3));
      uint8_t *ob = out_box(box) + row * 128;
      const uint32_t o0 = smem_u32(ob) + (((j0) ^ sw) << 4), o1 = smem_u32(ob) + (((j0 + 1) ^ sw) << 4);
      float base[16];
      if (!p.nf4) {
        const uint4 w0 = ld_shared_v4(o0);
        const uint4 w1 = ld_shared_v4(o1);
        const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          base[2 * i] = bf16_lo(w[i]);
          base[2 * i + 1] = bf16_hi(w[i]);
        }
      } else {
        // the block's 16 dequantized values as a register table (the same
        // bf16(RN32(L[c] RN32(q8 step))) elements as the standalone dequant), built
        // once per 64 values; codes of columns 16c .. 16c+15: 8 bytes of the row
        if ((c & 3) == 0) {
          const float scb = box == 0 ? sc[0] : box == 1 ? sc[1] : box == 2 ? sc[2] : sc[3];
          nf4_build_lut(L, scb, t);
        }
        const uint32_t byte0 = static_cast<uint32_t>(8 * c);   // within the row's 128 bytes
        const uint32_t ca = smem_u32(sBase + row * 128) + (((byte0 >> 4) ^ sw) << 4) + (byte0 & 15u);
        const uint2 cw = ld_shared_v2(ca);
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
      st_shared_v4(o0, o[0], o[1], o[2], o[3]);
      st_shared_v4(o1, o[4], o[5], o[6], o[7]);
    }
    // the tile's writes become visible to the TMA engine, then one thread stores it
    // (rows past N are clipped by the tensor map)
    fence_proxy_async_smem();
    asm volatile("bar.sync 1, 256;" ::: "memory");
    if (warp == 4 && lane == 0 && got) {
      for (int i = 0; i < nbox; ++i) tma_store_2d(&tm_out, out_box(i), k0 + 64 * i, n0);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      // the shared-memory source stays valid until the copies have read it
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
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
