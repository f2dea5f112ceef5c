// Rank-r contractions of the QLoRA adapter on tcgen05 ("QLoRA",
// ozercemkelahmet.com, How it works, Steps 4-6):
//   projections   XA = X A,  G = dY B^T              (rows = tokens)
//   gradients     dA = X^T (sG),  dB = dY^T (sXA)     (rows = input/output features)
// Every one is a tall-skinny product  D[rows, nn] = Act[rows, c] * Q[nn, c]^T
// with nn = r (rounded up to 16) or 2r (bf16 hi|lo halves of an fp32
// operand), so it is bound by reading the bf16 activation (X or dY) once.
//
// One CTA computes a 128-row tile over one split of the contraction.  The splits
// of a tile form a thread-block cluster (at most 8): each CTA stages its fp32
// partial tile in shared memory (reusing its operand ring, idle once the last
// MMA has committed), and rank q then sums rows [q R, (q+1) R) over the cluster
// in rank order through distributed shared memory (deterministic, no global
// scratch) and writes the final outputs in whole rows (a projection's transposed
// hi|lo halves through a shared-memory stage).  The activation side is the MMA's A operand:
//   K-major  (projections): Act = X / dY tile [128 tokens x 64 c], TMA box {64, 128}
//   MN-major (gradients):   Act^T tile [128 features x 64 tokens] from X / dY
//                           [tokens, features]: two TMA boxes {64 features, 64 tokens}
// Q is always K-major [nn rows x 64 c], TMA box {64, nn}.
// A ring slot holds `sub` such 64-wide steps under one barrier (the projections take
// two, so each activation row is read 256 contiguous bytes at a time).
// dA and dB contract over the same tokens, so one launch computes both: the row tiles
// of the second follow those of the first on the grid.
// Warps: 0 TMA producer, 1 TMEM allocator + MMA issuer, 4..7 epilogue.
#pragma once
#include "common.cuh"

namespace qlora {

constexpr int kLmThreads = 256;
constexpr int kLmRows = 128;
constexpr int kLmABytes = kLmRows * 128;   // 16 KB per stage

struct LoraMmaParams {
  int rows;              // output rows (tokens for projections, features for gradients)
  int nn;                // MMA N: multiple of 16, <= 256
  int stages_total;      // contraction steps of 64
  int stages_per_split;  // steps of 64 per split
  int num_stages;        // smem ring depth
  int sub;               // steps of 64 per ring slot (one wait, one expect_tx, sub TMA boxes)
  uint32_t tmem_cols;    // power of two >= max(32, nn)
  int splits;            // cluster size along the contraction
  int grad;              // 0: projection outputs, 1: gradient outputs
  int r;
  float s;
  // projection: out [rows, r] fp32, hl [rows, 2r] and/or hlT [2r, ldT] bf16 hi|lo of s*out
  // gradient:   out = sum of the hi and lo halves; layout 0 out[row][j], 1 out[j][row]
  float *out;
  uint16_t *hl;
  uint16_t *hlT;
  int ldT;
  int layout;
  uint64_t limit_ns;
  // A second gradient product in the same launch: row tiles [tiles0, gridDim.x) compute
  // it from the second pair of tensor maps.  It shares the contraction, nn and the
  // splits; it has its own rows, output and layout.  tiles0 = gridDim.x: none.
  int tiles0;
  int rows1;
  float *out1;
  int layout1;
  // Words that a later kernel of the same call expects to find zero (the fused GEMM's
  // split-tile arrival counters); CTA (0, 0) clears them.  May be null.
  unsigned int *zero;
  int zero_n;
  // Factor applied to the fp32 result before it is stored (1/(1-p) for products over
  // the dropped-out adapter input), for the first and the second product.
  float out_scale, out_scale1;
  int accumulate;        // gradients: add into out instead of overwriting it
};

constexpr int kLmClusterMax = 8;   // portable cluster size: at most 8 splits of a tile

// Row pitch (floats) of the fp32 partial tile staged for the cluster reduction: odd, so
// that both a warp over 32 rows of one column and a warp along one row hit 32 distinct
// shared-memory banks.
constexpr __host__ __device__ int lm_partial_pitch(int nn) { return nn + 1; }
constexpr __host__ __device__ int lm_partial_bytes(int nn) { return kLmRows * lm_partial_pitch(nn) * 4; }
// Shared memory the projection epilogue needs after the main loop: the partial tile and
// the stage of the transposed hi|lo halves (2r <= 2 nn rows of at most 128 + 2 values).
constexpr __host__ __device__ int lm_epilogue_bytes(int nn) { return lm_partial_bytes(nn) + 2 * nn * (kLmRows + 2) * 2; }

constexpr int kLmSmemMax = 200 * 1024;   // the kernels' dynamic shared-memory attribute

constexpr int lora_mma_smem_bytes(int nn, int stages, int sub) {
  return 1024 + stages * sub * (kLmABytes + nn * 128) + 256;
}

QDEV void split_hilo(float v, uint16_t &hi, uint16_t &lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
  hi = *reinterpret_cast<const uint16_t *>(&h);
  lo = *reinterpret_cast<const uint16_t *>(&l);
}

template <bool A_MN>
__global__ void __launch_bounds__(kLmThreads, 1)
    lora_mma_kernel(const __grid_constant__ CUtensorMap tm_act, const __grid_constant__ CUtensorMap tm_q,
                    const __grid_constant__ CUtensorMap tm_act1, const __grid_constant__ CUtensorMap tm_q1,
                    const __grid_constant__ LoraMmaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int S = p.num_stages;
  const int b_bytes = p.nn * 128;
  const int a_slot = p.sub * kLmABytes, b_slot = p.sub * b_bytes;
  uint8_t *sA = smem;
  uint8_t *sB = sA + S * a_slot;
  uint64_t *full = reinterpret_cast<uint64_t *>(sB + S * b_slot);
  uint64_t *empty = full + S;
  uint64_t *done = empty + S;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(done + 1);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (p.zero && blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = tid; i < p.zero_n; i += kLmThreads) p.zero[i] = 0u;
  const bool second = static_cast<int>(blockIdx.x) >= p.tiles0;
  const int row0 = (static_cast<int>(blockIdx.x) - (second ? p.tiles0 : 0)) * kLmRows;
  const int rows = second ? p.rows1 : p.rows;
  float *const out = second ? p.out1 : p.out;
  const int layout = second ? p.layout1 : p.layout;
  const float out_scale = second ? p.out_scale1 : p.out_scale;
  const CUtensorMap *const map_act = second ? &tm_act1 : &tm_act;
  const CUtensorMap *const map_q = second ? &tm_q1 : &tm_q;
  const int split = blockIdx.y;
  const int st0 = split * p.stages_per_split;
  const int st1 = min(p.stages_total, st0 + p.stages_per_split);
  const int nst = st1 - st0;
  const int nslot = (nst + p.sub - 1) / p.sub;   // ring slots this split fills

  if (tid == 0) {
    for (int i = 0; i < S; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Waiter wt{abort_flag, p.limit_ns};

  if (warp == 0 && lane == 0) {
    prefetch_tmap(map_act);
    prefetch_tmap(map_q);
    uint32_t armed = 0, last = 0;
    int s = 0;
    uint32_t ph = 0;
    for (int i = 0; i < nslot; ++i) {
      if (!wait_bar(&empty[s], ph ^ 1u, wt)) break;
      const int k0 = st0 + i * p.sub;
      const int ns = min(p.sub, st1 - k0);
      mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(ns * (kLmABytes + b_bytes)));
      for (int j = 0; j < ns; ++j) {
        const int c0 = (k0 + j) * 64;
        uint8_t *da = sA + s * a_slot + j * kLmABytes;
        if (A_MN) {
          tma_load_2d(da, map_act, &full[s], row0, c0);
          tma_load_2d(da + 8192, map_act, &full[s], row0 + 64, c0);
        } else {
          tma_load_2d(da, map_act, &full[s], c0, row0);
        }
        tma_load_2d(sB + s * b_slot + j * b_bytes, map_q, &full[s], c0, 0);
      }
      armed |= 1u << s;
      last = (last & ~(1u << s)) | (ph << s);
      if (++s == S) { s = 0; ph ^= 1u; }
    }
    volatile int no_abort = 0;
    const Waiter fw{&no_abort, p.limit_ns};
    for (int k = 0; k < S; ++k)
      if (armed & (1u << k)) wait_bar(&full[k], (last >> k) & 1u, fw);
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = make_idesc_bf16(kLmRows, p.nn, A_MN, false);
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int i = 0; i < nslot; ++i) {
      if (!wait_bar(&full[s], ph, wt)) { ok = false; break; }
      tc_fence_after();
      const int ns = min(p.sub, st1 - (st0 + i * p.sub));
      for (int j = 0; j < ns; ++j) {
        const uint32_t a = smem_u32(sA + s * a_slot + j * kLmABytes);
        const uint32_t b = smem_u32(sB + s * b_slot + j * b_bytes);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t ad = A_MN ? sw128_desc(a + k * 2048, 8192, 1024) : sw128_desc(a + k * 32, 16, 1024);
          const uint64_t bd = sw128_desc(b + k * 32, 16, 1024);
          mma_bf16_ss(tmem_base, ad, bd, idesc, (i > 0 || j > 0 || k > 0) ? 1u : 0u);
        }
      }
      mma_commit(&empty[s]);
      if (++s == S) { s = 0; ph ^= 1u; }
    }
    (void)ok;
    mma_commit(done);   // also drains every issued MMA before TMEM is released
  } else if (warp >= 4) {
    // TMEM -> this CTA's partial tile in shared memory (the operand ring is idle now)
    const int q = warp & 3;
    const int rl = q * 32 + lane;
    volatile int no_abort = 0;
    const Waiter dw{&no_abort, p.limit_ns};
    const bool got = __all_sync(0xffffffffu, wait_bar(done, 0, dw) ? 1 : 0);
    tc_fence_after();
    const int pitch = lm_partial_pitch(p.nn);
    float *dst = reinterpret_cast<float *>(smem) + rl * pitch;
    for (int c = 0; c < p.nn; c += 16) {
      uint32_t v[16];
      asm volatile(
          "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
          "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
          : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
            "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
            "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
          : "r"(tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(c)));
      tmem_wait_ld();
      const bool keep = got && nst > 0;
#pragma unroll
      for (int j = 0; j < 16; ++j) dst[c + j] = keep ? __uint_as_float(v[j]) : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }

  // ---- cluster reduction: rank q finishes rows [q R, (q+1) R) of the tile
  cluster_sync_all();
  {
    const int rank = static_cast<int>(cluster_ctarank());
    const int R = (kLmRows + p.splits - 1) / p.splits;
    const int r0 = rank * R, r1 = min(kLmRows, r0 + R);
    const int nr = max(0, r1 - r0);
    const uint32_t base = smem_u32(smem);
    const int pitch = lm_partial_pitch(p.nn);
    if (p.grad) {
      for (int i = tid; i < nr * p.r; i += kLmThreads) {
        int rr, j;
        if (layout == 0) { rr = i / p.r; j = i - rr * p.r; }     // j fastest: out[row][j]
        else { j = i / nr; rr = i - j * nr; }                     // row fastest: out[j][row]
        const int rl = r0 + rr, row = row0 + rl;
        if (row >= rows) continue;
        const uint32_t a = base + 4u * static_cast<uint32_t>(rl * pitch + j);
        const uint32_t b = a + 4u * static_cast<uint32_t>(p.r);
        // every rank's load is issued before the sum, which runs in rank order
        float pa[kLmClusterMax], pb[kLmClusterMax];
#pragma unroll
        for (int qq = 0; qq < kLmClusterMax; ++qq) {
          pa[qq] = qq < p.splits ? ld_dsmem_f32(map_rank(a, static_cast<uint32_t>(qq))) : 0.f;
          pb[qq] = qq < p.splits ? ld_dsmem_f32(map_rank(b, static_cast<uint32_t>(qq))) : 0.f;
        }
        float v = 0.f;
#pragma unroll
        for (int qq = 0; qq < kLmClusterMax; ++qq)
          if (qq < p.splits) v += pa[qq] + pb[qq];
        v = __fmul_rn(v, out_scale);
        float *o = (layout == 0) ? out + static_cast<int64_t>(row) * p.r + j : out + static_cast<int64_t>(j) * rows + row;
        *o = p.accumulate ? __fadd_rn(*o, v) : v;
      }
    } else {
      // Projection: j fastest, so the fp32 result and the row-major hi|lo halves go out
      // in whole rows; the transposed halves are staged in shared memory ([2r][nr],
      // after this CTA's own partial tile, which the peers may still be reading) and
      // written row by row once the rank's rows are done.
      uint16_t *stT = reinterpret_cast<uint16_t *>(smem + lm_partial_bytes(p.nn));
      const int tp = nr + 2;   // odd word pitch: a warp's stores along j hit distinct banks
      const int total = nr * p.r;
      for (int i0 = tid; i0 < total; i0 += 2 * kLmThreads) {
        // two elements per pass: all their loads are issued before either sum
        float pa[2][kLmClusterMax];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i = i0 + u * kLmThreads;
          const int rr = i / p.r, j = i - rr * p.r;
          const uint32_t a = base + 4u * static_cast<uint32_t>((r0 + rr) * pitch + j);
#pragma unroll
          for (int qq = 0; qq < kLmClusterMax; ++qq)
            pa[u][qq] = (i < total && qq < p.splits) ? ld_dsmem_f32(map_rank(a, static_cast<uint32_t>(qq))) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int i = i0 + u * kLmThreads;
          if (i >= total) continue;
          const int rr = i / p.r, j = i - rr * p.r;
          const int row = row0 + r0 + rr;
          if (row >= rows) continue;
          float v = 0.f;
#pragma unroll
          for (int qq = 0; qq < kLmClusterMax; ++qq)
            if (qq < p.splits) v += pa[u][qq];
          v = __fmul_rn(v, out_scale);
          if (out) out[static_cast<int64_t>(row) * p.r + j] = v;
          uint16_t h, l;
          split_hilo(p.s * v, h, l);
          if (p.hl) {
            p.hl[static_cast<int64_t>(row) * 2 * p.r + j] = h;
            p.hl[static_cast<int64_t>(row) * 2 * p.r + p.r + j] = l;
          }
          if (p.hlT) {
            stT[j * tp + rr] = h;
            stT[(p.r + j) * tp + rr] = l;
          }
        }
      }
      if (p.hlT) {
        __syncthreads();
        for (int i = tid; i < 2 * p.r * nr; i += kLmThreads) {
          const int jj = i / nr, rr = i - jj * nr;
          const int row = row0 + r0 + rr;
          if (row < rows) p.hlT[static_cast<int64_t>(jj) * p.ldT + row] = stT[jj * tp + rr];
        }
      }
    }
  }
  cluster_sync_all();   // no CTA leaves while a peer may still read its partial tile
}

// ---------------------------------------------------------------- helpers around it
// AT[j][k] = A[k][j]: the adapter A [K, r] as the K-major operand [r, K].
__global__ void __launch_bounds__(256) transpose_bf16_kernel(const uint16_t *__restrict__ A, int K,
                                                             int r, uint16_t *__restrict__ AT) {
  const int64_t total = static_cast<int64_t>(K) * r;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t j = i / K, k = i - j * K;
    AT[i] = A[k * r + j];
  }
}

// Xd = X (.) keep: the adapter input with its dropped elements set to zero (exact in
// bf16).  keep is a bit-packed mask of the n = M K elements, element e in bit e mod 8
// of byte e / 8; n is a multiple of 8.  Eight elements (16 bytes) per thread and step.
__global__ void __launch_bounds__(256) mask_input_kernel(const uint16_t *__restrict__ X,
                                                         const uint8_t *__restrict__ keep, int64_t n8,
                                                         uint16_t *__restrict__ Xd) {
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; u < n8;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 x = ld_global_nc_v4(X + 8 * u);
    const uint32_t b = keep[u];
    // bit 2i keeps the low half of word i, bit 2i+1 the high half
    auto m = [b](uint32_t w, int i) {
      const uint32_t lo = ((b >> (2 * i)) & 1u) ? 0x0000FFFFu : 0u;
      const uint32_t hi = ((b >> (2 * i + 1)) & 1u) ? 0xFFFF0000u : 0u;
      return w & (lo | hi);
    };
    *reinterpret_cast<uint4 *>(Xd + 8 * u) = make_uint4(m(x.x, 0), m(x.y, 1), m(x.z, 2), m(x.w, 3));
  }
}

// hlT [2r, ldT] = hi/lo of s*v for an fp32 v [M, r] (the saved XA in the backward).
__global__ void __launch_bounds__(256) hilo_t_kernel(const float *__restrict__ v, int M, int r, float s,
                                                     uint16_t *__restrict__ hlT, int ldT) {
  const int64_t total = static_cast<int64_t>(M) * r;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(i / M);
    const int m = static_cast<int>(i - static_cast<int64_t>(j) * M);
    uint16_t h, l;
    split_hilo(s * v[static_cast<int64_t>(m) * r + j], h, l);
    hlT[static_cast<int64_t>(j) * ldT + m] = h;
    hlT[static_cast<int64_t>(r + j) * ldT + m] = l;
  }
}

}  // namespace qlora
