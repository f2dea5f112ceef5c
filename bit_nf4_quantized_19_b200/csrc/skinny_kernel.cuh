// Few-token forward (M <= 16 tokens) of the QLoRA linear layer:
//     Y = X deq(W)^T + s (X A) B       ("QLoRA", ozercemkelahmet.com, How it works, Step 5)
// The work is bound by reading the packed 4-bit weight from HBM (0.52 bytes per
// weight) and by the instructions that decode it, so the design keeps every
// other cost off that path.  Two launches:
//   * qlora_xa_kernel: XA = X A (fp32 [M, r]) by one cluster of 8 CTAs, K split
//     across the cluster and reduced through distributed shared memory in rank
//     order.  It lets its dependent launch start at once;
//   * qlora_skinny_kernel, launched as that dependent (programmatic dependent
//     launch): everything it reads before its grid-dependency wait was written
//     by kernels that finished before the XA kernel started, and it reads XA only
//     after the wait, so the rank-r product runs beside it at no cost to it:
//     - each CTA owns 128 weight rows and one slice of K; the C CTAs of one
//       weight tile form a thread-block cluster along K and push their fp32
//       partial results into the shared memory of the rank that finishes those
//       rows, which sums them in rank order (deterministic, no global scratch);
//     - the code slice arrives by TMA, one 128-row x 128-byte box (128B
//       swizzle) per 256-value macro-block, each on its own mbarrier, so a warp
//       starts on macro-block mb as soon as that box has landed; this rank's
//       columns of B arrive by TMA too; the block constants are prefetched by
//       each lane into registers a few macro-blocks ahead; only the M real token
//       rows of X are staged (the fragments of absent tokens are zero registers);
//     - the NF4 codes are decoded in registers straight into the A-fragment
//       layout of mma.sync m16n8k16 (weight rows on M, tokens on N).  The
//       contraction index is permuted inside each macro-block so that the four
//       lanes sharing a fragment row each hold one whole 64-value block: lane c
//       of a row group takes block 4*mb + c, elements 4s..4s+3 at k-step s.  The
//       16-entry table bf16_RN(RN32(L[c] * RN32(q8 * step))) (the per-element
//       definition of the dequantized weight) is then built once per 64 decoded
//       values instead of once per 16.  X is read with the same permutation, so
//       the sum is the plain dot product over K taken in another order;
//     - the LoRA term s * XA B is added in fp32 when the owner finishes a row.
#pragma once
#include "common.cuh"

namespace qlora {

constexpr int kSkThreads = 256;
constexpr int kSkRows = 128;       // weight rows per CTA: 8 warps x 16
constexpr int kSkMaxCluster = 16;
constexpr int kSkMacro = 256;      // contraction values per macro-block (4 blocks of 64)
constexpr int kSkBoxBytes = kSkRows * (kSkMacro / 2);   // one macro-block of codes: 16 KB
constexpr int kSkPre = 4;          // macro-blocks of block constants prefetched ahead

struct SkinnyParams {
  const uint16_t *X;      // [M, K] bf16
  const uint8_t *codes;   // packed NF4 of W [N, K]
  const uint8_t *q8;      // null: single-level constants, step[block] = the block absmax
  const float *step;
  const uint16_t *B;      // [r, N] bf16
  const float *xa;        // [M, r] fp32, written by qlora_xa_kernel
  uint16_t *Y;            // [M, N] bf16
  int M, K, N, r;
  int ks;                 // K per cluster rank, a multiple of 256
  int xpitch;             // X row pitch, bf16 elements; element k sits at k + 4 (k / 64)
  int off_b, off_x, off_part, off_xa, off_bar;   // byte offsets from the 1024-aligned base
  uint64_t limit_ns;      // limit of every mbarrier wait
  float s;
  float levels[16];
};

// Two transposed 8x8 bf16 tiles: lanes 0-7 address the rows of the first, 8-15
// of the second; lane 4g+c receives rows 2c, 2c+1 of column g of each.
QDEV void ldmatrix_x2_trans(uint32_t addr, uint32_t &b0, uint32_t &b1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(b0), "=r"(b1)
               : "r"(addr));
}
QDEV void mma_16816_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared-memory X offset (elements) of contraction index k within the slice.
QDEV int sk_xoff(int k) { return k + 4 * (k >> 6); }

template <int C>
__global__ void __launch_bounds__(kSkThreads, 3) qlora_skinny_kernel(
    const __grid_constant__ CUtensorMap tm_codes, const __grid_constant__ CUtensorMap tm_b,
    const __grid_constant__ SkinnyParams p) {
  extern __shared__ __align__(16) uint8_t sk_raw[];
  uint8_t *sm = sk_raw + ((1024u - (smem_u32(sk_raw) & 1023u)) & 1023u);   // SW128 boxes need 1024 B
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const uint32_t rank = (C > 1) ? cluster_ctarank() : 0u;
  const int k0 = min(p.K, static_cast<int>(rank) * p.ks);   // trailing ranks may get an empty slice
  const int k1 = min(p.K, k0 + p.ks);
  const int kn = k1 - k0;                                    // multiple of 64 (K is a multiple of 128)
  const int nblk = kn >> 6;
  const int nmb = (nblk + 3) >> 2;
  const int w0 = blockIdx.y * kSkRows;
  const int xp = p.xpitch;
  constexpr int R = kSkRows / C;                             // output rows finished by each rank

  uint16_t *sB = reinterpret_cast<uint16_t *>(sm + p.off_b);       // [r][R]
  uint16_t *sX = reinterpret_cast<uint16_t *>(sm + p.off_x);       // [M][xp]
  float *sRecv = reinterpret_cast<float *>(sm + p.off_part);       // [C ranks][R rows][M tokens]
  float *sXA = reinterpret_cast<float *>(sm + p.off_xa);           // [M][r]
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + p.off_bar);   // [nmb] codes, then one for B
  uint64_t *bar_b = bars + (p.ks / kSkMacro);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bar_b + 1);
  const Waiter waiter{abort_flag, p.limit_ns};

  // ---- 1. every load of the CTA is issued first: X by all threads (cp.async,
  //         8 bytes each: an 8-byte piece never straddles a 64-value block of the
  //         padded layout); by one thread the code boxes, then this rank's B columns
  if (tid == 32) {
    prefetch_tmap(&tm_codes);
    prefetch_tmap(&tm_b);
  }
  for (int t = warp; t < p.M; t += kSkThreads / 32) {
    const uint16_t *xr = p.X + static_cast<int64_t>(t) * p.K + k0;
    const uint32_t xs = smem_u32(sX + t * xp);
    for (int ch = lane; ch < (kn >> 2); ch += 32)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(xs + 2 * sk_xoff(ch * 4)), "l"(xr + ch * 4)
                   : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  if (tid == 0) {
    *abort_flag = 0;
    for (int i = 0; i <= p.ks / kSkMacro; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
    for (int mb = 0; mb < nmb; ++mb) {
      mbar_arrive_expect_tx(&bars[mb], kSkBoxBytes);
      tma_load_2d(sm + mb * kSkBoxBytes, &tm_codes, &bars[mb], (k0 >> 1) + mb * (kSkMacro / 2), w0);
    }
    mbar_arrive_expect_tx(bar_b, static_cast<uint32_t>(p.r * R * 2));
    tma_load_2d(sB, &tm_b, bar_b, w0 + static_cast<int>(rank) * R, 0);
  }
  // block constants of this lane's rows, kSkPre macro-blocks ahead (raw q8 and step)
  const int ra = warp * 16 + g, rb = ra + 8;
  const int64_t ba = (static_cast<int64_t>(w0 + ra) * p.K + k0) >> 6;
  const int64_t bb = (static_cast<int64_t>(w0 + rb) * p.K + k0) >> 6;
  uint32_t qa[kSkPre], qb[kSkPre];
  float sa[kSkPre], sb[kSkPre];
#pragma unroll
  for (int i = 0; i < kSkPre; ++i) {
    const int blk = 4 * i + c;
    qa[i] = qb[i] = 0u;
    sa[i] = sb[i] = 0.f;
    if (blk < nblk) {
      // single-level constants (q8 null): code 1 and the block's own constant, so the
      // scale RN32(1 * a_b) = a_b exactly
      qa[i] = p.q8 ? p.q8[ba + blk] : 1u;
      qb[i] = p.q8 ? p.q8[bb + blk] : 1u;
      sa[i] = p.q8 ? p.step[(ba + blk) >> 8] : p.step[ba + blk];
      sb[i] = p.q8 ? p.step[(bb + blk) >> 8] : p.step[bb + blk];
    }
  }
  float L[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) L[i] = p.levels[i];
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();   // barrier init and X visible to every warp

  // ---- 2. main product over the macro-blocks
  const bool tok0 = g < p.M, tok1 = g + 8 < p.M;
  const int ntiles = p.M > 8 ? 2 : 1;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  bool ok = true;
  const uint32_t codes_base = smem_u32(sm);
  for (int mb = 0; mb < nmb; ++mb) {
    const uint32_t qa0 = qa[0], qb0 = qb[0];
    const float sa0 = sa[0], sb0 = sb[0];
#pragma unroll
    for (int i = 0; i + 1 < kSkPre; ++i) {
      qa[i] = qa[i + 1]; qb[i] = qb[i + 1]; sa[i] = sa[i + 1]; sb[i] = sb[i + 1];
    }
    {
      const int blk = 4 * (mb + kSkPre) + c;
      qa[kSkPre - 1] = qb[kSkPre - 1] = 0u;
      sa[kSkPre - 1] = sb[kSkPre - 1] = 0.f;
      if (blk < nblk) {
        qa[kSkPre - 1] = p.q8 ? p.q8[ba + blk] : 1u;
        qb[kSkPre - 1] = p.q8 ? p.q8[bb + blk] : 1u;
        sa[kSkPre - 1] = p.q8 ? p.step[(ba + blk) >> 8] : p.step[ba + blk];
        sb[kSkPre - 1] = p.q8 ? p.step[(bb + blk) >> 8] : p.step[bb + blk];
      }
    }
    ok = __all_sync(0xffffffffu, wait_bar(&bars[mb], 0, waiter));
    if (!ok) break;
    const int blk = mb * 4 + c;
    const bool valid = blk < nblk;
    // an absent block keeps zero codes and a zero table, so it decodes to zeros
    uint4 ca0 = make_uint4(0, 0, 0, 0), ca1 = ca0, cb0 = ca0, cb1 = ca0;
    Nf4Lut la{}, lb{};
    if (valid) {
      // 128B swizzle: 16-byte chunk j of row r sits at chunk j ^ (r & 7); here r & 7 = g
      const uint32_t box = codes_base + mb * kSkBoxBytes;
      const uint32_t c0 = static_cast<uint32_t>(((2 * c) ^ g) << 4), c1 = static_cast<uint32_t>(((2 * c + 1) ^ g) << 4);
      ca0 = ld_shared_v4(box + ra * 128 + c0);
      ca1 = ld_shared_v4(box + ra * 128 + c1);
      cb0 = ld_shared_v4(box + rb * 128 + c0);
      cb1 = ld_shared_v4(box + rb * 128 + c1);
      nf4_build_lut(L, __fmul_rn(static_cast<float>(qa0), sa0), la);
      nf4_build_lut(L, __fmul_rn(static_cast<float>(qb0), sb0), lb);
    }
    const uint32_t wa[8] = {ca0.x, ca0.y, ca0.z, ca0.w, ca1.x, ca1.y, ca1.z, ca1.w};
    const uint32_t wb[8] = {cb0.x, cb0.y, cb0.z, cb0.w, cb1.x, cb1.y, cb1.z, cb1.w};
    const uint32_t xbase = smem_u32(sX + g * xp + blk * 68);
    const bool x0ok = valid && tok0, x1ok = valid && tok1;
#pragma unroll
    for (int j = 0; j < 8; ++j) {                 // code word j: elements 8j .. 8j+7, k-steps 2j, 2j+1
      uint32_t oa[4], ob[4];
      nf4_decode8(wa[j], la, oa);
      nf4_decode8(wb[j], lb, ob);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t a[4] = {oa[2 * h], ob[2 * h], oa[2 * h + 1], ob[2 * h + 1]};
        const int s = 2 * j + h;
        uint2 x0 = make_uint2(0u, 0u);
        if (x0ok) x0 = ld_shared_v2(xbase + 8 * s);
        mma_16816_bf16(acc[0], a, x0.x, x0.y);
        if (ntiles > 1) {
          uint2 x1 = make_uint2(0u, 0u);
          if (x1ok) x1 = ld_shared_v2(xbase + (8 * xp + 4 * s) * 2);
          mma_16816_bf16(acc[1], a, x1.x, x1.y);
        }
      }
    }
  }

  // ---- 3. push the partial Y rows to the rank that finishes them: slot
  // [this rank][row within the owner's R][token] of the owner's receive buffer
  {
    const uint32_t recv = smem_u32(sRecv);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = h ? rb : ra;
      const uint32_t owner = static_cast<uint32_t>(row / R);
      const uint32_t base = recv + 4u * static_cast<uint32_t>((static_cast<int>(rank) * R + row % R) * p.M);
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int tk = nt * 8 + 2 * c + e;
          if (tk < p.M) {
            const uint32_t addr = map_rank(base + 4u * tk, owner);
            asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(acc[nt][2 * h + e]) : "memory");
          }
        }
      }
    }
  }
  // XA comes from the XA kernel: wait for that grid (a no-op when launched plainly)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  for (int i = tid; i < p.M * p.r; i += kSkThreads) sXA[i] = p.xa[i];
  ok = __all_sync(0xffffffffu, wait_bar(bar_b, 0, waiter)) && ok;

  // ---- 4. cluster barrier: every partial has landed in its owner's buffer; after
  // it no CTA touches another's shared memory, so each may finish and leave
  if (C > 1) cluster_sync_all(); else __syncthreads();
  for (int i = tid; i < R * p.M; i += kSkThreads) {
    const int tk = i / R, rr = i - tk * R;
    float v = 0.f;
#pragma unroll
    for (int q = 0; q < C; ++q) v += sRecv[(q * R + rr) * p.M + tk];
    float lora = 0.f;
    for (int j = 0; j < p.r; ++j)
      lora = fmaf(sXA[tk * p.r + j], __uint_as_float(static_cast<uint32_t>(sB[j * R + rr]) << 16), lora);
    const __nv_bfloat16 h = __float2bfloat16_rn(v + p.s * lora);
    p.Y[static_cast<int64_t>(tk) * p.N + w0 + static_cast<int>(rank) * R + rr] = *reinterpret_cast<const uint16_t *>(&h);
  }
}

// XA = X A for few tokens: one cluster of kXaCluster CTAs, rank q takes rows
// [q kx, (q+1) kx) of the contraction in chunks of `chunk` rows, each chunk of A
// (contiguous) and of every token row of X fetched by one bulk copy; X rows on
// the MMA's M (tokens), adapter columns on N.  Partials are summed by rank 0 in
// rank order.
constexpr int kXaCluster = 8;

struct XaParams {
  const uint16_t *X;   // [M, K] bf16 (the adapter input: dropped-out elements already zero)
  const uint16_t *A;   // [K, r] bf16
  float *xa;           // [M, r] fp32
  int M, K, r, kx;
  int chunk;           // contraction rows per pass, a multiple of 16
  uint64_t limit_ns;
  float scale;         // applied to the sum before it is stored (1/(1-p) under dropout)
};

inline int xa_chunk_rows(int r) { return r <= 64 ? 512 : 256; }
inline int xa_smem_bytes(int r) {
  const int ch = xa_chunk_rows(r);
  return 16 * (ch + 8) * 2 + ch * r * 2 + 8 * 128 * 4 + 16 * r * 4 + 32;
}

__global__ void __launch_bounds__(256, 1) qlora_xa_kernel(const __grid_constant__ XaParams p) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  extern __shared__ __align__(128) uint8_t xa_smem[];
  const int xpitch = p.chunk + 8;
  uint16_t *sX = reinterpret_cast<uint16_t *>(xa_smem);                          // [16][xpitch]
  uint8_t *sA = xa_smem + 16 * xpitch * 2;                                       // [chunk][r] dense
  float *sSlot = reinterpret_cast<float *>(sA + p.chunk * p.r * 2);              // [8 warps][16][8]
  float *sPart = sSlot + 8 * 128;                                                // [16][r]
  uint64_t *bar = reinterpret_cast<uint64_t *>(sPart + 16 * p.r);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(bar + 1);
  const Waiter waiter{abort_flag, p.limit_ns};
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, c = lane & 3;
  const uint32_t rank = cluster_ctarank();
  const int k0 = min(p.K, static_cast<int>(rank) * p.kx), k1 = min(p.K, k0 + p.kx);
  const bool tok0 = g < p.M, tok1 = g + 8 < p.M;
  const int jt = p.r >> 3;
  const int nsplit = jt >= 8 ? 1 : 8 / jt;
  const int my_t8 = (jt >= 8) ? warp : warp / nsplit, my_part = (jt >= 8) ? 0 : warp % nsplit;
  const bool active = (jt >= 8) || (warp < jt * nsplit);
  if (tid == 0) {
    *abort_flag = 0;
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  bool ok = true;
  int pass = 0;
  for (int a0 = k0; a0 < k1; a0 += p.chunk, ++pass) {
    const int rows = min(p.chunk, k1 - a0);
    __syncthreads();                                // barrier init seen; the previous chunk consumed
    if (tid == 0) {
      const uint32_t arow_bytes = static_cast<uint32_t>(rows * 2);
      mbar_arrive_expect_tx(bar, static_cast<uint32_t>(rows * p.r * 2) + arow_bytes * static_cast<uint32_t>(p.M));
      bulk_load(sA, p.A + static_cast<int64_t>(a0) * p.r, static_cast<uint32_t>(rows * p.r * 2), bar);
      for (int t = 0; t < p.M; ++t) bulk_load(sX + t * xpitch, p.X + static_cast<int64_t>(t) * p.K + a0, arow_bytes, bar);
    }
    const bool got = __syncthreads_and(wait_bar(bar, static_cast<uint32_t>(pass & 1), waiter)) != 0;
    ok = ok && got;
    if (!ok) break;
    if (active) {
      for (int kst = my_part; kst < rows / 16; kst += nsplit) {
        const uint32_t x0 = smem_u32(sX + g * xpitch + kst * 16 + 2 * c);
        const uint32_t x8 = smem_u32(sX + (g + 8) * xpitch + kst * 16 + 2 * c);
        uint32_t a[4] = {0u, 0u, 0u, 0u};
        if (tok0) {
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a[0]) : "r"(x0));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a[2]) : "r"(x0 + 16));
        }
        if (tok1) {
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a[1]) : "r"(x8));
          asm volatile("ld.shared.u32 %0, [%1];" : "=r"(a[3]) : "r"(x8 + 16));
        }
        const uint32_t arow = smem_u32(sA + (kst * 16 + (lane & 15)) * p.r * 2);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int t8 = my_t8 + u * 8;
          if (t8 < jt) {
            uint32_t b0, b1;
            ldmatrix_x2_trans(arow + t8 * 16, b0, b1);
            mma_16816_bf16(acc[u], a, b0, b1);
          }
        }
      }
    }
  }
  if (active) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int t8 = my_t8 + u * 8;
      if (t8 < jt) {
        float *dst = (nsplit == 1) ? sPart + t8 * 8 : sSlot + warp * 128;
        const int ld = (nsplit == 1) ? p.r : 8;
        dst[g * ld + 2 * c] = acc[u][0];
        dst[g * ld + 2 * c + 1] = acc[u][1];
        dst[(g + 8) * ld + 2 * c] = acc[u][2];
        dst[(g + 8) * ld + 2 * c + 1] = acc[u][3];
      }
    }
  }
  if (nsplit > 1) {
    __syncthreads();
    for (int i = tid; i < p.M * p.r; i += 256) {
      const int t = i / p.r, j = i - t * p.r, t8 = j >> 3;
      float v = 0.f;
      for (int q = 0; q < nsplit; ++q) v += sSlot[(t8 * nsplit + q) * 128 + t * 8 + (j & 7)];
      sPart[i] = v;
    }
  }
  cluster_sync_all();
  if (rank == 0) {
    const uint32_t base = smem_u32(sPart);
    for (int i = tid; i < p.M * p.r; i += 256) {
      float v = 0.f;
#pragma unroll
      for (int q = 0; q < kXaCluster; ++q) v += ld_dsmem_f32(map_rank(base + 4u * i, q));
      p.xa[i] = __fmul_rn(v, p.scale);
    }
  }
  cluster_sync_all();   // the peers' partials stay until rank 0 has read them
}

// Shared-memory plan of one launch; false when nothing fits in `limit` bytes.
struct SkinnyPlan {
  int C, ks, xpitch;
  int off_b, off_x, off_part, off_xa, off_bar, smem;
};

inline bool skinny_plan_for(int M, int K, int r, int C, int limit, SkinnyPlan &pl) {
  auto up16 = [](int v) { return (v + 15) & ~15; };
  const int macro = K / kSkMacro + ((K % kSkMacro) ? 1 : 0);
  pl.C = C;
  pl.ks = (macro + C - 1) / C * kSkMacro;
  const int xbase = pl.ks + pl.ks / 16;
  pl.xpitch = xbase + (((16 - xbase) % 64) + 64) % 64;
  const int nbars = pl.ks / kSkMacro + 1;
  // bulk-copy destinations first: the code boxes (1024-byte aligned for the
  // 128B swizzle), then B (128-byte aligned)
  int off = (pl.ks / kSkMacro) * kSkBoxBytes;
  pl.off_b = off;    off += (r * (kSkRows / C) * 2 + 127) & ~127;
  pl.off_x = off;    off += up16(M * pl.xpitch * 2);
  pl.off_part = off; off += up16(kSkRows * M * 4);   // sized by the tokens: a smaller CTA fits more per SM
  pl.off_xa = off;   off += up16(M * r * 4);
  pl.off_bar = off;  off += 8 * nbars + 16;
  pl.smem = off + 1024;                          // slack for aligning the base to 1024 bytes
  if (pl.off_b & 127) return false;
  return pl.smem <= limit;
}

}  // namespace qlora
