// Dequant-fused tcgen05 GEMM for the QLoRA linear layer (sm_100a).
//
// Forward ("QLoRA", ozercemkelahmet.com, How it works, Step 5; essay at
// fanfani.net, section "The crucial split"):
//     Y^T[n, m] = sum_k deq(W)[n, k] X[m, k]  +  sum_c B'[n, c] XAhl[m, c]
// dX (Step 6: gradients flow through the dequantized weights):
//     dX^T[k, m] = sum_n deq(W)[n, k] dY[m, n] +  sum_c A'[k, c] Ghl[m, c]
//
// The weight side is the MMA's A operand (M = 128 weight rows or columns per
// tile) and the tokens are the MMA's N (BN = 256 per tile), so every
// dequantized value feeds 256 tokens.  The rank-r LoRA term is appended as
// extra K steps in the same TMEM accumulator: the activation side carries
// s*XA (or s*G) split into bf16 hi and lo halves (c < r: hi, r <= c < 2r: lo)
// and the weight side repeats B^T (or A) twice, so the adapter term is
// accumulated to ~2^-16 relative precision, not bf16 precision.
//
// Warp roles (640 threads, one CTA per SM, persistent over tiles):
//   warp 0        TMA producer of the activation tiles (X / dY, or the LoRA
//                 hi/lo operand).
//   warp 1        TMEM allocator and single-thread MMA issuer.
//   warps 2, 3    weight producers, alternate stages: lane 0 TMA-loads the
//                 packed 4-bit codes of a stage into their own ring (so the small
//                 weight stream runs ahead of the activation ring instead of
//                 waiting behind it); all 32 lanes rebuild the stage's 128 block
//                 constants RN32(q8 * step) from the 8-bit codes and the fp32
//                 group constants (requested one own stage ahead) next to them.
//   warps 4..7    epilogue: TMEM -> registers -> bf16 -> global (masked rows).
//   warps 8..19   dequant producers, three warpgroups taking every third stage:
//                 packed codes + block constant -> bf16 tile in the
//                 128-byte-swizzled UMMA layout (one 64-value block per
//                 thread, decoded through a 16-entry table held in registers),
//                 then the LoRA weight tiles.
// Every wait is bounded (see Waiter); a wait that runs out aborts the block.
//
// CTA pairs (cta_group::2, clusters of two; output widths that are multiples of 256):
// a tile is 256 weight rows x 256 tokens.  Each CTA dequantizes its own 128 weight
// rows and loads its own 128 tokens of the activation tile, both into its own shared
// memory at the same offsets; the pair's leader (rank 0) issues one M = 256, N = 256
// product per K step over both CTAs' operands, writing each CTA's 128 rows into that
// CTA's TMEM, and its commits arrive on the barrier at the same offset in both CTAs.
// The peer's warp 1 passes each stage's readiness (its own 128 dequant arrivals and
// its own activation copy) on to the leader's full_B with a remote arrival; the
// peer's epilogue warps free the accumulator on the leader's tmem_empty.  Per
// CTA, the tensor core reads half as many activation bytes per weight byte as a
// single CTA does (the two halves of N are exchanged between the pair), and the
// activation tile crosses L2 once per 256 weight rows instead of once per 128.
//
// Last-wave split: with T tiles on G persistent CTAs, T mod G tiles are left for a
// last round in which most SMs would idle.  When at most G/2 remain, each of them
// is split along the contraction into two halves taken by CTAs 2i and 2i+1 (the
// second half also runs the LoRA steps).  Whichever half finishes first stores its
// fp32 partial tile to scratch and publishes it; the other adds that partial to its
// own accumulator and writes the output (last arriver).  A half learns its role
// from an atomic arrival counter per split tile, which a kernel earlier in the same
// call sets to zero.  The only wait is the last arriver's, for a partial whose
// writer has already arrived (so is running), which makes it independent of how
// the CTAs are scheduled.  The sum of two fp32 values does not depend on their
// order, so the result is the same whichever half finishes first.
#pragma once
#include "common.cuh"

namespace qlora {

constexpr int kGemmThreads = 640;
constexpr int kBN = 256;                  // tokens per tile (MMA N)
constexpr int kWT = 128;                  // weight-side rows per tile (MMA M)
constexpr int kBK = 64;                   // contraction per stage (one quant block)
#ifndef QLORA_GEMM_STAGES_W
#define QLORA_GEMM_STAGES_W 6
#endif
constexpr int kStagesW = QLORA_GEMM_STAGES_W;   // packed code + constant ring (4.5 KB stages)
constexpr int kAStageBytes = kWT * 128;   // 16 KB: 128 weight rows x 64 values
constexpr int kWStageBytes = 4096;        // packed codes of one stage
constexpr int kSStageBytes = 512;         // 128 fp32 block constants of one stage
constexpr uint32_t kSplitArrive = 1u;     // split-tile counter: one per arriving half
constexpr uint32_t kSplitReady = 16u;     // added once the first half's partial is stored
constexpr int kTmemCols = 512;            // two 256-column fp32 accumulators

constexpr int kMaxStagesAB = 6;

// The MMA stages: one ring of (activation tile, dequantized weight tile) pairs,
// released by a single commit per stage.  A CTA pair loads half the token tile per
// CTA, so its stages are half as large and the ring is deeper.
template <bool PAIR>
struct GemmShape {
  static constexpr int kStagesAB = PAIR ? 6 : 4;
  static constexpr int kBRows = PAIR ? kBN / 2 : kBN;    // tokens of the activation tile in this CTA
  static constexpr int kBStageBytes = kBRows * 128;       // 16 or 32 KB
  static constexpr int kTileRows = PAIR ? 2 * kWT : kWT;  // weight-side rows of one tile
  static constexpr int kSmemBytes = 1024 /*align slack*/ + kStagesAB * (kBStageBytes + kAStageBytes) +
                                    kStagesW * (kWStageBytes + kSStageBytes) + 1024 /*barriers, flags*/;
};
constexpr int kGemmSmemBytes = GemmShape<false>::kSmemBytes > GemmShape<true>::kSmemBytes
                                   ? GemmShape<false>::kSmemBytes
                                   : GemmShape<true>::kSmemBytes;
static_assert(kGemmSmemBytes <= 227 * 1024, "GEMM shared memory exceeds the per-CTA limit");
static_assert(GemmShape<true>::kStagesAB <= kMaxStagesAB && GemmShape<false>::kStagesAB <= kMaxStagesAB, "");
static_assert(kStagesW <= 32 && kMaxStagesAB <= 32, "ring bookkeeping uses 32-bit masks");
static_assert(kStagesW % 2 == 0, "the two weight producer warps each keep to the slots of one parity");
static_assert(kGemmThreads == 256 + 3 * 128,
              "warps 0..7, then three dequant warpgroups; the dequant loop gives stage a to warpgroup a mod 3");
// A dequant warpgroup's previous stage was a - 3, whose wait needed A stage a - 3 - S
// consumed; with S >= 3 that covers a - 2S, so its wait on A slot a never sees the
// barrier two phases behind.  Its wait on W slot w comes after the A slot is free,
// which needs the W stage kStagesW earlier to map to an A stage at least S back.
static_assert(GemmShape<false>::kStagesAB >= 3 && GemmShape<true>::kStagesAB >= 3,
              "the A-slot phase argument needs at least three A stages");
static_assert(kStagesW >= GemmShape<false>::kStagesAB && kStagesW >= GemmShape<true>::kStagesAB,
              "the W-slot phase argument needs at least as many W stages as A stages");

enum GemmMode : int { kModeFwd = 0, kModeDx = 1 };

struct GemmParams {
  int M;             // tokens
  int n_out;         // output row length (N for fwd, K for dX)
  int num_m_tiles;   // ceil(M / 256)
  int num_w_tiles;   // weight-side tiles: n_out / 128 (single CTA) or n_out / 256 (CTA pair)
  int group_m;       // token tiles per raster group (see tile_coords)
  int kb_main;       // main stages: K/64 (fwd) or N/64 (dX)
  int kb_lora;       // LoRA stages: ceil(2r / 64)
  int r;
  int lora_ld;       // row pitch of the LoRA weight operand source: N (B [r,N]) or r (A [K,r])
  int KB;            // 64-value blocks per weight row: K / 64
  const uint8_t *q8;       // 8-bit block constants of W, [N * KB]; null: single-level
  const float *step;       // fp32 group constants, one per 256 blocks (single-level: one per block)
  const uint16_t *lora_w;  // fwd: B [r, N];  dX: A [K, r]
  uint16_t *out;     // Y [M, N] or dX [M, K]
  uint64_t limit_ns;
  int split_base;    // first tile of the split last round (a multiple of the unit count)
  int split_count;   // tiles split into two contraction halves (0: no split)
  int kb_mid;        // first main stage of the second half
  float *scratch;    // [split_count][tile rows / 128][128][256] fp32 partials of the half that arrives first
  unsigned int *flags;   // [split_count][tile rows / 128] arrival counters, zero at launch
  // dX under adapter-input dropout (null otherwise): the keep mask of X [M, K], bit-packed
  // (element m K + k in bit (m K + k) mod 32 of word (m K + k) / 32).  The adapter term
  // then gets its own accumulator and is added as keep * keep_scale * term per element.
  const uint32_t *keep32;
  float keep_scale;      // 1 / (1 - p)
  float levels[16];
};

// The work items of a unit (a CTA, or a CTA pair) u of G: whole tiles u + i*G below
// split_base, then (when a last round is split) one half of tile split_base + u/2:
// part 1 = main stages [0, kb_mid), part 2 = [kb_mid, kb_main) plus the LoRA stages.
struct GemmItem {
  int tile, kb0, kb1, part;
  bool lora;
};

// The unit this CTA belongs to, and the number of units.
template <bool PAIR>
QDEV int gemm_unit() { return PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x); }
template <bool PAIR>
QDEV int gemm_units() { return PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x); }

template <bool PAIR>
QDEV bool gemm_item(const GemmParams &p, int num_tiles, int it, GemmItem &w) {
  const int G = gemm_units<PAIR>(), b = gemm_unit<PAIR>();
  const int whole_end = p.split_count ? p.split_base : num_tiles;
  const int t = b + it * G;
  if (t < whole_end) {
    w.tile = t; w.kb0 = 0; w.kb1 = p.kb_main; w.part = 0; w.lora = true;
    return true;
  }
  if (!p.split_count || it != whole_end / G || b >= 2 * p.split_count) return false;
  w.tile = p.split_base + (b >> 1);
  w.part = 1 + (b & 1);
  w.kb0 = (w.part == 1) ? 0 : p.kb_mid;
  w.kb1 = (w.part == 1) ? p.kb_mid : p.kb_main;
  w.lora = (w.part == 2);
  return true;
}

// Token tile and weight-side tile of tile index t.  Tiles are taken in groups of
// group_m token tiles: within a group the token tile varies fastest, so the CTAs
// running at the same time share group_m activation tiles (kept in L2 while the group
// sweeps the weight) and each weight tile they stream serves group_m of them, instead
// of one activation tile against every weight tile of the layer (which re-reads the
// whole weight from DRAM once per token tile when it does not fit in L2).
QDEV void tile_coords(const GemmParams &p, int t, int &mt, int &wt) {
  const int per_group = p.group_m * p.num_w_tiles;
  const int grp = t / per_group;
  const int m_base = grp * p.group_m;
  const int gm = min(p.group_m, p.num_m_tiles - m_base);
  const int idx = t - grp * per_group;
  mt = m_base + idx % gm;
  wt = idx / gm;
}

// One weight producer warp's walk over the W stages it owns (global W stage
// counter c = c0 + j with c mod 2 = wp), with the block indices of its lane's four
// constants kept incrementally: slot idx = lane + 32 i holds
//   fwd: weight row w0 + idx, block kb;
//   dX:  weight row kb*64 + (idx & 63), block w0/64 + (idx >> 6).
template <int MODE, bool PAIR>
struct WStageCursor {
  bool have;
  int it, kb0, n, j, w0;
  uint32_t c0;          // global W stage counter at the item's first stage
  int64_t b[4];         // block index of the item's first stage
  int64_t inc;          // block index step from one stage to the next

  QDEV void enter(const GemmParams &p, int num_tiles, int lane) {
    GemmItem w;
    have = gemm_item<PAIR>(p, num_tiles, it, w);
    if (!have) return;
    kb0 = w.kb0;
    n = w.kb1 - w.kb0;
    int mti, wti;
    tile_coords(p, w.tile, mti, wti);
    w0 = wti * GemmShape<PAIR>::kTileRows + (PAIR ? static_cast<int>(cluster_ctarank()) * kWT : 0);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int idx = lane + 32 * i;
      if (MODE == kModeFwd) b[i] = static_cast<int64_t>(w0 + idx) * p.KB + kb0;
      else b[i] = static_cast<int64_t>(kb0 * kBK + (idx & 63)) * p.KB + (w0 >> 6) + (idx >> 6);
    }
    inc = (MODE == kModeFwd) ? 1 : static_cast<int64_t>(kBK) * p.KB;
  }
  // moves past the ends of items until stage j lies inside one (or none is left)
  QDEV void settle(const GemmParams &p, int num_tiles, int lane) {
    while (have && j >= n) {
      j -= n;
      c0 += static_cast<uint32_t>(n);
      ++it;
      enter(p, num_tiles, lane);
    }
  }
  QDEV void start(const GemmParams &p, int num_tiles, int lane, uint32_t wp) {
    it = 0;
    c0 = 0;
    j = static_cast<int>(wp);
    enter(p, num_tiles, lane);
    settle(p, num_tiles, lane);
  }
  QDEV void advance(const GemmParams &p, int num_tiles, int lane) {
    j += 2;
    settle(p, num_tiles, lane);
  }
  // raw constants of stage j: (q8, step) or, single-level, (1, the block's absmax)
  QDEV void load(const GemmParams &p, uint32_t (&q)[4], float (&st)[4]) const {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int64_t bi = b[i] + static_cast<int64_t>(j) * inc;
      if (p.q8) {
        q[i] = __ldg(p.q8 + bi);
        st[i] = __ldg(p.step + (bi >> 8));
      } else {
        q[i] = 1u;
        st[i] = __ldg(p.step + bi);
      }
    }
  }
};

QDEV void epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

template <int MODE, bool PAIR>
__global__ void __launch_bounds__(kGemmThreads, 1)
    qlora_gemm_kernel(const __grid_constant__ CUtensorMap tm_act,   // X or dY, bf16 [M, contraction]
                      const __grid_constant__ CUtensorMap tm_codes, // packed codes, u8 [N, K/2]
                      const __grid_constant__ CUtensorMap tm_lora,  // hi/lo LoRA operand, bf16 [M, 2r]
                      const __grid_constant__ GemmParams p) {
  using S = GemmShape<PAIR>;
  constexpr int kStages = S::kStagesAB;
  constexpr int kBStage = S::kBStageBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t *sB = smem;
  uint8_t *sA = sB + kStages * kBStage;
  uint8_t *sW = sA + kStages * kAStageBytes;
  float *sS = reinterpret_cast<float *>(sW + kStagesW * kWStageBytes);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sS + kStagesW * (kSStageBytes / 4));
  uint64_t *full_B = bars;                  // activation tile landed (and, at a pair's leader, the peer's stage)
  uint64_t *full_A = full_B + kStages;      // dequantized tile written (128 thread arrivals)
  uint64_t *empty_A = full_A + kStages;     // MMAs of the stage done: both tiles free
  uint64_t *full_W = empty_A + kStages;
  uint64_t *empty_W = full_W + kStagesW;
  uint64_t *tmem_full = empty_W + kStagesW;
  uint64_t *tmem_empty = tmem_full + 2;
  uint64_t *drain = tmem_empty + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  int *abort_flag = reinterpret_cast<int *>(tmem_slot + 1);
  float *sL = reinterpret_cast<float *>(abort_flag + 1);
  volatile int *split_role = reinterpret_cast<volatile int *>(sL + 16);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int row_off = static_cast<int>(rank) * kWT;           // this CTA's weight rows in a tile
  const int tok_off = static_cast<int>(rank) * S::kBRows;     // this CTA's tokens of a tile

  if (tid == 0) {
    // full_B: this CTA's expect_tx arrival, plus at a pair's leader the peer's forwarded
    // "my stage is ready"; full_A: one arrival per dequant thread of this CTA, each after
    // its own stores and proxy fence
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full_B[i], (PAIR && leader) ? 2 : 1);
      mbar_init(&full_A[i], 128);
      mbar_init(&empty_A[i], 1);
    }
    // full_W: the TMA's expect_tx arrival plus one per lane of the weight producer;
    // empty_W: one per consumer thread, each once it has used what it read
    for (int i = 0; i < kStagesW; ++i) { mbar_init(&full_W[i], 33); mbar_init(&empty_W[i], 128); }
    // tmem_empty: one per epilogue warp (both CTAs' at a pair's leader)
    for (int i = 0; i < 2; ++i) { mbar_init(&tmem_full[i], 1); mbar_init(&tmem_empty[i], PAIR ? 8 : 4); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < 16) sL[tid] = p.levels[tid];
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_act);
    prefetch_tmap(&tm_codes);
    prefetch_tmap(&tm_lora);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  // a pair's barriers are initialized before either CTA arrives on the other's
  if (PAIR) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Waiter wt{abort_flag, p.limit_ns};

  const int num_tiles = p.num_m_tiles * p.num_w_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------ activation producer
    if (lane == 0) {
      int bs = 0;
      uint32_t bph = 0;
      uint32_t armedB = 0, lastB = 0;          // bit s: armed at least once / parity of last arming
      bool ok = true;
      GemmItem w;
      for (int it = 0; ok && gemm_item<PAIR>(p, num_tiles, it, w); ++it) {
        int mti, wti;
        tile_coords(p, w.tile, mti, wti);
        const int m0 = mti * kBN + tok_off;
        const int nmain = w.kb1 - w.kb0, nst = nmain + (w.lora ? p.kb_lora : 0);
        for (int j = 0; j < nst; ++j) {
          if (!wait_bar(&empty_A[bs], bph ^ 1u, wt)) { ok = false; break; }
          mbar_arrive_expect_tx(&full_B[bs], kBStage);
          if (j < nmain)
            tma_load_2d(sB + bs * kBStage, &tm_act, &full_B[bs], (w.kb0 + j) * kBK, m0);
          else
            tma_load_2d(sB + bs * kBStage, &tm_lora, &full_B[bs], (j - nmain) * kBK, m0);
          armedB |= 1u << bs;
          lastB = (lastB & ~(1u << bs)) | (bph << bs);
          if (++bs == kStages) { bs = 0; bph ^= 1u; }
        }
      }
      // Every issued copy lands before the block may exit (bounded).  At a pair's
      // leader a phase also needs the peer's forwarded arrival, which comes once the
      // peer's own copy of that stage has landed, or not at all after an abort: the
      // wait is bounded either way, and this CTA's copies have landed when it ends.
      volatile int no_abort = 0;
      const Waiter final_wt{&no_abort, p.limit_ns};
      for (int s = 0; s < kStages; ++s)
        if (armedB & (1u << s)) wait_bar(&full_B[s], (lastB >> s) & 1u, final_wt);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ weight producers
    // Warp 2 takes the even W stages, warp 3 the odd ones (the W ring has an even
    // number of slots, so each warp keeps to its own slots).  Per stage, lane 0
    // TMA-loads the packed codes and all 32 lanes rebuild the 128 block constants;
    // the raw constants of a warp's next stage are requested before it waits for the
    // current one.
    const uint32_t wp = static_cast<uint32_t>(warp - 2);
    WStageCursor<MODE, PAIR> cur;
    cur.start(p, num_tiles, lane, wp);
    uint32_t qc[4] = {0u, 0u, 0u, 0u}, qn[4] = {0u, 0u, 0u, 0u};
    float sc[4] = {0.f, 0.f, 0.f, 0.f}, sn[4] = {0.f, 0.f, 0.f, 0.f};
    if (cur.have) cur.load(p, qc, sc);
    uint32_t armedW = 0, lastW = 0;
    while (cur.have) {
      WStageCursor<MODE, PAIR> nx = cur;
      nx.advance(p, num_tiles, lane);
      if (nx.have) nx.load(p, qn, sn);
      const uint32_t c = cur.c0 + static_cast<uint32_t>(cur.j);
      const int ws = static_cast<int>(c % kStagesW);
      const uint32_t wph = (c / kStagesW) & 1u;
      // warp-uniform: every lane arrives on full_W below
      if (!__all_sync(0xffffffffu, wait_bar(&empty_W[ws], wph ^ 1u, wt))) break;
      if (lane == 0) {
        const int kb = cur.kb0 + cur.j;
        // the slot's previous codes were read through the generic proxy; the TMA
        // below rewrites them through the async proxy: order the two
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&full_W[ws], kWStageBytes);
        if (MODE == kModeFwd) {
          // codes: 32 bytes (64 values of K) x 128 weight rows
          tma_load_2d(sW + ws * kWStageBytes, &tm_codes, &full_W[ws], kb * 32, cur.w0);
        } else {
          // codes: 64 bytes (128 values of K from w0) x 64 weight rows n = kb*64..
          tma_load_2d(sW + ws * kWStageBytes, &tm_codes, &full_W[ws], cur.w0 / 2, kb * kBK);
        }
        armedW |= 1u << ws;
        lastW = (lastW & ~(1u << ws)) | (wph << ws);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
        sS[ws * 128 + lane + 32 * i] = __fmul_rn(static_cast<float>(qc[i]), sc[i]);
      mbar_arrive(&full_W[ws]);
      cur = nx;
#pragma unroll
      for (int i = 0; i < 4; ++i) { qc[i] = qn[i]; sc[i] = sn[i]; }
    }
    if (lane == 0) {
      volatile int no_abort = 0;
      const Waiter final_wt{&no_abort, p.limit_ns};
      for (int s = 0; s < kStagesW; ++s)
        if (armedW & (1u << s)) wait_bar(&full_W[s], (lastW >> s) & 1u, final_wt);
    }
  } else if (warp == 1 && leader) {
    // ------------------------------------------------------------ MMA issuer
    // A lean loop: descriptors of stage 0 are built once; a stage adds its byte
    // offset >> 4 to the start-address field, a K=16 step adds 32 B (K-major)
    // or 4096 B (MN-major, two 8-row groups) >> 4; one commit per stage frees
    // both tiles of the stage (in both CTAs of a pair).
    if (lane == 0) {
      constexpr int kM = PAIR ? 2 * kWT : kWT;
      constexpr uint32_t idesc_main = make_idesc_bf16(kM, kBN, MODE == kModeDx, false);
      constexpr uint32_t idesc_lora = make_idesc_bf16(kM, kBN, MODE == kModeFwd, false);
      constexpr uint32_t a_step_main = (MODE == kModeDx) ? (4096u >> 4) : (32u >> 4);
      constexpr uint32_t a_step_lora = (MODE == kModeFwd) ? (4096u >> 4) : (32u >> 4);
      const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
      const uint64_t ad_main0 = (MODE == kModeDx) ? sw128_desc(a0, 1024, 2048) : sw128_desc(a0, 16, 1024);
      const uint64_t ad_lora0 = (MODE == kModeFwd) ? sw128_desc(a0, 1024, 2048) : sw128_desc(a0, 16, 1024);
      const uint64_t bd0 = sw128_desc(b0, 16, 1024);
      const int kb_lora = p.kb_lora;
      const int lora_steps_total = (2 * p.r) / 16;
      // under dropout (dX only) one tile at a time: main product in columns [0, 256),
      // adapter term in [256, 512)
      const bool two_acc = (MODE == kModeDx) && (p.keep32 != nullptr);
      const int nacc = two_acc ? 1 : 2;
      auto mma = [&](uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t accumulate) {
        if constexpr (PAIR) mma_bf16_ss_pair(d, ad, bd, idesc, accumulate);
        else mma_bf16_ss(d, ad, bd, idesc, accumulate);
      };
      auto commit = [&](uint64_t *bar) {
        if constexpr (PAIR) mma_commit_pair(bar, static_cast<uint16_t>(0x3));
        else mma_commit(bar);
      };
      int st = 0, acc = 0;
      uint32_t ph = 0, accph = 0;
      bool ok = true;
      GemmItem w;
      for (int it = 0; ok && gemm_item<PAIR>(p, num_tiles, it, w); ++it) {
        if (!wait_bar(&tmem_empty[acc], accph ^ 1u, wt)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        const uint32_t d_lora = two_acc ? tmem_base + static_cast<uint32_t>(kBN) : d_tmem;
        for (int kb = 0; kb < w.kb1 - w.kb0; ++kb) {
          if (!wait_bar(&full_A[st], ph, wt) || !wait_bar(&full_B[st], ph, wt)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = ad_main0 + static_cast<uint64_t>(st * (kAStageBytes >> 4));
          const uint64_t bd = bd0 + static_cast<uint64_t>(st * (kBStage >> 4));
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma(d_tmem, ad + k * a_step_main, bd + k * 2, idesc_main, (kb | k) ? 1u : 0u);
          commit(&empty_A[st]);
          if (++st == kStages) { st = 0; ph ^= 1u; }
        }
        for (int ls = 0; ok && w.lora && ls < kb_lora; ++ls) {
          if (!wait_bar(&full_A[st], ph, wt) || !wait_bar(&full_B[st], ph, wt)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = ad_lora0 + static_cast<uint64_t>(st * (kAStageBytes >> 4));
          const uint64_t bd = bd0 + static_cast<uint64_t>(st * (kBStage >> 4));
          const int nk = min(4, lora_steps_total - ls * 4);
          for (int k = 0; k < nk; ++k)
            mma(d_lora, ad + k * a_step_lora, bd + k * 2, idesc_lora, (two_acc && (ls | k) == 0) ? 0u : 1u);
          commit(&empty_A[st]);
          if (++st == kStages) { st = 0; ph ^= 1u; }
        }
        if (!ok) break;
        commit(&tmem_full[acc]);
        if (++acc == nacc) { acc = 0; accph ^= 1u; }
      }
      // All issued MMAs complete before TMEM (and, in a pair, the peer's operands) is
      // released (bounded).
      commit(drain);
      volatile int no_abort = 0;
      const Waiter final_wt{&no_abort, p.limit_ns};
      wait_bar(drain, 0, final_wt);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ pair peer: forwarder
    // The peer's own stage (its dequantized tile, 128 thread arrivals, and its
    // activation copy) completes on its own barriers; once both have, the stage is
    // passed on to the leader's full_B of that stage, in stage order.  The peer's
    // stores were made visible to the tensor core by each thread's proxy fence, and
    // its copy had landed, before this thread observed the two phases.
    if (PAIR && lane == 0) {
      int bs = 0;
      uint32_t bph = 0;
      bool ok = true;
      GemmItem w;
      for (int it = 0; ok && gemm_item<PAIR>(p, num_tiles, it, w); ++it) {
        const int nst = (w.kb1 - w.kb0) + (w.lora ? p.kb_lora : 0);
        for (int j = 0; j < nst; ++j) {
          if (!wait_bar(&full_A[bs], bph, wt) || !wait_bar(&full_B[bs], bph, wt)) { ok = false; break; }
          mbar_arrive_remote(&full_B[bs], 0u);
          if (++bs == kStages) { bs = 0; bph ^= 1u; }
        }
      }
      // the leader's MMAs read this CTA's shared memory and write its TMEM: they
      // complete before either is released (bounded)
      volatile int no_abort = 0;
      const Waiter final_wt{&no_abort, p.limit_ns};
      wait_bar(drain, 0, final_wt);
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;             // TMEM lane quadrant of this warp
    const int row = q * 32 + lane;      // weight-side row within this CTA's 128
    constexpr int kParts = S::kTileRows / kWT;                       // 128-row parts per tile
    const bool two_acc = (MODE == kModeDx) && (p.keep32 != nullptr);
    const int nacc = two_acc ? 1 : 2;
    const int64_t keep_words = static_cast<int64_t>(p.n_out) >> 5;   // mask words per token
    int acc = 0;
    uint32_t accph = 0;
    GemmItem w;
    for (int it = 0; gemm_item<PAIR>(p, num_tiles, it, w); ++it) {
      int mti, wti;
      tile_coords(p, w.tile, mti, wti);
      const int m0 = mti * kBN;
      const int w0 = wti * S::kTileRows + row_off;
      // warp-uniform decision: the TMEM loads below are .sync.aligned
      const bool got = __all_sync(0xffffffffu, wait_bar(&tmem_full[acc], accph, wt) ? 1 : 0);
      if (!got) break;
      tc_fence_after();
      const int sidx = (w.tile - p.split_base) * kParts + static_cast<int>(rank);   // split tiles only
      float *prow = (w.part != 0) ? p.scratch + (static_cast<int64_t>(sidx) * kWT + row) * kBN : nullptr;
      // role: 0 a whole tile; 1 the first half of a split tile to finish (stores its
      // partial); 2 the second (adds the partial and writes the output)
      int role = 0;
      if (w.part != 0) {
        if (warp == 4 && lane == 0) {
          const uint32_t old = atom_acq_rel_add_u32(p.flags + sidx, kSplitArrive);
          const int rl = ((old & (kSplitReady - 1u)) == 0u) ? 1 : 2;
          if (rl == 2) {
            // the other half has arrived, so it is running: wait (bounded) for its partial
            const uint64_t t0 = globaltimer_ns();
            while (ld_acquire_u32(p.flags + sidx) < kSplitReady) {
              if (*reinterpret_cast<volatile int *>(abort_flag) || globaltimer_ns() - t0 > p.limit_ns) {
                *reinterpret_cast<volatile int *>(abort_flag) = 1;
                atomicOr(&g_device_status, kStatTimeout);
                break;
              }
            }
          }
          *split_role = rl;
        }
        epilogue_bar();
        role = *split_role;
        if (role == 2) __threadfence();
      }
      uint16_t *outc = p.out + w0 + row;
      for (int cc = 0; cc < kBN / 16; ++cc) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                               static_cast<uint32_t>(acc * kBN + cc * 16),
                           v);
        tmem_wait_ld();
        if (two_acc && w.lora) {
          // this tile's contribution: main + keep * (1/(1-p)) * adapter term, per element;
          // the warp's 32 rows are 32 consecutive input features, one mask word per token
          const int mb = m0 + cc * 16;
          const int64_t kw = (w0 + q * 32) >> 5;
          uint32_t lv[16];
          tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                 static_cast<uint32_t>(kBN + cc * 16),
                             lv);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int m = mb + j;
            const uint32_t word = (m < p.M) ? __ldg(p.keep32 + static_cast<int64_t>(m) * keep_words + kw) : 0u;
            if ((word >> lane) & 1u)
              v[j] = __float_as_uint(__fadd_rn(__uint_as_float(v[j]), __fmul_rn(p.keep_scale, __uint_as_float(lv[j]))));
          }
        }
        if (role == 1) {
          float4 *d4 = reinterpret_cast<float4 *>(prow + cc * 16);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            d4[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          continue;
        }
        if (role == 2) {
          const float4 *s4 = reinterpret_cast<const float4 *>(prow + cc * 16);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float4 f = __ldcg(s4 + j);
            v[4 * j] = __float_as_uint(__uint_as_float(v[4 * j]) + f.x);
            v[4 * j + 1] = __float_as_uint(__uint_as_float(v[4 * j + 1]) + f.y);
            v[4 * j + 2] = __float_as_uint(__uint_as_float(v[4 * j + 2]) + f.z);
            v[4 * j + 3] = __float_as_uint(__uint_as_float(v[4 * j + 3]) + f.w);
          }
        }
        const int mb = m0 + cc * 16;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int m = mb + j;
          if (m < p.M) {
            const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(v[j]));
            outc[static_cast<int64_t>(m) * p.n_out] = *reinterpret_cast<const uint16_t *>(&h);
          }
        }
      }
      if (role == 1) {
        // publish the partial tile: every epilogue thread's stores, then one release
        __threadfence();
        epilogue_bar();
        if (warp == 4 && lane == 0) red_release_add_u32(p.flags + sidx, kSplitReady);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR && !leader) mbar_arrive_remote(&tmem_empty[acc], 0u);
        else mbar_arrive(&tmem_empty[acc]);
      }
      if (++acc == nacc) { acc = 0; accph ^= 1u; }
    }
  } else if (warp >= 8) {
    // ------------------------------------------------------------ dequant producers
    const int t = (tid - 256) & 127;    // row slot within the stage
    const int grp = (tid - 256) >> 7;   // warpgroup g takes the stages a with a mod 3 = g
    float L[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) L[i] = sL[i];
    uint32_t a_cnt = 0, w_cnt = 0;      // stages seen so far (all / main only)
    bool ok = true;
    GemmItem w;
    for (int it = 0; ok && gemm_item<PAIR>(p, num_tiles, it, w); ++it) {
      int mti, wti;
      tile_coords(p, w.tile, mti, wti);
      const int w0 = wti * S::kTileRows + row_off;
      const int nmain = w.kb1 - w.kb0, nst = nmain + (w.lora ? p.kb_lora : 0);
      for (int j = 0; j < nst; ++j, ++a_cnt) {
        const bool main = j < nmain;
        const uint32_t my_w = w_cnt;
        if (main) ++w_cnt;
        if ((a_cnt % 3u) != static_cast<uint32_t>(grp)) continue;
        const int as = static_cast<int>(a_cnt % kStages);
        const uint32_t aph = (a_cnt / kStages) & 1u;
        if (main) {
          const int ws = static_cast<int>(my_w % kStagesW);
          const uint32_t wph = (my_w / kStagesW) & 1u;
          // warp-uniform: the per-warp arrivals below need every lane on the same path.
          // The A slot first: once it is free the MMA has consumed A stage
          // a_cnt - kStages and every stage before it, so the dequant of W stage
          // my_w - kStagesW (an earlier A stage, whichever warpgroup took it) has passed
          // its own wait on this W slot, whose barrier is then at least in the phase this
          // wait names.  (Waiting on full_W first could see a phase two behind and take
          // the previous parity's completion for this one.)
          const bool w_ok = wait_bar(&empty_A[as], aph ^ 1u, wt) && wait_bar(&full_W[ws], wph, wt);
          if (!__all_sync(0xffffffffu, w_ok)) { ok = false; break; }
          uint32_t src, dst;
          int swz;
          float sc;
          if (MODE == kModeFwd) {
            // row t of the tile: weight row w0+t, 64 values of K (one block), K-major
            src = smem_u32(sW + ws * kWStageBytes + t * 32);
            sc = sS[ws * 128 + t];
            dst = smem_u32(sA + as * kAStageBytes + t * 128);
            swz = t & 7;
          } else {
            // weight row n = kb*64 + nl, 64 values of K from w0 + 64*kk; MN-major:
            // K index nl, M group kk
            const int nl = t & 63, kk = t >> 6;
            src = smem_u32(sW + ws * kWStageBytes + nl * 64 + kk * 32);
            sc = sS[ws * 128 + kk * 64 + nl];
            dst = smem_u32(sA + as * kAStageBytes + (nl >> 3) * 2048 + kk * 1024 + (nl & 7) * 128);
            swz = nl & 7;
          }
          const uint4 c0 = ld_shared_v4(src);
          const uint4 c1 = ld_shared_v4(src + 16);
          Nf4Lut lut;
          nf4_build_lut(L, sc, lut);
          const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t o[4];
            nf4_decode8(cw[c], lut, o);
            st_shared_v4(dst + ((c ^ swz) << 4), o[0], o[1], o[2], o[3]);
          }
          // the W slot is released by every thread itself, and only once the decode
          // above has used the codes and the constant it read: the producer then
          // rewrites the constants and (after a proxy fence) lets a TMA rewrite the codes
          mbar_arrive(&empty_W[ws]);
          // every thread publishes its own row: its stores, the fence that makes them
          // visible to the tensor core's (async proxy) reads, then its arrival
          fence_proxy_async_smem();
          mbar_arrive(&full_A[as]);
        } else {
          // LoRA weight-side stage: c in [ls*64, ls*64+64), value = src(c mod r) for c < 2r
          const int ls = j - nmain;
          if (!__all_sync(0xffffffffu, wait_bar(&empty_A[as], aph ^ 1u, wt))) { ok = false; break; }
          const uint32_t abase = smem_u32(sA + as * kAStageBytes);
          if (MODE == kModeFwd) {
            // MN-major: K index cr (0..63), M group mg: B[c mod r][w0 + 64 mg ..]
            const int cr = t & 63, mg = t >> 6;
            const int c = ls * 64 + cr;
            const uint32_t d = abase + (cr >> 3) * 2048 + mg * 1024 + (cr & 7) * 128;
            const uint16_t *srcg = p.lora_w + static_cast<int64_t>(c % p.r) * p.lora_ld + w0 + mg * 64;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
              uint4 v = make_uint4(0, 0, 0, 0);
              if (c < 2 * p.r) v = *reinterpret_cast<const uint4 *>(srcg + ch * 8);
              st_shared_v4(d + ((ch ^ (cr & 7)) << 4), v.x, v.y, v.z, v.w);
            }
          } else {
            // K-major: row t = input feature k = w0 + t: A[k][c mod r] for c < 2r
            const uint32_t d = abase + t * 128;
            const uint16_t *srcg = p.lora_w + static_cast<int64_t>(w0 + t) * p.lora_ld;
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
              const int c = ls * 64 + ch * 8;
              uint4 v = make_uint4(0, 0, 0, 0);
              if (c < 2 * p.r) v = *reinterpret_cast<const uint4 *>(srcg + (c % p.r));
              st_shared_v4(d + ((ch ^ (t & 7)) << 4), v.x, v.y, v.z, v.w);
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(&full_A[as]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  // neither CTA of a pair leaves while the other may still arrive on its barriers
  if (PAIR) cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, kTmemCols);
    else tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace qlora
