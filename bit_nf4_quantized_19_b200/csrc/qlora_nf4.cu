// libqlora_nf4.so: C ABI of the QLoRA NF4 frozen-base linear layer (see
// include/qlora_nf4.h for the contract of every entry point).
#include "qlora_nf4.h"

#include <atomic>
#include <cstring>
#include <map>
#include <mutex>

#include "common.cuh"
#include "gemm_kernel.cuh"
#include "lora_mma.cuh"
#include "merge_kernel.cuh"
#include "nf4_table.hpp"
#include "quant_kernels.cuh"
#include "skinny_kernel.cuh"

using namespace qlora;

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr int64_t kSkinnyMaxTokens = 16;   // forward with at most this many tokens: one-launch kernel
std::atomic<uint32_t> g_wait_limit_us{2000000u};
std::atomic<int> g_gemm_pairing{1};        // CTA-pair GEMM where the output width allows it

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qlora_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

constexpr int kSkSmemLimit = 200 * 1024;

template <int C>
cudaError_t set_skinny_attrs() {
  cudaError_t e = cudaFuncSetAttribute(qlora_skinny_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSkSmemLimit);
  if (e == cudaSuccess && C > 8)
    e = cudaFuncSetAttribute(qlora_skinny_kernel<C>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

// Persistent units of the fused GEMM: single CTAs, and CTA pairs (clusters of two)
// that the device can hold at once with one CTA per SM (0: no pairs).
struct GemmUnits {
  int ctas = 148;
  int pairs = 74;
};

struct DeviceInfo {
  int sms = 0;
  int major = 0;
  bool gemm_attr_set = false;
  GemmUnits units;
};

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

qlora_status device_info(DeviceInfo **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_NO_DEVICE;
  if (dev < 0 || dev >= kMaxDevices) return QLORA_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DeviceInfo &d = g_dev[dev];
  if (d.sms == 0) {
    int sms = 0, major = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return QLORA_ERR_CUDA;
    d.sms = sms;
    d.major = major;
  }
  if (d.major != 10) return QLORA_ERR_NO_DEVICE;
  if (!d.gemm_attr_set) {
    if (cudaFuncSetAttribute(qlora_gemm_kernel<kModeFwd, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGemmSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(qlora_gemm_kernel<kModeDx, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGemmSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(qlora_gemm_kernel<kModeFwd, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGemmSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(qlora_gemm_kernel<kModeDx, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGemmSmemBytes) != cudaSuccess)
      return QLORA_ERR_CUDA;
    if (cudaFuncSetAttribute(lora_mma_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kLmSmemMax) !=
            cudaSuccess ||
        cudaFuncSetAttribute(lora_mma_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, kLmSmemMax) !=
            cudaSuccess ||
        cudaFuncSetAttribute(nf4_quantize_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kQuantSmemBytes) !=
            cudaSuccess ||
        cudaFuncSetAttribute(qlora_xa_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             xa_smem_bytes(64) > xa_smem_bytes(128) ? xa_smem_bytes(64) : xa_smem_bytes(128)) !=
            cudaSuccess ||
        set_skinny_attrs<1>() != cudaSuccess || set_skinny_attrs<2>() != cudaSuccess ||
        set_skinny_attrs<4>() != cudaSuccess || set_skinny_attrs<8>() != cudaSuccess ||
        set_skinny_attrs<16>() != cudaSuccess ||
        cudaFuncSetAttribute(nf4_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             merge_smem_max()) != cudaSuccess)
      return QLORA_ERR_CUDA;
    d.units.ctas = d.sms;
    d.units.pairs = 0;
    {
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3(static_cast<unsigned>(d.sms / 2 * 2), 1, 1);
      cfg.blockDim = dim3(kGemmThreads, 1, 1);
      cfg.dynamicSmemBytes = kGemmSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (d.sms >= 2 &&
          cudaOccupancyMaxActiveClusters(&n, qlora_gemm_kernel<kModeFwd, true>, &cfg) == cudaSuccess && n > 0)
        d.units.pairs = n < d.sms / 2 ? n : d.sms / 2;
      (void)cudaGetLastError();
    }
    d.gemm_attr_set = true;
  }
  *out = &d;
  return QLORA_OK;
}

// ------------------------------------------------------------------ launch timing
struct Profiler {
  std::mutex mu;
  bool on = false;
  int dev = -1;
  long long count = 0;
  cudaEvent_t ev[2 * QLORA_PROFILE_CAP];
  int kind[QLORA_PROFILE_CAP];
  bool created = false;
};
Profiler g_prof;

bool prof_ensure_events() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (g_prof.created && g_prof.dev == dev) return true;
  if (g_prof.created) {
    for (auto &e : g_prof.ev) cudaEventDestroy(e);
    g_prof.created = false;
  }
  for (auto &e : g_prof.ev)
    if (cudaEventCreate(&e) != cudaSuccess) return false;
  g_prof.created = true;
  g_prof.dev = dev;
  return true;
}

// Records a start event on construction and a stop event on destruction,
// around one kernel launch, when profiling is enabled.
class LaunchTimer {
 public:
  LaunchTimer(int kind, cudaStream_t st) : st_(st) {
    if (!g_prof.on) return;
    std::lock_guard<std::mutex> lk(g_prof.mu);
    slot_ = static_cast<int>(g_prof.count % QLORA_PROFILE_CAP);
    g_prof.kind[slot_] = kind;
    ++g_prof.count;
    cudaEventRecord(g_prof.ev[2 * slot_], st_);
  }
  ~LaunchTimer() {
    if (slot_ >= 0) cudaEventRecord(g_prof.ev[2 * slot_ + 1], st_);
  }

 private:
  cudaStream_t st_;
  int slot_ = -1;
};

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool make_map_2d(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner,
                 uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                 CUtensorMapSwizzle sw) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ workspace
size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct Workspace {
  char *base;
  size_t used;
  size_t cap;
  void *take(size_t bytes) {
    const size_t off = align256(used);
    if (off + bytes > cap) return nullptr;
    used = off + bytes;
    return base + off;
  }
};

// ---- launch geometry of the rank-r contractions (lora_mma_kernel)
constexpr int kLmMaxSplits = kLmClusterMax;
// Ring geometry of the rank-r launches: steps of 64 per ring slot, the ring's byte
// budget and the fewest slots, for the projections (K-major) and the gradients.
// Measured on the 65B-shaped step: two steps per slot and a 192 KB ring took the
// projections from 466 to 417 us per step; the same geometry made the gradients
// slower (305 to 329 us), so they keep one step per slot in a 110 KB ring.
struct LmRing {
  int sub, bytes, min_slots;
};
constexpr LmRing kLmRingProject{2, 192 * 1024, 2};
constexpr LmRing kLmRingGrad{1, 110 * 1024, 3};

// Ring depths a plan may take: at least the ring's fewest slots and enough slots to
// hold what the epilogue keeps in the idle ring (the fp32 partial tile and, for a
// projection, the stage of its transposed hi|lo halves); at most the ring's byte
// budget (and 8 slots), unless the epilogue needs more.
struct LmSlots {
  int min, max;
};
constexpr LmSlots lm_slots(const LmRing &ring, int nn, bool projection) {
  const int stage_bytes = ring.sub * (kLmABytes + nn * 128);
  const int epi_bytes = projection ? lm_epilogue_bytes(nn) : lm_partial_bytes(nn);
  int lo = (epi_bytes + stage_bytes - 1) / stage_bytes;
  if (lo < ring.min_slots) lo = ring.min_slots;
  int hi = ring.bytes / stage_bytes;
  if (hi > 8) hi = 8;
  if (hi < lo) hi = lo;
  return LmSlots{lo, hi};
}
// Every plan the host can pick fits the attribute: projections have nn = r rounded up
// to 16 (r <= 128), gradients nn = 2r.
constexpr bool lm_plans_fit() {
  for (int nn = 16; nn <= 128; nn += 16)
    if (lora_mma_smem_bytes(nn, lm_slots(kLmRingProject, nn, true).max, kLmRingProject.sub) > kLmSmemMax) return false;
  for (int nn = 16; nn <= 256; nn += 16)
    if (lora_mma_smem_bytes(nn, lm_slots(kLmRingGrad, nn, false).max, kLmRingGrad.sub) > kLmSmemMax) return false;
  return true;
}
static_assert(lm_plans_fit(), "a rank-r ring plan exceeds the shared-memory attribute");

struct LmGeom {
  int nn, row_tiles, stages_total, sps, splits, num_stages, sub;
  uint32_t tmem_cols;
};

// Clusters of one rank-r configuration the GPU holds at once (0 if the runtime cannot
// say).  Cluster placement is per GPC, so this is well below sms * CTAs-per-SM / splits
// for large shared-memory rings; the answer is cached per configuration.
template <bool A_MN>
int lm_max_clusters(int splits, int smem) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> cache;
  std::lock_guard<std::mutex> lk(mu);
  const auto key = std::make_pair(splits, smem);
  const auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(1, static_cast<unsigned>(splits), 1);
  cfg.blockDim = dim3(kLmThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(splits);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, lora_mma_kernel<A_MN>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  cache[key] = n;
  return n;
}

// Split count and ring depth: the fewest waves of clusters, then the most splits (more
// CTAs streaming the activation at once), then the deepest ring.  Each extra wave costs
// a CTA's whole fixed latency (setup, first load, cluster reduction), which at these
// sizes is as long as its streaming.
template <bool A_MN>
LmGeom lm_geom(int64_t rows, int64_t contraction, int nn, int sms) {
  LmGeom g{};
  g.nn = nn;
  g.row_tiles = static_cast<int>((rows + kLmRows - 1) / kLmRows);
  g.stages_total = static_cast<int>((contraction + 63) / 64);
  uint32_t tc = 32;
  while (tc < static_cast<uint32_t>(nn)) tc <<= 1;
  g.tmem_cols = tc;
  const LmRing ring = A_MN ? kLmRingGrad : kLmRingProject;
  g.sub = ring.sub;
  const LmSlots slots = lm_slots(ring, nn, !A_MN);
  const int st_min = slots.min, st_max = slots.max;
  int64_t best_waves = -1;
  for (int c = kLmMaxSplits; c >= 1; c >>= 1) {   // the splits of a tile form one cluster
    if (c > 1 && c > g.stages_total) continue;
    const int total = g.stages_total > 0 ? g.stages_total : 1;
    const int sps = (total + c - 1) / c;
    const int splits = (total + sps - 1) / sps;
    for (int S = st_max; S >= st_min; --S) {
      int active = lm_max_clusters<A_MN>(splits, lora_mma_smem_bytes(nn, S, g.sub));
      if (active <= 0) active = (2 * sms) / splits;   // the runtime could not say
      if (active <= 0) continue;
      const int64_t waves = (g.row_tiles + active - 1) / active;
      if (best_waves < 0 || waves < best_waves) {
        best_waves = waves;
        g.sps = sps;
        g.splits = splits;
        g.num_stages = S;
      }
      if (waves == 1) break;   // a deeper ring that still fits in one wave is preferred
    }
  }
  return g;
}

int nn_proj(int r) { return (r + 15) / 16 * 16; }
int64_t pad8(int64_t m) { return (m + 7) / 8 * 8; }

// Shape of one fused GEMM launch (see gemm_kernel.cuh): single CTAs with 128-row weight
// tiles, or CTA pairs with 256-row tiles when the output width is a multiple of 256;
// and its last-wave split, where the tiles left for the last round are split along the
// contraction when at most half the units (CTAs or pairs) remain.
struct GemmSplit {
  bool pair = false;
  int base = 0, count = 0;
  int parts() const { return pair ? 2 : 1; }     // 128-row partial tiles per split tile
  size_t scratch_bytes() const { return static_cast<size_t>(count) * parts() * kWT * kBN * 4; }
  size_t flag_bytes() const { return static_cast<size_t>(count) * parts() * 4; }
};
bool gemm_pairable(int64_t n_out, const GemmUnits &u) { return n_out % (2 * kWT) == 0 && u.pairs > 0; }
GemmSplit gemm_split(int64_t M, int64_t n_out, int64_t contraction, const GemmUnits &u, bool pair) {
  GemmSplit g;
  g.pair = pair;
  const int64_t units = pair ? u.pairs : u.ctas;
  const int64_t tiles = ((M + kBN - 1) / kBN) * (n_out / (pair ? 2 * kWT : kWT));
  const int64_t grid = tiles < units ? tiles : units;
  if (grid <= 0 || contraction / kBK < 2) return g;
  const int64_t rem = tiles % grid;
  if (rem > 0 && 2 * rem <= grid) {
    g.base = static_cast<int>(tiles - rem);
    g.count = static_cast<int>(rem);
  }
  return g;
}
// The variant a call uses, fixed once per call.
GemmSplit gemm_plan(int64_t M, int64_t n_out, int64_t contraction, const GemmUnits &u) {
  return gemm_split(M, n_out, contraction, u, g_gemm_pairing.load() != 0 && gemm_pairable(n_out, u));
}
size_t split_workspace(const GemmSplit &g) { return align256(g.scratch_bytes()) + align256(g.flag_bytes()); }
// Workspace sizes do not depend on the variant switch: the larger of the two.
size_t split_workspace_any(int64_t M, int64_t n_out, int64_t contraction, const GemmUnits &u) {
  size_t a = split_workspace(gemm_split(M, n_out, contraction, u, false));
  if (gemm_pairable(n_out, u)) {
    const size_t b = split_workspace(gemm_split(M, n_out, contraction, u, true));
    if (b > a) a = b;
  }
  return a;
}

// Scratch of one split GEMM launch, carved from the workspace before the call's first
// launch: its arrival counters are cleared by the rank-r projection that precedes the
// GEMM in the same call.
struct SplitScratch {
  GemmSplit g;
  float *partial = nullptr;
  unsigned int *flags = nullptr;
};

size_t fwd_workspace(int64_t M, int64_t N, int64_t K, int r, const GemmUnits &u) {
  size_t b = 0;
  b += align256(static_cast<size_t>(r) * K * 2);               // A^T
  b += align256(static_cast<size_t>(M) * 2 * r * 2);           // s*XA hi/lo
  b += align256(static_cast<size_t>(M) * r * 4);               // XA when XA_out is NULL
  b += split_workspace_any(M, N, K, u);                      // last-wave partial tiles
  return b + 256;
}

size_t bwd_workspace(int64_t M, int64_t N, int64_t K, int r, const GemmUnits &u) {
  size_t b = 0;
  b += align256(static_cast<size_t>(r) * K * 2);               // A^T (XA recompute)
  b += align256(static_cast<size_t>(M) * r * 4);               // G
  b += align256(static_cast<size_t>(M) * 2 * r * 2);           // s*G hi/lo
  b += align256(static_cast<size_t>(2 * r) * pad8(M) * 2);     // s*G hi/lo transposed
  b += align256(static_cast<size_t>(2 * r) * pad8(M) * 2);     // s*XA hi/lo transposed
  b += align256(static_cast<size_t>(M) * r * 4);               // XA recomputed
  b += split_workspace_any(M, K, N, u);                      // last-wave partial tiles (dX)
  return b + 256;
}

bool take_split(Workspace &ws, const GemmSplit &g, SplitScratch &out) {
  out.g = g;
  if (!g.count) return true;
  out.partial = static_cast<float *>(ws.take(g.scratch_bytes()));
  out.flags = static_cast<unsigned int *>(ws.take(g.flag_bytes()));
  return out.partial && out.flags;
}

qlora_status check_nf4(const qlora_nf4_t *Wq) {
  if (!Wq || !Wq->codes || !Wq->step) return QLORA_ERR_INVALID_ARG;   // q8 null: single-level constants
  if (Wq->rows <= 0 || Wq->cols <= 0) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(Wq->codes) || (Wq->q8 && !aligned16(Wq->q8)) || !aligned16(Wq->step))
    return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

qlora_status check_linear_shape(int64_t M, const qlora_nf4_t *Wq, int r) {
  if (M < 1 || M > (1ll << 30)) return QLORA_ERR_INVALID_ARG;
  if (r < 8 || r > 128 || (r % 8) != 0) return QLORA_ERR_INVALID_ARG;
  if (Wq->rows % 128 != 0 || Wq->cols % 128 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (Wq->rows > (1ll << 24) || Wq->cols > (1ll << 24)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  return QLORA_OK;
}

int grid_for(int64_t total, int sms) {
  int64_t g = (total + 255) / 256;
  if (g > static_cast<int64_t>(sms) * 8) g = static_cast<int64_t>(sms) * 8;
  return g < 1 ? 1 : static_cast<int>(g);
}

// One operand pair of a rank-r product: act [act_rows (tokens), act_cols (features)]
// row-major bf16, q [q_rows, q_cols] bf16 with a row pitch of q_pitch elements, and the
// number of output rows.
struct LmOperands {
  const uint16_t *act;
  int64_t act_rows, act_cols;
  const uint16_t *q;
  int64_t q_rows, q_cols, q_pitch;
  int64_t rows;
};

template <bool A_MN>
bool lm_maps(const LmOperands &o, int nn, CUtensorMap *tm_act, CUtensorMap *tm_q) {
  return make_map_2d(tm_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o.act, o.act_cols, o.act_rows, o.act_cols * 2,
                     64, A_MN ? 64 : kLmRows, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_map_2d(tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o.q, o.q_cols, o.q_rows, o.q_pitch * 2, 64,
                     static_cast<uint32_t>(nn), CU_TENSOR_MAP_SWIZZLE_128B);
}

// D[rows, nn] = act (K-major rows x c, or MN-major c x rows) * q^T, split over the
// contraction inside clusters of g.splits CTAs that reduce in rank order; the final
// outputs are written by the kernel (projection or gradient form, see LoraMmaParams).
// With `second`, the same launch also computes a second gradient product over the same
// contraction (p.out1 / p.layout1 set by the caller); its row tiles follow the first's.
template <bool A_MN>
qlora_status launch_lora_mma(const LmOperands &o, int64_t contraction, int nn, LoraMmaParams p, int sms,
                             cudaStream_t st, const LmOperands *second = nullptr) {
  const int64_t tiles0 = (o.rows + kLmRows - 1) / kLmRows;
  const int64_t tiles1 = second ? (second->rows + kLmRows - 1) / kLmRows : 0;
  const LmGeom g = lm_geom<A_MN>((tiles0 + tiles1) * kLmRows, contraction, nn, sms);
  CUtensorMap tm_act, tm_q, tm_act1, tm_q1;
  if (!lm_maps<A_MN>(o, nn, &tm_act, &tm_q)) return QLORA_ERR_CUDA;
  if (second) {
    if (!lm_maps<A_MN>(*second, nn, &tm_act1, &tm_q1)) return QLORA_ERR_CUDA;
    p.rows1 = static_cast<int>(second->rows);
  } else {
    tm_act1 = tm_act;
    tm_q1 = tm_q;
    p.rows1 = static_cast<int>(o.rows);
    p.out1 = p.out;
    p.layout1 = p.layout;
  }
  p.tiles0 = static_cast<int>(tiles0);
  p.rows = static_cast<int>(o.rows);
  p.nn = nn;
  p.stages_total = g.stages_total;
  p.stages_per_split = g.sps;
  p.num_stages = g.num_stages;
  p.sub = g.sub;
  p.tmem_cols = g.tmem_cols;
  p.splits = g.splits;
  p.limit_ns = static_cast<uint64_t>(g_wait_limit_us.load()) * 1000ull;
  const int smem = lora_mma_smem_bytes(nn, g.num_stages, g.sub);
  if (smem > kLmSmemMax) return QLORA_ERR_UNSUPPORTED_SHAPE;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(g.row_tiles), static_cast<unsigned>(g.splits), 1);
  cfg.blockDim = dim3(kLmThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = static_cast<unsigned>(g.splits);
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  LaunchTimer lt(A_MN ? QLORA_K_GRAD : QLORA_K_PROJECT, st);
  return cuda_status(cudaLaunchKernelEx(&cfg, lora_mma_kernel<A_MN>, tm_act, tm_q, tm_act1, tm_q1, p));
}

// XA = X A (or G = dY B^T): fp32 [M, r] plus hi/lo of s*result in [M, 2r] and/or [2r, pad8(M)].
// The fp32 result is multiplied by out_scale before it is stored and split (1/(1-p) for
// the product over a dropped-out adapter input).
qlora_status launch_projection(const uint16_t *act, int64_t M, int64_t C, const uint16_t *qT,
                               int r, float s, float *out, uint16_t *hl, uint16_t *hlT, int sms,
                               cudaStream_t st, const SplitScratch *clear = nullptr,
                               float out_scale = 1.0f) {
  LoraMmaParams p{};
  p.out_scale = p.out_scale1 = out_scale;
  if (clear && clear->g.count) {
    p.zero = clear->flags;
    p.zero_n = clear->g.count * clear->g.parts();
  }
  p.grad = 0;
  p.r = r;
  p.s = s;
  p.out = out;
  p.hl = hl;
  p.hlT = hlT;
  p.ldT = static_cast<int>(pad8(M));
  const LmOperands o{act, M, C, qT, r, C, C, M};
  return launch_lora_mma<false>(o, C, nn_proj(r), p, sms, st);
}

qlora_status launch_hilo_t(const float *v, int64_t M, int r, float s, uint16_t *hlT, int sms,
                           cudaStream_t st) {
  LaunchTimer lt(QLORA_K_PREP, st);
  hilo_t_kernel<<<grid_for(M * r, sms), 256, 0, st>>>(v, static_cast<int>(M), r, s, hlT,
                                                       static_cast<int>(pad8(M)));
  return cuda_status(cudaGetLastError());
}

// Both adapter gradients in one launch, each act^T * (hi + lo) over the M tokens:
// dA [K, r] = scale_dA * X^T (s G) from X [M, K] (the adapter input: under dropout its
// kept elements, with scale_dA = 1/(1-p)) and ghlT [2r, pad8(M)];
// dB [r, N] = (s XA)^T dY from dY [M, N] and xahlT [2r, pad8(M)].
// With `accumulate` both are added into dA and dB.
qlora_status launch_grads(const uint16_t *X, const uint16_t *dY, int64_t M, int64_t K, int64_t N,
                          const uint16_t *ghlT, const uint16_t *xahlT, int r, float *dA, float *dB,
                          int sms, cudaStream_t st, float scale_dA = 1.0f, int accumulate = 0) {
  LoraMmaParams p{};
  p.grad = 1;
  p.out_scale = scale_dA;
  p.out_scale1 = 1.0f;
  p.accumulate = accumulate;
  p.r = r;
  p.out = dA;
  p.layout = 0;
  p.out1 = dB;
  p.layout1 = 1;
  const LmOperands a{X, M, K, ghlT, 2 * r, M, pad8(M), K};
  const LmOperands b{dY, M, N, xahlT, 2 * r, M, pad8(M), N};
  return launch_lora_mma<true>(a, M, 2 * r, p, sms, st, &b);
}

// Xd = X (.) keep (bit-packed mask), n = M K elements, a multiple of 8.
qlora_status launch_mask(const uint16_t *X, const uint8_t *keep, int64_t n, uint16_t *Xd, int sms, cudaStream_t st) {
  LaunchTimer lt(QLORA_K_PREP, st);
  mask_input_kernel<<<grid_for(n / 8, sms), 256, 0, st>>>(X, keep, n / 8, Xd);
  return cuda_status(cudaGetLastError());
}

qlora_status launch_transpose(const uint16_t *A, int64_t K, int r, uint16_t *AT, int sms, cudaStream_t st) {
  LaunchTimer lt(QLORA_K_PREP, st);
  transpose_bf16_kernel<<<grid_for(K * r, sms), 256, 0, st>>>(A, static_cast<int>(K), r, AT);
  return cuda_status(cudaGetLastError());
}

// Few-token forward: one cluster launch, no workspace.  Clusters of C CTAs split K
// into C slices of ks (a multiple of 256) values, one cluster per 128 weight rows.
// C is chosen for the fewest waves of clusters (the device holds only so many at
// once: the count comes from the occupancy query, cached per plan), then in the order
// 8, 4, 16, 2, 1.  8 splits give each weight tile the most SMs; fewer splits keep a
// tall weight (many row tiles) in one wave, where 8 would leave a partial second wave
// of short-lived CTAs.  False when no plan fits: the caller then takes the general path.
template <int C>
cudaError_t skinny_occupancy(int smem, int *n) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(C), 1, 1);
  cfg.blockDim = dim3(kSkThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaOccupancyMaxActiveClusters(n, qlora_skinny_kernel<C>, &cfg);
}

std::mutex g_sk_occ_mu;
std::map<std::pair<int, int>, int> g_sk_occ[kMaxDevices];

// Clusters of plan pl the current device holds at once (0: none).
int skinny_resident(const SkinnyPlan &pl) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  const std::pair<int, int> key{pl.C, pl.smem};
  {
    std::lock_guard<std::mutex> lk(g_sk_occ_mu);
    auto it = g_sk_occ[dev].find(key);
    if (it != g_sk_occ[dev].end()) return it->second;
  }
  int n = 0;
  cudaError_t e = cudaErrorInvalidValue;
  switch (pl.C) {
    case 1: e = skinny_occupancy<1>(pl.smem, &n); break;
    case 2: e = skinny_occupancy<2>(pl.smem, &n); break;
    case 4: e = skinny_occupancy<4>(pl.smem, &n); break;
    case 8: e = skinny_occupancy<8>(pl.smem, &n); break;
    case 16: e = skinny_occupancy<16>(pl.smem, &n); break;
    default: break;
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  std::lock_guard<std::mutex> lk(g_sk_occ_mu);
  g_sk_occ[dev][key] = n;
  return n;
}

bool skinny_choose(int64_t M, int64_t N, int64_t K, int r, SkinnyPlan &pl) {
  const int64_t macro = (K + kSkMacro - 1) / kSkMacro;
  const int64_t row_tiles = N / kSkRows;
  int64_t best_waves = 0;
  bool found = false;
  for (const int C : {8, 4, 16, 2, 1}) {
    if (C > 1 && C > macro) continue;   // a slice holds at least one 256-value macro-block
    SkinnyPlan cand{};
    if (!skinny_plan_for(static_cast<int>(M), static_cast<int>(K), r, C, kSkSmemLimit, cand)) continue;
    const int resident = skinny_resident(cand);
    if (resident <= 0) continue;
    const int64_t waves = (row_tiles + resident - 1) / resident;
    if (!found || waves < best_waves) {
      pl = cand;
      best_waves = waves;
      found = true;
    }
  }
  return found;
}

// xa_src is the adapter input (X, or X (.) keep under dropout) and xa_scale the factor of
// its product (1, or 1/(1-p)).
qlora_status launch_skinny(const uint16_t *X, int64_t M, const qlora_nf4_t *Wq, const uint16_t *A,
                           const uint16_t *B, int r, float s, uint16_t *Y, float *xa,
                           const SkinnyPlan &pl, cudaStream_t st, const uint16_t *xa_src, float xa_scale) {
  const int64_t N = Wq->rows, K = Wq->cols;
  // 1. XA = X A by one cluster; it lets the dependent launch below start at once
  {
    XaParams xp{};
    xp.X = xa_src;
    xp.scale = xa_scale;
    xp.A = A;
    xp.xa = xa;
    xp.M = static_cast<int>(M);
    xp.K = static_cast<int>(K);
    xp.r = r;
    xp.kx = static_cast<int>((K / kXaCluster + 15) / 16 * 16);
    xp.chunk = xa_chunk_rows(r);
    xp.limit_ns = static_cast<uint64_t>(g_wait_limit_us.load()) * 1000ull;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(kXaCluster, 1, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = static_cast<size_t>(xa_smem_bytes(r));
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kXaCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    LaunchTimer lt(QLORA_K_PROJECT, st);
    const qlora_status e = cuda_status(cudaLaunchKernelEx(&cfg, qlora_xa_kernel, xp));
    if (e != QLORA_OK) return e;
  }
  // 2. the weight pass, a programmatic dependent of the XA launch
  SkinnyParams p{};
  p.X = X;
  p.codes = Wq->codes;
  p.q8 = Wq->q8;
  p.step = Wq->step;
  p.B = B;
  p.xa = xa;
  p.Y = Y;
  p.M = static_cast<int>(M);
  p.K = static_cast<int>(K);
  p.N = static_cast<int>(N);
  p.r = r;
  p.ks = pl.ks;
  p.xpitch = pl.xpitch;
  p.off_b = pl.off_b;
  p.off_x = pl.off_x;
  p.off_part = pl.off_part;
  p.off_xa = pl.off_xa;
  p.off_bar = pl.off_bar;
  p.limit_ns = static_cast<uint64_t>(g_wait_limit_us.load()) * 1000ull;
  p.s = s;
  std::memcpy(p.levels, nf4_tables().levels, sizeof(p.levels));
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(pl.C), static_cast<unsigned>(N / kSkRows), 1);
  cfg.blockDim = dim3(kSkThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(pl.smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(pl.C);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  LaunchTimer lt(QLORA_K_SKINNY, st);
  const int R = kSkRows / pl.C;
  CUtensorMap tm_codes, tm_b;
  if (!make_map_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq->codes, K / 2, N, K / 2, kSkMacro / 2,
                   kSkRows, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, N, r, 2 * N, R, r, CU_TENSOR_MAP_SWIZZLE_NONE))
    return QLORA_ERR_CUDA;
  switch (pl.C) {
    case 1: return cuda_status(cudaLaunchKernelEx(&cfg, qlora_skinny_kernel<1>, tm_codes, tm_b, p));
    case 2: return cuda_status(cudaLaunchKernelEx(&cfg, qlora_skinny_kernel<2>, tm_codes, tm_b, p));
    case 4: return cuda_status(cudaLaunchKernelEx(&cfg, qlora_skinny_kernel<4>, tm_codes, tm_b, p));
    case 8: return cuda_status(cudaLaunchKernelEx(&cfg, qlora_skinny_kernel<8>, tm_codes, tm_b, p));
    case 16: return cuda_status(cudaLaunchKernelEx(&cfg, qlora_skinny_kernel<16>, tm_codes, tm_b, p));
    default: return QLORA_ERR_UNSUPPORTED_SHAPE;
  }
}

// One fused GEMM launch.  MODE fwd: Y = X deq(W)^T + LoRA; MODE dx: dX = dY deq(W) + LoRA.
// `sp` is the launch's split scratch, its counters already cleared in stream order.
// keep (dX only, may be null): the bit-packed dropout mask of the adapter input, with
// keep_scale = 1/(1-p).
template <int MODE>
qlora_status launch_gemm(const uint16_t *act, int64_t M, const qlora_nf4_t *Wq,
                         const uint16_t *lora_act_hl, const uint16_t *lora_w, int r,
                         uint16_t *out, const SplitScratch &sp, const GemmUnits &u, cudaStream_t st,
                         const uint8_t *keep = nullptr, float keep_scale = 1.0f) {
  const int64_t N = Wq->rows, K = Wq->cols;
  const int64_t n_out = (MODE == kModeFwd) ? N : K;
  const int64_t contraction = (MODE == kModeFwd) ? K : N;
  const bool pair = sp.g.pair;
  if (pair && !gemm_pairable(n_out, u)) return QLORA_ERR_WORKSPACE;
  // a pair's CTAs each load half of the 256-token activation tile
  const int b_rows = pair ? kBN / 2 : kBN;
  CUtensorMap tm_act, tm_codes, tm_lora;
  if (!make_map_2d(&tm_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act, contraction, M, contraction * 2,
                   kBK, b_rows, CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  if (MODE == kModeFwd) {
    if (!make_map_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq->codes, K / 2, N, K / 2, 32, kWT,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
      return QLORA_ERR_CUDA;
  } else {
    if (!make_map_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq->codes, K / 2, N, K / 2, 64, 64,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
      return QLORA_ERR_CUDA;
  }
  if (!make_map_2d(&tm_lora, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora_act_hl, 2 * r, M, 4 * r, kBK,
                   b_rows, CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;

  GemmParams p{};
  p.M = static_cast<int>(M);
  p.n_out = static_cast<int>(n_out);
  p.num_m_tiles = static_cast<int>((M + kBN - 1) / kBN);
  p.num_w_tiles = static_cast<int>(n_out / (pair ? 2 * kWT : kWT));
  {
    // token tiles per raster group.  A packed weight that fits the budget stays in L2
    // while every token tile sweeps it (one group of one); a larger one is swept by
    // groups of as many activation tiles as fit the budget, each weight tile read once
    // per group.
    constexpr int64_t budget = 40ll << 20;   // bytes of L2 for the group's activation tiles
    const int64_t w_bytes = n_out * contraction / 2;
    const int64_t act_tile = static_cast<int64_t>(kBN) * contraction * 2;
    int64_t g = (w_bytes <= budget) ? 1 : budget / act_tile;
    if (g < 1) g = 1;
    if (g > p.num_m_tiles) g = p.num_m_tiles;
    p.group_m = static_cast<int>(g);
  }
  p.kb_main = static_cast<int>(contraction / kBK);
  p.kb_lora = (2 * r + kBK - 1) / kBK;
  p.r = r;
  p.lora_ld = (MODE == kModeFwd) ? static_cast<int>(N) : r;
  p.KB = static_cast<int>(K / 64);
  p.q8 = Wq->q8;
  p.step = Wq->step;
  p.lora_w = lora_w;
  p.out = out;
  p.limit_ns = static_cast<uint64_t>(g_wait_limit_us.load()) * 1000ull;
  const Nf4Tables &T = nf4_tables();
  std::memcpy(p.levels, T.levels, sizeof(p.levels));
  const int tiles = p.num_m_tiles * p.num_w_tiles;
  const int units = pair ? u.pairs : u.ctas;
  const int grid_units = tiles < units ? tiles : units;
  const GemmSplit g = gemm_split(M, n_out, contraction, u, pair);
  if (g.count != sp.g.count || g.base != sp.g.base) return QLORA_ERR_WORKSPACE;
  p.split_base = g.base;
  p.split_count = g.count;
  p.kb_mid = p.kb_main / 2;
  p.scratch = sp.partial;
  p.flags = sp.flags;
  p.keep32 = (MODE == kModeDx) ? reinterpret_cast<const uint32_t *>(keep) : nullptr;
  p.keep_scale = keep_scale;
  LaunchTimer lt(MODE == kModeFwd ? QLORA_K_GEMM_FWD : QLORA_K_GEMM_DX, st);
  if (!pair) {
    qlora_gemm_kernel<MODE, false><<<grid_units, kGemmThreads, kGemmSmemBytes, st>>>(tm_act, tm_codes, tm_lora, p);
    return cuda_status(cudaGetLastError());
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * grid_units), 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = kGemmSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cuda_status(cudaLaunchKernelEx(&cfg, qlora_gemm_kernel<MODE, true>, tm_act, tm_codes, tm_lora, p));
}

// ------------------------------------------------------------------ the linear layer
// keep (nullable): bit-packed keep mask of the adapter input X [M, K] (element m K + k
// in bit (m K + k) mod 8 of byte (m K + k) / 8); kept values are scaled by 1/(1-p).
qlora_status check_dropout(const uint8_t *keep, float p) {
  if (!keep) return QLORA_OK;
  if (!(p >= 0.0f && p < 1.0f)) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(keep)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

size_t mask_workspace(int64_t M, int64_t K) { return align256(static_cast<size_t>(M) * K * 2); }

qlora_status linear_fwd_impl(const uint16_t *X, int64_t M, const qlora_nf4_t *Wq, const uint16_t *A,
                             const uint16_t *B, int r, float s, const uint8_t *keep, float drop_p,
                             uint16_t *Y, float *XA_out, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
  qlora_status st = check_nf4(Wq);
  if (st != QLORA_OK) return st;
  if (!X || !A || !B || !Y) return QLORA_ERR_INVALID_ARG;
  if ((st = check_linear_shape(M, Wq, r)) != QLORA_OK) return st;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y) ||
      (XA_out && !aligned16(XA_out)) || (workspace && !aligned16(workspace)))
    return QLORA_ERR_MISALIGNED;
  if (!(s == s)) return QLORA_ERR_INVALID_ARG;
  if ((st = check_dropout(keep, drop_p)) != QLORA_OK) return st;
  DeviceInfo *d = nullptr;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  const int64_t N = Wq->rows, K = Wq->cols;
  const size_t need = fwd_workspace(M, N, K, r, d->units) + (keep ? mask_workspace(M, K) : 0);
  if (!workspace || workspace_bytes < need) return QLORA_ERR_WORKSPACE;
  Workspace ws{static_cast<char *>(workspace), 0, workspace_bytes};
  // the adapter input: X, or X (.) keep under dropout (its products then carry 1/(1-p))
  const uint16_t *xin = X;
  const float xscale = keep ? 1.0f / (1.0f - drop_p) : 1.0f;
  if (keep) {
    uint16_t *Xd = static_cast<uint16_t *>(ws.take(static_cast<size_t>(M) * K * 2));
    if (!Xd) return QLORA_ERR_WORKSPACE;
    if ((st = launch_mask(X, keep, M * K, Xd, d->sms, stream)) != QLORA_OK) return st;
    xin = Xd;
  }
  if (M <= kSkinnyMaxTokens) {
    SkinnyPlan pl{};
    if (skinny_choose(M, N, K, r, pl)) {
      float *xa = XA_out ? XA_out : static_cast<float *>(ws.take(static_cast<size_t>(M) * r * 4));
      if (!xa) return QLORA_ERR_WORKSPACE;
      return launch_skinny(X, M, Wq, A, B, r, s, Y, xa, pl, stream, xin, xscale);
    }
  }

  uint16_t *AT = static_cast<uint16_t *>(ws.take(static_cast<size_t>(r) * K * 2));
  uint16_t *hl = static_cast<uint16_t *>(ws.take(static_cast<size_t>(M) * 2 * r * 2));
  float *xa = XA_out ? XA_out : static_cast<float *>(ws.take(static_cast<size_t>(M) * r * 4));
  SplitScratch sp;
  if (!AT || !hl || !xa || !take_split(ws, gemm_plan(M, N, K, d->units), sp)) return QLORA_ERR_WORKSPACE;
  // XA = X A (fp32) and s*XA as bf16 hi|lo, the activation side of the LoRA K-steps;
  // the projection also clears the GEMM's split counters
  if ((st = launch_transpose(A, K, r, AT, d->sms, stream)) != QLORA_OK) return st;
  if ((st = launch_projection(xin, M, K, AT, r, s, xa, hl, nullptr, d->sms, stream, &sp, xscale)) != QLORA_OK)
    return st;
  return launch_gemm<kModeFwd>(X, M, Wq, hl, B, r, Y, sp, d->units, stream);
}

qlora_status linear_bwd_impl(const uint16_t *dY, const uint16_t *X, const float *XA, int64_t M,
                             const qlora_nf4_t *Wq, const uint16_t *A, const uint16_t *B, int r, float s,
                             const uint8_t *keep, float drop_p, int accumulate, uint16_t *dX, float *dA,
                             float *dB, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
  qlora_status st = check_nf4(Wq);
  if (st != QLORA_OK) return st;
  if (!dY || !X || !A || !B || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if ((st = check_linear_shape(M, Wq, r)) != QLORA_OK) return st;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(dA) ||
      !aligned16(dB) || (dX && !aligned16(dX)) || (XA && !aligned16(XA)) ||
      (workspace && !aligned16(workspace)))
    return QLORA_ERR_MISALIGNED;
  if (!(s == s)) return QLORA_ERR_INVALID_ARG;
  if ((st = check_dropout(keep, drop_p)) != QLORA_OK) return st;
  DeviceInfo *d = nullptr;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  const int64_t N = Wq->rows, K = Wq->cols;
  const size_t need = bwd_workspace(M, N, K, r, d->units) + (keep ? mask_workspace(M, K) : 0);
  if (!workspace || workspace_bytes < need) return QLORA_ERR_WORKSPACE;
  Workspace ws{static_cast<char *>(workspace), 0, workspace_bytes};
  const uint16_t *xin = X;
  const float xscale = keep ? 1.0f / (1.0f - drop_p) : 1.0f;
  if (keep) {
    uint16_t *Xd = static_cast<uint16_t *>(ws.take(static_cast<size_t>(M) * K * 2));
    if (!Xd) return QLORA_ERR_WORKSPACE;
    if ((st = launch_mask(X, keep, M * K, Xd, d->sms, stream)) != QLORA_OK) return st;
    xin = Xd;
  }
  const size_t hlT_bytes = static_cast<size_t>(2 * r) * pad8(M) * 2;
  uint16_t *AT = static_cast<uint16_t *>(ws.take(static_cast<size_t>(r) * K * 2));
  float *G = static_cast<float *>(ws.take(static_cast<size_t>(M) * r * 4));
  uint16_t *ghl = static_cast<uint16_t *>(ws.take(static_cast<size_t>(M) * 2 * r * 2));
  uint16_t *ghlT = static_cast<uint16_t *>(ws.take(hlT_bytes));
  uint16_t *xahlT = static_cast<uint16_t *>(ws.take(hlT_bytes));
  float *xa_ws = static_cast<float *>(ws.take(static_cast<size_t>(M) * r * 4));
  SplitScratch sp;
  if (!AT || !G || !ghl || !ghlT || !xahlT || !xa_ws) return QLORA_ERR_WORKSPACE;
  if (dX && !take_split(ws, gemm_plan(M, K, N, d->units), sp)) return QLORA_ERR_WORKSPACE;
  // s*XA hi|lo transposed [2r, M] (from the saved XA, or recomputed from the adapter input)
  if (XA) {
    if ((st = launch_hilo_t(XA, M, r, s, xahlT, d->sms, stream)) != QLORA_OK) return st;
  } else {
    if ((st = launch_transpose(A, K, r, AT, d->sms, stream)) != QLORA_OK) return st;
    if ((st = launch_projection(xin, M, K, AT, r, s, xa_ws, nullptr, xahlT, d->sms, stream, nullptr, xscale)) !=
        QLORA_OK)
      return st;
  }
  // G = dY B^T; s*G hi|lo in [M, 2r] (dX GEMM) and [2r, M] (dA); clears the dX GEMM's
  // split counters
  if ((st = launch_projection(dY, M, N, B, r, s, G, ghl, ghlT, d->sms, stream, &sp)) != QLORA_OK) return st;
  if (dX) {
    if ((st = launch_gemm<kModeDx>(dY, M, Wq, ghl, A, r, dX, sp, d->units, stream, keep, xscale)) != QLORA_OK)
      return st;
  }
  // dA = (1/(1-p)) X_kept^T (s G)  [K, r];  dB = (s XA)^T dY  [r, N]
  return launch_grads(xin, dY, M, K, N, ghlT, xahlT, r, dA, dB, d->sms, stream, xscale, accumulate);
}

}  // namespace

// ==================================================================== C ABI
extern "C" {

int qlora_version(void) { return kVersion; }

const char *qlora_status_string(qlora_status s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case QLORA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_TIMEOUT: return "device wait timed out";
    case QLORA_ERR_DEVICE_CHECK: return "device-side check failed";
    case QLORA_ERR_WORKSPACE: return "workspace missing or too small";
    case QLORA_ERR_NO_DEVICE: return "no sm_100 device";
  }
  return "unknown status";
}

void qlora_nf4_levels(float out[16]) {
  const Nf4Tables &T = nf4_tables();
  for (int i = 0; i < 16; ++i) out[i] = T.levels[i];
}

size_t qlora_nf4_bytes(int64_t rows, int64_t cols, size_t *codes_bytes, size_t *q8_bytes,
                       size_t *step_bytes) {
  if (rows <= 0 || cols <= 0) {
    if (codes_bytes) *codes_bytes = 0;
    if (q8_bytes) *q8_bytes = 0;
    if (step_bytes) *step_bytes = 0;
    return 0;
  }
  const uint64_t n = static_cast<uint64_t>(rows) * static_cast<uint64_t>(cols);
  const uint64_t nb = (n + 63) / 64;
  const size_t c = static_cast<size_t>((n + 1) / 2);
  const size_t q = static_cast<size_t>(nb);
  const size_t s = static_cast<size_t>(4 * ((nb + 255) / 256));
  if (codes_bytes) *codes_bytes = c;
  if (q8_bytes) *q8_bytes = q;
  if (step_bytes) *step_bytes = s;
  return c + q + s;
}

size_t qlora_nf4_single_bytes(int64_t rows, int64_t cols, size_t *codes_bytes, size_t *step_bytes) {
  if (rows <= 0 || cols <= 0) {
    if (codes_bytes) *codes_bytes = 0;
    if (step_bytes) *step_bytes = 0;
    return 0;
  }
  const uint64_t n = static_cast<uint64_t>(rows) * static_cast<uint64_t>(cols);
  const size_t c = static_cast<size_t>((n + 1) / 2), s = static_cast<size_t>(4 * ((n + 63) / 64));
  if (codes_bytes) *codes_bytes = c;
  if (step_bytes) *step_bytes = s;
  return c + s;
}

qlora_status qlora_nf4_quantize(const uint16_t *W, int64_t rows, int64_t cols,
                                const qlora_nf4_t *out, qlora_stream_t stream) {
  if (!W || !out || rows <= 0 || cols <= 0) return QLORA_ERR_INVALID_ARG;
  if (out->rows != rows || out->cols != cols) return QLORA_ERR_INVALID_ARG;
  qlora_status st = check_nf4(out);
  if (st != QLORA_OK) return st;
  if (!aligned16(W)) return QLORA_ERR_MISALIGNED;
  DeviceInfo *d = nullptr;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  const Nf4Tables &T = nf4_tables();
  if (!T.ok) return QLORA_ERR_DEVICE_CHECK;
  QuantTables tab;
  for (int i = 0; i < kQuantBins256; ++i) {
    tab.bins[i].t = 2.0f;                         // inert: reachable only from non-finite blocks
    tab.bins[i].c = 0;
  }
  for (int j = -32; j <= 32; ++j) tab.bins[j + 32] = T.bins[j & (kQuantBins - 1)];
  std::memcpy(tab.rcp, T.rcp, sizeof(tab.rcp));
  const int64_t n = rows * cols;
  const int64_t groups = (n + kGroupElems - 1) / kGroupElems;
  if (groups > 0x7FFFFFFFll) return QLORA_ERR_UNSUPPORTED_SHAPE;
  LaunchTimer lt(QLORA_K_QUANTIZE, stream);
  const int64_t ctas = static_cast<int64_t>(d->sms) * kQuantCtasPerSm;
  const int64_t grid = groups < ctas ? groups : ctas;
  nf4_quantize_kernel<<<static_cast<unsigned>(grid > 0 ? grid : 1), kQuantThreads, kQuantSmemBytes, stream>>>(
      W, n, out->codes, out->q8, out->step, tab, static_cast<uint64_t>(g_wait_limit_us.load()) * 1000ull);
  return cuda_status(cudaGetLastError());
}

qlora_status qlora_nf4_dequant(const qlora_nf4_t *Wq, uint16_t *W_out, qlora_stream_t stream) {
  qlora_status st = check_nf4(Wq);
  if (st != QLORA_OK) return st;
  if (!W_out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W_out)) return QLORA_ERR_MISALIGNED;
  DeviceInfo *d = nullptr;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  Levels lv;
  std::memcpy(lv.v, nf4_tables().levels, sizeof(lv.v));
  const int64_t n = Wq->rows * Wq->cols;
  int64_t units = n >> 4;
  int64_t grid = (units + 255) / 256;
  if (grid > static_cast<int64_t>(d->sms) * 16) grid = static_cast<int64_t>(d->sms) * 16;
  if (grid < 1) grid = 1;
  LaunchTimer lt(QLORA_K_DEQUANT, stream);
  nf4_dequant_kernel<<<static_cast<unsigned>(grid), 256, 0, stream>>>(Wq->codes, Wq->q8, Wq->step, n,
                                                                      W_out, lv);
  return cuda_status(cudaGetLastError());
}

size_t qlora_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
  if (M < 1 || N < 1 || K < 1 || r < 1) return 0;
  GemmUnits u;
  DeviceInfo *d = nullptr;
  if (device_info(&d) == QLORA_OK) u = d->units;
  const size_t f = fwd_workspace(M, N, K, r, u), b = bwd_workspace(M, N, K, r, u);
  return f > b ? f : b;
}

size_t qlora_linear_dropout_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) {
  const size_t b = qlora_linear_workspace_bytes(M, N, K, r);
  return b ? b + mask_workspace(M, K) : 0;
}

qlora_status qlora_linear_fwd(const uint16_t *X, int64_t M, const qlora_nf4_t *Wq,
                              const uint16_t *A, const uint16_t *B, int r, float s, uint16_t *Y,
                              float *XA_out, void *workspace, size_t workspace_bytes,
                              qlora_stream_t stream) {
  return linear_fwd_impl(X, M, Wq, A, B, r, s, nullptr, 0.0f, Y, XA_out, workspace, workspace_bytes, stream);
}

qlora_status qlora_linear_fwd_ex(const uint16_t *X, int64_t M, const qlora_nf4_t *Wq,
                                 const uint16_t *A, const uint16_t *B, int r, float s,
                                 const uint8_t *keep, float dropout_p, uint16_t *Y, float *XA_out,
                                 void *workspace, size_t workspace_bytes, qlora_stream_t stream) {
  return linear_fwd_impl(X, M, Wq, A, B, r, s, keep, dropout_p, Y, XA_out, workspace, workspace_bytes, stream);
}

qlora_status qlora_linear_bwd(const uint16_t *dY, const uint16_t *X, const float *XA, int64_t M,
                              const qlora_nf4_t *Wq, const uint16_t *A, const uint16_t *B, int r,
                              float s, uint16_t *dX, float *dA, float *dB, void *workspace,
                              size_t workspace_bytes, qlora_stream_t stream) {
  return linear_bwd_impl(dY, X, XA, M, Wq, A, B, r, s, nullptr, 0.0f, 0, dX, dA, dB, workspace,
                         workspace_bytes, stream);
}

qlora_status qlora_linear_bwd_ex(const uint16_t *dY, const uint16_t *X, const float *XA, int64_t M,
                                 const qlora_nf4_t *Wq, const uint16_t *A, const uint16_t *B, int r,
                                 float s, const uint8_t *keep, float dropout_p, int accumulate,
                                 uint16_t *dX, float *dA, float *dB, void *workspace,
                                 size_t workspace_bytes, qlora_stream_t stream) {
  return linear_bwd_impl(dY, X, XA, M, Wq, A, B, r, s, keep, dropout_p, accumulate, dX, dA, dB, workspace,
                         workspace_bytes, stream);
}

qlora_status qlora_nf4_merge(const qlora_nf4_t *Wq, const uint16_t *W16, int64_t N, int64_t K,
                             const uint16_t *A, const uint16_t *B, int r, float s, uint16_t *W_out,
                             qlora_stream_t stream) {
  if ((Wq == nullptr) == (W16 == nullptr) || !A || !B || !W_out) return QLORA_ERR_INVALID_ARG;
  if (N < 1 || K < 1 || N > (1ll << 24) || K > (1ll << 24) || N * K > (1ll << 40)) return QLORA_ERR_INVALID_ARG;
  if (r < 8 || r > 128 || (r % 8) != 0 || !(s == s)) return QLORA_ERR_INVALID_ARG;
  if ((N % 8) != 0 || (K % 64) != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (Wq) {
    const qlora_status st = check_nf4(Wq);
    if (st != QLORA_OK) return st;
    if (Wq->rows != N || Wq->cols != K) return QLORA_ERR_INVALID_ARG;
  }
  if (!aligned16(A) || !aligned16(B) || !aligned16(W_out) || (W16 && !aligned16(W16)))
    return QLORA_ERR_MISALIGNED;
  DeviceInfo *d = nullptr;
  qlora_status st = device_info(&d);
  if (st != QLORA_OK) return st;
  MergeParams p{};
  if (Wq) {
    p.q8 = Wq->q8;
    p.step = Wq->step;
  }
  p.nf4 = Wq ? 1 : 0;
  p.N = static_cast<int>(N);
  p.K = static_cast<int>(K);
  p.stages = (r + 63) / 64;
  p.s = s;
  p.limit_ns = static_cast<uint64_t>(g_wait_limit_us.load()) * 1000ull;
  std::memcpy(p.levels, nf4_tables().levels, sizeof(p.levels));
  CUtensorMap tm_bt, tm_a, tm_base, tm_out;
  // B [r, N]: x = n (inner), y = j; A [K, r]: x = j (inner), y = k.  Boxes reach j = 64 per
  // stage; rows j >= r are outside the tensors and arrive as zeros.  The base: W16
  // [N, K] in boxes {64 k, 128 n}, or the packed codes [N, K/2 bytes] in boxes
  // {128 bytes, 128 n}; the output [N, K] in boxes {64 k, 128 n}; all 128B-swizzled.
  if (!make_map_2d(&tm_bt, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, N, r, N * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tm_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, r, K, r * 2, 64, kMgCols, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_2d(&tm_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W_out, K, N, K * 2, 64, kMgRows,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  const bool base_ok =
      Wq ? make_map_2d(&tm_base, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq->codes, K / 2, N, K / 2, 128, kMgRows,
                       CU_TENSOR_MAP_SWIZZLE_128B)
         : make_map_2d(&tm_base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W16, K, N, K * 2, 64, kMgRows,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (!base_ok) return QLORA_ERR_CUDA;
  dim3 grid(static_cast<unsigned>((K + kMgCols - 1) / kMgCols), static_cast<unsigned>((N + kMgRows - 1) / kMgRows));
  LaunchTimer lt(QLORA_K_MERGE, stream);
  nf4_merge_kernel<<<grid, kMgThreads, merge_smem_bytes(p.stages, Wq != nullptr), stream>>>(tm_bt, tm_a, tm_base,
                                                                                            tm_out, p);
  return cuda_status(cudaGetLastError());
}

qlora_status qlora_get_device_status(qlora_stream_t stream, uint32_t *flags) {
  if (!flags) return QLORA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return QLORA_ERR_CUDA;
  uint32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return QLORA_ERR_CUDA;
  *flags = v;
  if (v & kStatTimeout) return QLORA_ERR_TIMEOUT;
  if (v & (kStatNonFinite | kStatLayout)) return QLORA_ERR_DEVICE_CHECK;
  return QLORA_OK;
}

qlora_status qlora_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  if (on) {
    if (!prof_ensure_events()) return QLORA_ERR_CUDA;
    g_prof.count = 0;
  }
  g_prof.on = on != 0;
  return QLORA_OK;
}

int qlora_profile_read(int max, int *kinds, float *ms) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  if (!g_prof.created) return 0;
  const long long n = g_prof.count;
  const long long first = n > QLORA_PROFILE_CAP ? n - QLORA_PROFILE_CAP : 0;
  int out = 0;
  for (long long i = first; i < n && out < max; ++i, ++out) {
    const int slot = static_cast<int>(i % QLORA_PROFILE_CAP);
    if (cudaEventSynchronize(g_prof.ev[2 * slot + 1]) != cudaSuccess) return -1;
    float t = 0.f;
    if (cudaEventElapsedTime(&t, g_prof.ev[2 * slot], g_prof.ev[2 * slot + 1]) != cudaSuccess) return -1;
    if (kinds) kinds[out] = g_prof.kind[slot];
    if (ms) ms[out] = t;
  }
  return static_cast<int>(n > 0x7FFFFFFF ? 0x7FFFFFFF : n);
}

uint32_t qlora_set_wait_limit_us(uint32_t limit_us) {
  if (limit_us < 1) limit_us = 1;
  return g_wait_limit_us.exchange(limit_us);
}

int qlora_set_gemm_pairing(int enable) { return g_gemm_pairing.exchange(enable ? 1 : 0); }

qlora_status qlora_gemm_units(int *ctas, int *pairs) {
  DeviceInfo *d = nullptr;
  const qlora_status st = device_info(&d);
  if (st != QLORA_OK) return st;
  if (ctas) *ctas = d->units.ctas;
  if (pairs) *pairs = d->units.pairs;
  return QLORA_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ wait self-test
namespace {
__global__ void selftest_wait_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // nothing ever arrives on it
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const Waiter w{&abort_flag, limit_ns};
  if (threadIdx.x == 0) (void)wait_bar(&bar, 0, w);
}
}  // namespace

extern "C" qlora_status qlora_selftest_wait_timeout(uint32_t timeout_us, qlora_stream_t stream) {
  if (timeout_us < 1 || timeout_us > 10000000u) return QLORA_ERR_INVALID_ARG;
  DeviceInfo *d = nullptr;
  qlora_status st = device_info(&d);
  if (st != QLORA_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(timeout_us) * 1000ull);
  return cuda_status(cudaGetLastError());
}

// ------------------------------------------------------------------ forward without a workspace
// For callers that cannot allocate device memory (a plain host program linking only
// this library, or a runtime whose device memory is all planned up front): the
// forward's scratch comes from one file-scope device array instead of a caller
// workspace.  Every GPU that loads the library holds this array until exit.
namespace {
constexpr size_t kNoallocScratchBytes = QLORA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

struct NoallocSlot {
  bool ready = false;
  void *ptr = nullptr;
};
NoallocSlot g_noalloc_slot[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the array on the current device, looked up once per device
// (in host code the array's name is only a host-side stand-in, not a device address).
qlora_status noalloc_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return QLORA_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  NoallocSlot &slot = g_noalloc_slot[dev];
  if (!slot.ready) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return QLORA_ERR_CUDA;
    slot.ptr = p;
    slot.ready = true;
  }
  *out = slot.ptr;
  return QLORA_OK;
}
}  // namespace

extern "C" qlora_status qlora_linear_fwd_noalloc(const uint16_t *X, int64_t M, const qlora_nf4_t *Wq,
                                                 const uint16_t *A, const uint16_t *B, int r, float s,
                                                 uint16_t *Y, float *XA_out, qlora_stream_t stream) {
  qlora_status st = check_nf4(Wq);
  if (st != QLORA_OK) return st;
  if ((st = check_linear_shape(M, Wq, r)) != QLORA_OK) return st;
  DeviceInfo *d = nullptr;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  if (fwd_workspace(M, Wq->rows, Wq->cols, r, d->units) > kNoallocScratchBytes) return QLORA_ERR_WORKSPACE;
  void *scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != QLORA_OK) return st;
  return qlora_linear_fwd(X, M, Wq, A, B, r, s, Y, XA_out, scratch, kNoallocScratchBytes, stream);
}
