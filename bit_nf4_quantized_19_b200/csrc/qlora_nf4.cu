// libqlora_nf4.so: C ABI of the QLoRA NF4 frozen-base linear layer (see
// include/qlora_nf4.h for the contract of every entry point).
#include "qlora_nf4.h"

#include <atomic>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "gemm_kernel.cuh"
#include "lora_kernels.cuh"
#include "nf4_table.hpp"
#include "quant_kernels.cuh"

using namespace qlora;

namespace {

constexpr int kVersion = 100;  // 0.1.0
std::atomic<uint32_t> g_wait_limit_us{2000000u};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qlora_status cuda_status(cudaError_t e) { return e == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA; }

struct DeviceInfo {
  int sms = 0;
  int major = 0;
  bool gemm_attr_set = false;
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
    if (cudaFuncSetAttribute(qlora_gemm_kernel<kModeFwd>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGemmSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(qlora_gemm_kernel<kModeDx>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kGemmSmemBytes) != cudaSuccess)
      return QLORA_ERR_CUDA;
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

int grad_splits(int64_t M, int64_t C, int sms) {
  const int64_t ctiles = (C + kGradCT - 1) / kGradCT;
  int64_t splits = (2 * static_cast<int64_t>(sms) + ctiles - 1) / ctiles;
  const int64_t maxs = (M + kGradTM - 1) / kGradTM;
  if (splits > maxs) splits = maxs;
  if (splits < 1) splits = 1;
  if (splits > 64) splits = 64;
  return static_cast<int>(splits);
}

size_t fwd_workspace(int64_t M, int64_t N, int64_t K, int r) {
  size_t b = 0;
  b += align256(static_cast<size_t>(N) * (K / 64) * 4);        // expanded constants
  b += align256(static_cast<size_t>(M) * 2 * r * 2);           // s*XA hi/lo
  b += align256(static_cast<size_t>(M) * r * 4);               // XA when XA_out is NULL
  return b + 256;
}

size_t bwd_workspace(int64_t M, int64_t N, int64_t K, int r, int sms) {
  size_t b = 0;
  b += align256(static_cast<size_t>(N) * (K / 64) * 4);
  b += align256(static_cast<size_t>(M) * r * 4);               // G
  b += align256(static_cast<size_t>(M) * 2 * r * 2);           // s*G hi/lo
  b += align256(static_cast<size_t>(M) * r * 4);               // XA recomputed
  b += align256(static_cast<size_t>(M) * 2 * r * 2);           // its hi/lo (unused output)
  b += align256(static_cast<size_t>(grad_splits(M, K, sms)) * K * r * 4);
  b += align256(static_cast<size_t>(grad_splits(M, N, sms)) * N * r * 4);
  return b + 256;
}

qlora_status check_nf4(const qlora_nf4_t *Wq) {
  if (!Wq || !Wq->codes || !Wq->q8 || !Wq->step) return QLORA_ERR_INVALID_ARG;
  if (Wq->rows <= 0 || Wq->cols <= 0) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(Wq->codes) || !aligned16(Wq->q8) || !aligned16(Wq->step)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

qlora_status check_linear_shape(int64_t M, const qlora_nf4_t *Wq, int r) {
  if (M < 1 || M > (1ll << 30)) return QLORA_ERR_INVALID_ARG;
  if (r < 8 || r > 128 || (r % 8) != 0) return QLORA_ERR_INVALID_ARG;
  if (Wq->rows % 128 != 0 || Wq->cols % 128 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (Wq->rows > (1ll << 24) || Wq->cols > (1ll << 24)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  return QLORA_OK;
}

qlora_status launch_expand_scales(const qlora_nf4_t *Wq, float *S, cudaStream_t st, int sms) {
  const int N = static_cast<int>(Wq->rows), KB = static_cast<int>(Wq->cols / 64);
  const int64_t total = static_cast<int64_t>(N) * KB;
  int grid = static_cast<int>((total + 255) / 256);
  if (grid > sms * 8) grid = sms * 8;
  LaunchTimer lt(QLORA_K_EXPAND, st);
  nf4_expand_scales_kernel<<<grid, 256, 0, st>>>(Wq->q8, Wq->step, N, KB, S);
  return cuda_status(cudaGetLastError());
}

qlora_status launch_project(const uint16_t *P, int64_t M, int64_t C, const uint16_t *Q,
                            bool q_rows_are_c, int r, float s, float *out, uint16_t *hl,
                            cudaStream_t st) {
  const int grid = static_cast<int>((M + kProjTM - 1) / kProjTM);
  const size_t smem = (kProjTM * (kProjKC + 1) + kProjKC * r) * sizeof(float);
  LaunchTimer lt(QLORA_K_PROJECT, st);
  lora_project_kernel<<<grid, kProjThreads, smem, st>>>(P, static_cast<int>(M), static_cast<int>(C),
                                                        Q, q_rows_are_c ? 1 : 0, r, s, out, hl);
  return cuda_status(cudaGetLastError());
}

qlora_status launch_grad(const uint16_t *P, const float *F, int64_t M, int64_t C, int r, float s,
                         int layout, float *out, float *part, int sms, cudaStream_t st) {
  const int splits = grad_splits(M, C, sms);
  const int tps = static_cast<int>(((M + splits - 1) / splits + kGradTM - 1) / kGradTM * kGradTM);
  dim3 grid(static_cast<unsigned>((C + kGradCT - 1) / kGradCT), static_cast<unsigned>(splits));
  const size_t smem = (kGradTM * kGradCT + kGradTM * r) * sizeof(float);
  {
    LaunchTimer lt(QLORA_K_GRAD, st);
    lora_grad_partial_kernel<<<grid, kGradThreads, smem, st>>>(P, F, static_cast<int>(M),
                                                               static_cast<int>(C), r, tps, part);
  }
  if (cudaGetLastError() != cudaSuccess) return QLORA_ERR_CUDA;
  int rgrid = static_cast<int>((C * r + 255) / 256);
  if (rgrid > sms * 8) rgrid = sms * 8;
  LaunchTimer lt(QLORA_K_GRAD_REDUCE, st);
  lora_grad_reduce_kernel<<<rgrid, 256, 0, st>>>(part, splits, static_cast<int>(C), r, s, layout, out);
  return cuda_status(cudaGetLastError());
}

// One fused GEMM launch.  MODE fwd: Y = X deq(W)^T + LoRA; MODE dx: dX = dY deq(W) + LoRA.
template <int MODE>
qlora_status launch_gemm(const uint16_t *act, int64_t M, const qlora_nf4_t *Wq, const float *S,
                         const uint16_t *lora_act_hl, const uint16_t *lora_w, int r,
                         uint16_t *out, int sms, cudaStream_t st) {
  const int64_t N = Wq->rows, K = Wq->cols;
  const int64_t contraction = (MODE == kModeFwd) ? K : N;
  CUtensorMap tm_act, tm_codes, tm_scale, tm_lora;
  if (!make_map_2d(&tm_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act, contraction, M, contraction * 2,
                   kBK, kBN, CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;
  if (MODE == kModeFwd) {
    if (!make_map_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq->codes, K / 2, N, K / 2, 32, kWT,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d(&tm_scale, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, S, N, K / 64, N * 4, kWT, 1,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
      return QLORA_ERR_CUDA;
  } else {
    if (!make_map_2d(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, Wq->codes, K / 2, N, K / 2, 64, 64,
                     CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d(&tm_scale, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, S, N, K / 64, N * 4, 64, 2,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
      return QLORA_ERR_CUDA;
  }
  if (!make_map_2d(&tm_lora, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lora_act_hl, 2 * r, M, 4 * r, kBK,
                   kBN, CU_TENSOR_MAP_SWIZZLE_128B))
    return QLORA_ERR_CUDA;

  GemmParams p{};
  p.M = static_cast<int>(M);
  p.n_out = static_cast<int>((MODE == kModeFwd) ? N : K);
  p.num_m_tiles = static_cast<int>((M + kBN - 1) / kBN);
  p.num_w_tiles = static_cast<int>(((MODE == kModeFwd) ? N : K) / kWT);
  p.kb_main = static_cast<int>(contraction / kBK);
  p.kb_lora = (2 * r + kBK - 1) / kBK;
  p.r = r;
  p.lora_ld = (MODE == kModeFwd) ? static_cast<int>(N) : r;
  p.lora_w = lora_w;
  p.out = out;
  p.limit_ns = static_cast<uint64_t>(g_wait_limit_us.load()) * 1000ull;
  const Nf4Tables &T = nf4_tables();
  std::memcpy(p.levels, T.levels, sizeof(p.levels));
  const int tiles = p.num_m_tiles * p.num_w_tiles;
  const int grid = tiles < sms ? tiles : sms;
  LaunchTimer lt(MODE == kModeFwd ? QLORA_K_GEMM_FWD : QLORA_K_GEMM_DX, st);
  qlora_gemm_kernel<MODE><<<grid, kGemmThreads, kGemmSmemBytes, st>>>(tm_act, tm_codes, tm_scale,
                                                                      tm_lora, p);
  return cuda_status(cudaGetLastError());
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
  std::memcpy(tab.bins, T.bins, sizeof(tab.bins));
  const int64_t n = rows * cols;
  const int64_t groups = (n + kGroupElems - 1) / kGroupElems;
  if (groups > 0x7FFFFFFFll) return QLORA_ERR_UNSUPPORTED_SHAPE;
  LaunchTimer lt(QLORA_K_QUANTIZE, stream);
  nf4_quantize_kernel<<<static_cast<unsigned>(groups), 256, 0, stream>>>(W, n, out->codes, out->q8,
                                                                         out->step, tab);
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
  int sms = 148;
  DeviceInfo *d = nullptr;
  if (device_info(&d) == QLORA_OK) sms = d->sms;
  const size_t f = fwd_workspace(M, N, K, r), b = bwd_workspace(M, N, K, r, sms);
  return f > b ? f : b;
}

qlora_status qlora_linear_fwd(const uint16_t *X, int64_t M, const qlora_nf4_t *Wq,
                              const uint16_t *A, const uint16_t *B, int r, float s, uint16_t *Y,
                              float *XA_out, void *workspace, size_t workspace_bytes,
                              qlora_stream_t stream) {
  qlora_status st = check_nf4(Wq);
  if (st != QLORA_OK) return st;
  if (!X || !A || !B || !Y) return QLORA_ERR_INVALID_ARG;
  if ((st = check_linear_shape(M, Wq, r)) != QLORA_OK) return st;
  if (!aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(Y) ||
      (XA_out && !aligned16(XA_out)) || (workspace && !aligned16(workspace)))
    return QLORA_ERR_MISALIGNED;
  if (!(s == s)) return QLORA_ERR_INVALID_ARG;
  DeviceInfo *d = nullptr;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  const int64_t N = Wq->rows, K = Wq->cols;
  if (!workspace || workspace_bytes < fwd_workspace(M, N, K, r)) return QLORA_ERR_WORKSPACE;
  Workspace ws{static_cast<char *>(workspace), 0, workspace_bytes};
  float *S = static_cast<float *>(ws.take(static_cast<size_t>(N) * (K / 64) * 4));
  uint16_t *hl = static_cast<uint16_t *>(ws.take(static_cast<size_t>(M) * 2 * r * 2));
  float *xa = XA_out ? XA_out : static_cast<float *>(ws.take(static_cast<size_t>(M) * r * 4));
  if (!S || !hl || !xa) return QLORA_ERR_WORKSPACE;
  if ((st = launch_expand_scales(Wq, S, stream, d->sms)) != QLORA_OK) return st;
  if ((st = launch_project(X, M, K, A, true, r, s, xa, hl, stream)) != QLORA_OK) return st;
  return launch_gemm<kModeFwd>(X, M, Wq, S, hl, B, r, Y, d->sms, stream);
}

qlora_status qlora_linear_bwd(const uint16_t *dY, const uint16_t *X, const float *XA, int64_t M,
                              const qlora_nf4_t *Wq, const uint16_t *A, const uint16_t *B, int r,
                              float s, uint16_t *dX, float *dA, float *dB, void *workspace,
                              size_t workspace_bytes, qlora_stream_t stream) {
  qlora_status st = check_nf4(Wq);
  if (st != QLORA_OK) return st;
  if (!dY || !X || !A || !B || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if ((st = check_linear_shape(M, Wq, r)) != QLORA_OK) return st;
  if (!aligned16(dY) || !aligned16(X) || !aligned16(A) || !aligned16(B) || !aligned16(dA) ||
      !aligned16(dB) || (dX && !aligned16(dX)) || (XA && !aligned16(XA)) ||
      (workspace && !aligned16(workspace)))
    return QLORA_ERR_MISALIGNED;
  if (!(s == s)) return QLORA_ERR_INVALID_ARG;
  DeviceInfo *d = nullptr;
  if ((st = device_info(&d)) != QLORA_OK) return st;
  const int64_t N = Wq->rows, K = Wq->cols;
  if (!workspace || workspace_bytes < bwd_workspace(M, N, K, r, d->sms)) return QLORA_ERR_WORKSPACE;
  Workspace ws{static_cast<char *>(workspace), 0, workspace_bytes};
  float *S = static_cast<float *>(ws.take(static_cast<size_t>(N) * (K / 64) * 4));
  float *G = static_cast<float *>(ws.take(static_cast<size_t>(M) * r * 4));
  uint16_t *ghl = static_cast<uint16_t *>(ws.take(static_cast<size_t>(M) * 2 * r * 2));
  float *xa_ws = static_cast<float *>(ws.take(static_cast<size_t>(M) * r * 4));
  uint16_t *xa_hl = static_cast<uint16_t *>(ws.take(static_cast<size_t>(M) * 2 * r * 2));
  float *partA = static_cast<float *>(ws.take(static_cast<size_t>(grad_splits(M, K, d->sms)) * K * r * 4));
  float *partB = static_cast<float *>(ws.take(static_cast<size_t>(grad_splits(M, N, d->sms)) * N * r * 4));
  if (!S || !G || !ghl || !xa_ws || !xa_hl || !partA || !partB) return QLORA_ERR_WORKSPACE;
  const float *xa = XA;
  if (!xa) {
    if ((st = launch_project(X, M, K, A, true, r, 1.0f, xa_ws, xa_hl, stream)) != QLORA_OK) return st;
    xa = xa_ws;
  }
  // G = dY B^T (and s*G hi/lo for the fused dX GEMM)
  if ((st = launch_project(dY, M, N, B, false, r, s, G, ghl, stream)) != QLORA_OK) return st;
  if (dX) {
    if ((st = launch_expand_scales(Wq, S, stream, d->sms)) != QLORA_OK) return st;
    if ((st = launch_gemm<kModeDx>(dY, M, Wq, S, ghl, A, r, dX, d->sms, stream)) != QLORA_OK)
      return st;
  }
  // dA = s X^T G  [K, r];  dB = s XA^T dY  [r, N]
  if ((st = launch_grad(X, G, M, K, r, s, 0, dA, partA, d->sms, stream)) != QLORA_OK) return st;
  return launch_grad(dY, xa, M, N, r, s, 1, dB, partB, d->sms, stream);
}

qlora_status qlora_get_device_status(qlora_stream_t stream, uint32_t *flags) {
  if (!flags) return QLORA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return QLORA_ERR_CUDA;
  uint32_t v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return QLORA_ERR_CUDA;
  *flags = v;
  if (v & kStatTimeout) return QLORA_ERR_TIMEOUT;
  if (v & kStatNonFinite) return QLORA_ERR_DEVICE_CHECK;
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
