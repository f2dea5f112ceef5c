/*
 * qlora_nf4.h -- C ABI of libqlora_nf4.so: the frozen-base linear layer of QLoRA
 * with blockwise NF4 weights and double-quantized block constants, on B200
 * (sm_100a).
 *
 * Method sources (page title, site, section):
 *   [NF4]   "QLoRA" (ai360xpert.com/papers/qlora), How It Works 1-2;
 *           "QLoRA: Efficient Finetuning of Quantized LLMs" (crackai.dev/papers/qlora),
 *           How It Works 1-2 and Training Flow.
 *   [STEPS] "QLoRA" (ozercemkelahmet.com/tools/qlora), How it works, Steps 1-6,
 *           and "A worked example".
 *   [SPLIT] "QLoRA" essay (fanfani.net/articles/qlora), section "The crucial split" and
 *           its display formula (4-bit W expanded to 16 bits, used in W_0 + BA).
 *
 * Conventions for every entry point
 *   - bf16 tensors are passed as pointers to IEEE bfloat16 bit patterns (uint16_t).
 *   - Every tensor pointer is DEVICE memory owned by the caller, row-major, dense.
 *     The library never allocates or frees memory; scratch space is passed in
 *     explicitly as `workspace` (size from qlora_linear_workspace_bytes).
 *   - Every pointer must be 16-byte aligned (QLORA_ERR_MISALIGNED otherwise).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  Argument, shape and alignment errors are reported synchronously
 *     before anything is launched; launch failures map to QLORA_ERR_CUDA.
 *   - Kernels never trap.  A device-side problem (a bounded wait that ran out, a
 *     non-finite weight block) sets a per-device status word that
 *     qlora_get_device_status() reads and clears.
 *   - Weight layout: W is [N, K] (out x in, the nn.Linear layout), flattened
 *     row-major for quantization.  X [M, K], Y [M, N], A [K, r], B [r, N].
 *   - Results are deterministic: every reduction runs in a fixed order.  The one
 *     atomic, the arrival counter of a GEMM tile split in two contraction halves,
 *     only decides which half adds the other's partial sum, and a sum of two
 *     fp32 values does not depend on their order.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t. */
typedef struct CUstream_st *qlora_stream_t;

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,       /* null pointer, bad size, r out of range      */
  QLORA_ERR_MISALIGNED = 2,        /* a pointer is not 16-byte aligned            */
  QLORA_ERR_UNSUPPORTED_SHAPE = 3, /* shape the fused GEMM does not cover         */
  QLORA_ERR_CUDA = 4,              /* a CUDA runtime/driver call failed            */
  QLORA_ERR_TIMEOUT = 5,           /* a device wait hit its time limit             */
  QLORA_ERR_DEVICE_CHECK = 6,      /* a device-side check failed (non-finite data) */
  QLORA_ERR_WORKSPACE = 7,         /* workspace missing or too small               */
  QLORA_ERR_NO_DEVICE = 8          /* no sm_100 device current                     */
} qlora_status;

/* Bits of the device status word (qlora_get_device_status). */
#define QLORA_DEVSTAT_TIMEOUT   1u
#define QLORA_DEVSTAT_NONFINITE 2u
#define QLORA_DEVSTAT_LAYOUT    4u   /* a kernel found its shared memory misplaced and did nothing */

/*
 * A quantized weight.  The struct itself lives in host memory; its three arrays
 * are device memory owned by the caller.  n = rows * cols values, flattened
 * row-major, are split into 64-value blocks ([STEPS] Step 1) and the block
 * constants into groups of 256 ([STEPS] Step 3).
 *   codes : ceil(n/2) bytes, two 4-bit codes per byte, element 2j in bits 0-3
 *           and element 2j+1 in bits 4-7; an odd tail leaves bits 4-7 zero.
 *   q8    : ceil(n/64) bytes, the 8-bit code of each block's absmax constant.
 *   step  : ceil(n/16384) floats, the fp32 second-level constant of each group;
 *           block b's constant is reconstructed as RN32(q8[b] * step[b/256]).
 * Single-level constants ([STEPS] Step 2 without Step 3: one 32-bit constant per
 * block, half a bit per value): q8 = NULL and step holds ceil(n/64) floats, block
 * b's absmax itself (4.5 bits per value in all).  Every entry point that takes a
 * qlora_nf4_t accepts either form; quantize writes the form its `out` names.
 */
typedef struct {
  uint8_t *codes;
  uint8_t *q8;
  float *step;
  int64_t rows; /* N (out features) */
  int64_t cols; /* K (in features)  */
} qlora_nf4_t;

/* Library version, major*10000 + minor*100 + patch. */
int qlora_version(void);

/* Human-readable name of a status code (static string). */
const char *qlora_status_string(qlora_status s);

/*
 * The 16 NF4 levels the library uses, sorted ascending, in `out[16]` (host
 * memory).  Built on the host from the inverse normal CDF at evenly spaced
 * probabilities in [0.5, (1-1/32 + 1-1/30)/2]: 8 positive levels, 7 negative,
 * one exact zero, normalised to [-1, 1] ([NF4]: levels at normal quantiles,
 * the same probability mass in every bin).
 */
void qlora_nf4_levels(float out[16]);

/*
 * Byte sizes of the three arrays of a rows x cols weight (any pointer may be
 * NULL).  Returns their sum: n/2 + n/64 + 4*n/16384 rounded up per array, i.e.
 * 4.126953125 bits per value when n is a multiple of 16384.
 */
size_t qlora_nf4_bytes(int64_t rows, int64_t cols, size_t *codes_bytes,
                       size_t *q8_bytes, size_t *step_bytes);

/* Byte sizes for single-level constants: codes as above, 4*ceil(n/64) of step. */
size_t qlora_nf4_single_bytes(int64_t rows, int64_t cols, size_t *codes_bytes, size_t *step_bytes);

/*
 * Quantize a bf16 weight W[rows, cols] ([STEPS] Steps 1-3, [NF4]).
 *   a_b  = max |w| over each 64-value block (the last block may be partial);
 *   code = nearest level to RN32(w / a_b) (ties to the lower index; a_b = 0 gives
 *          the zero level);
 *   c_g  = max a_b over each group of 256 blocks; step_g = RN32(c_g / 255);
 *   q8_b = min(255, round_half_even(RN32(a_b / step_g)))   (0 when c_g = 0).
 * With out->q8 = NULL (single-level constants) step[b] = a_b instead.
 * Any n = rows*cols >= 1.  `out` is a host struct whose arrays (sized by
 * qlora_nf4_bytes) receive the result; rows/cols in `out` must equal the
 * arguments.  Non-finite input values give unspecified codes and set
 * QLORA_DEVSTAT_NONFINITE.
 */
qlora_status qlora_nf4_quantize(const uint16_t *W, int64_t rows, int64_t cols,
                                const qlora_nf4_t *out, qlora_stream_t stream);

/*
 * Dequantize to bf16 ([STEPS] "A worked example" 4; [SPLIT]):
 *   W_out[i] = bf16_RN( RN32( L[code_i] * RN32(q8[b] * step[b/256]) ) ),
 * or bf16_RN( RN32( L[code_i] * step[b] ) ) with single-level constants.
 * W_out holds rows*cols bf16 values.
 */
qlora_status qlora_nf4_dequant(const qlora_nf4_t *Wq, uint16_t *W_out,
                               qlora_stream_t stream);

/*
 * Workspace bytes needed by qlora_linear_fwd / qlora_linear_bwd for an M-token
 * call on an N x K weight with LoRA rank r (the same size serves both calls).
 * The size depends on the current device's SM count (the fused GEMM splits the
 * tiles of its last round and keeps their partial sums here); query it on the
 * device the calls will run on.
 */
size_t qlora_linear_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);

/*
 * Forward of one adapted linear layer ([STEPS] Step 5, row-vector form):
 *   XA = X A                      (fp32 [M, r], written to XA_out if not NULL)
 *   Y  = X deq(W)^T + s * XA B    (bf16 [M, N])
 * deq(W) is formed on chip in bf16, exactly as qlora_nf4_dequant, and never
 * written to memory.  Accumulation is fp32.  s = alpha / r.
 * Shapes: M >= 1; N % 128 == 0; K % 128 == 0; r % 8 == 0, 8 <= r <= 128.
 * Execution: with M <= 16 tokens (and a contraction short enough for its
 * shared-memory plan) the call takes the few-token path: X A in one small
 * launch and the weight pass as its programmatic dependent.  Otherwise it
 * launches, in order on `stream`, the transpose of A, the rank-r projection
 * X A (which also clears the GEMM's split counters in the workspace) and the
 * fused dequant GEMM, which rebuilds the block constants RN32(q8 * step) on
 * chip.  All work is ordered after what `stream` already holds and before what
 * is enqueued to `stream` later; no other stream is used, and the call can be
 * captured into a CUDA graph and replayed with new inputs in the same buffers.
 */
qlora_status qlora_linear_fwd(const uint16_t *X, int64_t M, const qlora_nf4_t *Wq,
                              const uint16_t *A, const uint16_t *B, int r, float s,
                              uint16_t *Y, float *XA_out, void *workspace,
                              size_t workspace_bytes, qlora_stream_t stream);

/*
 * Forward with dropout on the adapter input ("QLoRA", ozercemkelahmet.com, "A code
 * example with common libraries": lora_dropout), otherwise as qlora_linear_fwd:
 *   Xd = X (.) keep / (1 - p)     (inverted dropout; the frozen path sees X itself)
 *   XA = Xd A                     (fp32 [M, r])
 *   Y  = X deq(W)^T + s * XA B
 * keep: device, bit-packed mask of X [M, K] drawn by the caller (Bernoulli(1 - p)
 * per element): element m K + k is kept when bit (m K + k) mod 8 of byte
 * (m K + k) / 8 is set; 16-byte aligned; M*K/8 bytes.  NULL: no dropout (p is then
 * ignored).  p in [0, 1).  X (.) keep is formed exactly (a zeroing) in the
 * workspace, whose size is then qlora_linear_dropout_workspace_bytes; the fp32
 * product is multiplied by 1/(1-p) before it is stored.
 */
qlora_status qlora_linear_fwd_ex(const uint16_t *X, int64_t M, const qlora_nf4_t *Wq,
                                 const uint16_t *A, const uint16_t *B, int r, float s,
                                 const uint8_t *keep, float dropout_p, uint16_t *Y, float *XA_out,
                                 void *workspace, size_t workspace_bytes, qlora_stream_t stream);

/* Workspace bytes of the _ex calls with a dropout mask: the plain size plus room for
 * X (.) keep (M*K bf16). */
size_t qlora_linear_dropout_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);

/*
 * Forward without a workspace argument, for callers that cannot allocate device
 * memory: for example a host program that links only this library and has no
 * device allocator of its own, or a runtime that hands out all device memory
 * from an arena planned up front and forbids allocations at call time.  (No
 * counterpart in the paper: this is a packaging variant of qlora_linear_fwd.)
 *
 * Computes exactly what qlora_linear_fwd computes, with its scratch space taken
 * from one array of QLORA_NOALLOC_SCRATCH_BYTES that the library reserves in
 * device memory of every GPU that loads it (held until the process exits).
 * Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *   - Returns QLORA_ERR_WORKSPACE, before launching anything, when the call
 *     needs more scratch than that (the need grows with M and r, plus up to
 *     9.7 MB for the split partial tiles of the GEMM's last round; 4096 tokens on
 *     a 4096 x 4096 weight with r = 16 need about 9.6 MB; at r = 16 the first
 *     calls that do not fit come at about 55 k tokens).
 *   - The first call on each device looks up the array's device address with
 *     cudaGetSymbolAddress while that device is current; make that first call
 *     before any stream capture on the device.
 *   - Every call on a device shares the one array, so calls whose executions
 *     overlap on the GPU (different streams, or host threads) race on it and
 *     corrupt each other's results; serialize them.  No byte of the array needs
 *     to start at zero: each call writes every scratch byte before reading it.
 * Other arguments, shapes and errors as qlora_linear_fwd.
 */
#define QLORA_NOALLOC_SCRATCH_BYTES (16u << 20)
qlora_status qlora_linear_fwd_noalloc(const uint16_t *X, int64_t M, const qlora_nf4_t *Wq,
                                      const uint16_t *A, const uint16_t *B, int r, float s,
                                      uint16_t *Y, float *XA_out, qlora_stream_t stream);

/*
 * Backward of the adapted linear layer ([STEPS] Step 6: gradients flow through
 * the dequantized weights into the adapters; W is frozen, no dW).  Ordering and
 * graph capture as qlora_linear_fwd (everything runs on `stream`):
 *   G  = dY B^T                   (fp32 [M, r], internal)
 *   dX = dY deq(W) + s * G A^T    (bf16 [M, K]; skipped when dX is NULL)
 *   dA = s * X^T G                (fp32 [K, r])
 *   dB = s * XA^T dY              (fp32 [r, N])
 * XA may be the forward's XA_out (fp32 [M, r]) or NULL (recomputed).
 * Shapes as qlora_linear_fwd.
 */
qlora_status qlora_linear_bwd(const uint16_t *dY, const uint16_t *X, const float *XA,
                              int64_t M, const qlora_nf4_t *Wq, const uint16_t *A,
                              const uint16_t *B, int r, float s, uint16_t *dX,
                              float *dA, float *dB, void *workspace,
                              size_t workspace_bytes, qlora_stream_t stream);

/*
 * The adapter folded into a 16-bit weight for serving ("QLoRA", ozercemkelahmet.com,
 * How it works, Step 8 and section "Merging after QLoRA"):
 *   W_out[n][k] = bf16_RN( base[n][k] + s * sum_j B[j][n] A[k][j] )
 * base is the bf16 original W16 [N, K] (the page's preferred route) or the
 * dequantized NF4 weight Wq (exactly the element qlora_nf4_dequant gives); pass
 * exactly one of them.  The sum s*(A B)^T + base is formed with one fp32 FMA per
 * element (the rank-r product accumulated in fp32 on the tensor cores) and rounded
 * once to bf16.  N a multiple of 8, K of 64; r in [8, 128], a multiple of 8.
 * W_out [N, K] bf16 must not overlap the inputs.
 */
qlora_status qlora_nf4_merge(const qlora_nf4_t *Wq, const uint16_t *W16, int64_t N, int64_t K,
                             const uint16_t *A, const uint16_t *B, int r, float s,
                             uint16_t *W_out, qlora_stream_t stream);

/*
 * Backward with adapter-input dropout and gradient accumulation ("QLoRA",
 * ozercemkelahmet.com, "A code example with common libraries": lora_dropout;
 * "Training arguments": gradient_accumulation_steps), otherwise as
 * qlora_linear_bwd.  With the forward's mask (same keep, same p):
 *   G  = dY B^T
 *   dX = dY deq(W) + s * (G A^T) (.) keep / (1 - p)   (one bf16 rounding)
 *   dA = s * Xd^T G,  Xd = X (.) keep / (1 - p)
 *   dB = s * XA^T dY  (XA from qlora_linear_fwd_ex, or recomputed from Xd if NULL)
 * accumulate != 0 adds the results into dA and dB instead of overwriting them (the
 * micro-batches of one optimizer step).  keep, p and the workspace as in
 * qlora_linear_fwd_ex; keep = NULL: no dropout.
 */
qlora_status qlora_linear_bwd_ex(const uint16_t *dY, const uint16_t *X, const float *XA,
                                 int64_t M, const qlora_nf4_t *Wq, const uint16_t *A,
                                 const uint16_t *B, int r, float s, const uint8_t *keep,
                                 float dropout_p, int accumulate, uint16_t *dX, float *dA,
                                 float *dB, void *workspace, size_t workspace_bytes,
                                 qlora_stream_t stream);

/*
 * Synchronizes `stream`, then returns the device status word of the current
 * device in *flags (QLORA_DEVSTAT_* bits) and clears it.  Returns
 * QLORA_ERR_TIMEOUT / QLORA_ERR_DEVICE_CHECK when the corresponding bit was set
 * (DEVICE_CHECK for NONFINITE and LAYOUT).
 */
qlora_status qlora_get_device_status(qlora_stream_t stream, uint32_t *flags);

/*
 * Self-test of the bounded device wait: launches one block that waits on a
 * shared-memory barrier nothing ever arrives on, with a limit of `timeout_us`
 * microseconds (1..10^7).  The wait gives up, records QLORA_DEVSTAT_TIMEOUT and
 * the kernel returns normally; the host then reads the flag with
 * qlora_get_device_status().  No trap, no hang.
 */
qlora_status qlora_selftest_wait_timeout(uint32_t timeout_us, qlora_stream_t stream);

/*
 * Time limit of every bounded device wait in the GEMM pipelines, in
 * microseconds (default 2,000,000).  Process-wide; returns the previous value.
 */
uint32_t qlora_set_wait_limit_us(uint32_t limit_us);

/*
 * Shape of the fused GEMM launches (forward Y and backward dX).  With pairing on
 * (the default), a launch whose output width (N forward, K for dX) is a multiple
 * of 256 runs as clusters of two CTAs that share each 256-row weight tile x
 * 256-token tile (one M = 256 tensor-core product over both CTAs' shared memory);
 * other widths, and every launch with pairing off, use one CTA per 128-row tile.
 * Both shapes accumulate each output over the same K steps in the same order;
 * only the last-wave split (which tiles of the last round are divided into two
 * contraction halves, summed in fp32) depends on the shape, so results may differ
 * by one bf16 ulp between the shapes, and each shape is deterministic.
 * Process-wide, read once per call; workspace sizes cover either shape.
 * Returns the previous setting (0 or 1).
 */
int qlora_set_gemm_pairing(int enable);

/*
 * Persistent units of the fused GEMM on the current device: *ctas single CTAs (the
 * SM count) and *pairs CTA pairs that the device can hold at once (0 when it cannot
 * place clusters of two).  Either pointer may be NULL.  QLORA_ERR_NO_DEVICE
 * without a B200-class device.
 */
qlora_status qlora_gemm_units(int *ctas, int *pairs);

/*
 * Kernel timing for measurement tools.  While enabled, the library records a
 * pair of CUDA events on the launching stream around every launch of its own
 * kernels, in a ring of QLORA_PROFILE_CAP entries (the oldest entries are
 * overwritten).  Enabling clears the ring.  Events are created on first use,
 * on the current device.
 */
#define QLORA_PROFILE_CAP 4096
typedef enum {
  QLORA_K_QUANTIZE = 0,     /* nf4 quantize + double quant          */
  QLORA_K_DEQUANT = 1,      /* standalone dequant                   */
  QLORA_K_PREP = 2,         /* operand preparation: A^T, hi/lo of a */
                            /* saved XA                             */
  QLORA_K_PROJECT = 3,      /* XA = X A or G = dY B^T (+ hi/lo)     */
  QLORA_K_GEMM_FWD = 4,     /* fused dequant GEMM, forward          */
  QLORA_K_GEMM_DX = 5,      /* fused dequant GEMM, dX               */
  QLORA_K_GRAD = 6,         /* adapter gradients dA and dB (one     */
                            /* launch computes both)                */
  QLORA_K_SKINNY = 7,       /* few-token forward                    */
  QLORA_K_MERGE = 8         /* adapter merged into a 16-bit weight  */
} qlora_kernel_kind;

qlora_status qlora_profile_enable(int on);

/*
 * Synchronizes the recorded events and copies up to `max` entries (oldest
 * first) into kinds[] (qlora_kernel_kind) and ms[] (elapsed milliseconds, host
 * memory).  Returns the number of entries recorded since enabling (may exceed
 * `max`), or -1 on a CUDA error.
 */
int qlora_profile_read(int max, int *kinds, float *ms);

#ifdef __cplusplus
}
#endif
#endif /* QLORA_NF4_H */
