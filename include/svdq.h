/*
 * svdq.h - C ABI of the B200 (sm_100a) SVDQuant W4A4 + low-rank linear layer.
 *
 * The layer computes (msModelSlim "SVDQuant Low-Rank Residual Quantization
 * Algorithm Terminology Entry", section 2.3, the dual-path output equation,
 * with the bias of the migration identity added):
 *
 *     Y = Q(X diag(s)^-1) Q(R) + (X diag(s)^-1 L1) L2 + b
 *
 * with s the smoothing factor of section 2.3 eq. 2, L1 L2 the rank-r truncated
 * SVD of the migrated weight diag(s) W (section 2.2; eq. 3) and R the residual
 * quantized to 4 bits per group along K ("SVDQuant: Absorbing Outliers by
 * Low-Rank Components for 4-Bit Diffusion Models", abstract).
 *
 * Conventions for every call:
 *  - All tensors are plain row-major device pointers unless a parameter says
 *    "host". X is bf16 [M, K], W is bf16 [K, N] (Y = X W + b), Y is bf16 [M, N].
 *    Device pointers must be 16-byte aligned.
 *  - Ownership: the caller owns every pointer it passes (X, Y, W, bias, the
 *    calibration statistic, LoRA factors, workspaces, the stream). The library
 *    never frees them and keeps no reference after the call returns, except
 *    that work queued on `stream` reads/writes them until it completes.
 *    A layer handle owns its prepared device buffers; svdq_destroy frees them.
 *  - Streams: `stream` is a cudaStream_t (NULL = legacy default stream). All
 *    device work is queued on it; svdq_linear_forward and
 *    svdq_quantize_activations never synchronize the host. A handle is used by
 *    one stream at a time; svdq_attach_lora must be stream-ordered with the
 *    forwards that precede it.
 *  - Devices: a layer lives on the device that was current when it was
 *    prepared. Calls that launch work on a layer (forward, quantize
 *    activations, attach) must be made with that device current; otherwise
 *    they return SVDQ_ERR_INVALID_ARG and launch nothing.
 *  - Errors: every call returns an svdq_status and never aborts or throws.
 *    Argument errors (shapes, NULL or misaligned pointers, sizes) are
 *    reported before any device work is queued.
 *    svdq_last_error() returns a thread-local description of the last failure.
 *    Launch failures come back as SVDQ_ERR_CUDA. A pipeline wait inside a
 *    kernel that gives up (it never blocks forever) is reported by
 *    svdq_device_status() as SVDQ_ERR_DEVICE_TIMEOUT.
 *  - Shape limits: K a multiple of 128; N a multiple of 16; M >= 1;
 *    0 <= rank (after any LoRA concatenation) <= 256 (section 2.6 recommends
 *    rank <= 128; the larger limit leaves room for LoRA adapters); only 2-D
 *    linear weights (section 2.6). Rank 0 is the smoothing-only special case
 *    the entry's related terms name (SmoothQuant): no branch, R = diag(s) W.
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(SVDQ_BUILD) && defined(__GNUC__)
#define SVDQ_API __attribute__((visibility("default")))
#else
#define SVDQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,     /* bad pointer, shape, alignment or workspace size */
  SVDQ_ERR_UNSUPPORTED = 2,     /* no sm_100 device, or a shape outside the limits above */
  SVDQ_ERR_OOM = 3,             /* a device allocation of the library failed */
  SVDQ_ERR_CUDA = 4,            /* a CUDA / cuSOLVER call or a kernel launch failed */
  SVDQ_ERR_NUMERIC = 5,         /* the SVD did not converge or produced non-finite values */
  SVDQ_ERR_DEVICE_TIMEOUT = 6   /* a kernel gave up a pipeline wait (see svdq_device_status) */
} svdq_status;

typedef enum {
  SVDQ_INT4_G64 = 0,  /* symmetric INT4, 64 values per group along K, fp32 scale = amax/7 */
  SVDQ_NVFP4_G16 = 1  /* E2M1 values, 16 per group along K, E4M3 group scale, fp32 tensor scale */
} svdq_format;

/* svdq_config.flags */
enum {
  SVDQ_NO_SMOOTHING = 1  /* s = 1 for every channel (no migration; an ablation of eq. 1-2) */
};

typedef struct {
  int K;            /* input features (rows of W) */
  int N;            /* output features (columns of W) */
  int rank;         /* r of the truncated SVD, 0..256 (0: no low-rank branch) */
  float alpha;      /* migration strength of eq. 2, in [0, 1] */
  float s_min;      /* lower clamp of s in eq. 2 (> 0; 1e-5 is the documented default) */
  svdq_format fmt;  /* 4-bit format of Q(.) */
  unsigned int flags; /* 0, or SVDQ_NO_SMOOTHING */
} svdq_config;

/* LoRA adapter slots a layer holds at once. */
#define SVDQ_MAX_ADAPTERS 8

typedef struct svdq_layer* svdq_layer_t;

typedef struct {
  int K, N, rank;   /* rank includes attached LoRA adapters */
  int rank_pad;     /* rank rounded up to a multiple of 32 (layout of the branch buffers; 0 when rank is 0) */
  int fmt;          /* svdq_format */
  float alpha;
  float g_x;        /* NVFP4 static activation tensor scale (1 for INT4) */
  float g_w;        /* NVFP4 residual tensor scale (1 for INT4) */
  float t_scale;    /* factor applied to T before its bf16 store: 1 (INT4) or 1/(g_x g_w) (NVFP4) */
  int base_rank;    /* rank of the SVD factors alone */
  unsigned int flags;          /* svdq_config.flags of the layer */
  unsigned int adapter_slots;  /* bit a set: adapter slot a holds an adapter */
  int adapter_col_start[SVDQ_MAX_ADAPTERS + 1]; /* slot a owns branch columns [start[a], start[a+1]);
                                                   the base factors own [0, start[0]) */
} svdq_layer_info;

/* Activation statistic A_scale of eq. 2 (section 2.3: per-channel absolute
 * maximum of the activations) over a calibration batch.
 *   X            device bf16 [M, K]
 *   absmax_inout device float [K]; updated in place to max(absmax, max_m |X[m,k]|),
 *                so several calibration batches can be folded in. Initialise
 *                it to zeros before the first batch. */
SVDQ_API svdq_status svdq_calibrate_absmax(const void* X, int M, int K, float* absmax_inout, void* stream);

/* Offline preparation (section 2.1, in order: migrate, decompose, quantize):
 *  1. W_scale[k] = max_n |W[k,n]| (the weight statistic of eq. 2, per input
 *     channel); s = A_scale^alpha / W_scale^(1-alpha) computed in float64 on the
 *     host (sqrt/sqrt for alpha = 0.5), rounded to float32, clamped at s_min
 *     (s = 1 where a statistic is 0); inv_s = 1/s in float32.
 *  2. W_hat = fp32(s_k W[k,n]) (eq. 1); float64 SVD of W_hat (cuSOLVER gesvd);
 *     L1 = U_r, L2 = Sigma_r V_r^T, each column of L1 signed so that its
 *     largest-magnitude entry is positive, both rounded to bf16.
 *  3. R = fp32(W_hat - L1 L2) (float64 sums, j = 0..r-1 in order), quantized
 *     per output column in groups of G along K.
 *   W          device bf16 [K, N]
 *   bias       device bf16 [N], or NULL for no bias
 *   act_absmax device float [K] (from svdq_calibrate_absmax)
 *   out        receives the new handle (NULL on failure)
 * Synchronizes `stream` (the SVD's convergence flag is read on the host). */
SVDQ_API svdq_status svdq_prepare_weights(const svdq_config* cfg, const void* W, const void* bias, const float* act_absmax,
                                 void* stream, svdq_layer_t* out);

/* As svdq_prepare_weights, with the bf16 factors given instead of computed
 * (e.g. from an offline SVD): L1 device bf16 [K, rank], L2 device bf16
 * [rank, N]. Steps 1 and 3 are unchanged. */
SVDQ_API svdq_status svdq_prepare_weights_with_factors(const svdq_config* cfg, const void* W, const void* bias,
                                              const float* act_absmax, const void* L1, const void* L2, void* stream,
                                              svdq_layer_t* out);

/* Bytes of workspace svdq_linear_forward needs for M rows: the activation
 * codes and scales, T, and the activation kernel's float partials of T over
 * its shares of K (their number depends on M, K, the rank and the device's SM
 * count, so query this on the device the layer lives on). */
SVDQ_API svdq_status svdq_workspace_size(svdq_layer_t layer, int M, size_t* bytes);

/* The hot path: Y = Q(X diag(s)^-1) Q(R) + (X diag(s)^-1 L1) L2 + b, bf16 out.
 * Two kernels on `stream`: (1) smoothing + group quantization of X + the
 * down-projection T = x_hat L1 in one pass over X; (2) the 4-bit GEMM whose
 * epilogue adds T L2 and the bias before a single bf16 store of Y.
 *   X          device bf16 [M, K]
 *   Y          device bf16 [M, N] (overwritten)
 *   workspace  device buffer of at least svdq_workspace_size(layer, M) bytes,
 *              256-byte aligned; its contents need no initialisation.
 * M_pad / 128 = ceil(M / 128) must not exceed 65536 (the layer keeps one
 * arrival counter per 128-row block for the activation kernel; they return
 * to zero at the end of every launch, which is why a layer serves one stream
 * at a time). */
SVDQ_API svdq_status svdq_linear_forward(svdq_layer_t layer, const void* X, int M, void* Y, void* workspace,
                                size_t workspace_bytes, void* stream);

/* svdq_linear_forward with per-kernel timing: events[0..2] are cudaEvent_t the
 * caller created; they are recorded on `stream` before the activation kernel,
 * between the two kernels and after the GEMM. Same work, same launches. */
SVDQ_API svdq_status svdq_linear_forward_profiled(svdq_layer_t layer, const void* X, int M, void* Y, void* workspace,
                                                  size_t workspace_bytes, void* stream, void* const* events);

/* The MLP block of two layers, Y = down(GELU(up(X))), fused across the
 * boundary between them: the up layer's GEMM epilogue rounds its output to
 * bf16, applies GELU (the erf form in float32, erfc as exp(-x^2) times a
 * fitted polynomial for erfcx, absolute error under 1e-6) and rounds to bf16
 * (h, what a plain
 * composition of the layers would pass on), then smooths and quantizes
 * h for the down layer straight into the down layer's activation codes and
 * scales, and contracts it with the down layer's factor for the down layer's
 * branch input T. h itself never goes to device memory. Abstract: the
 * low-rank branch is fused into the low-bit kernels to cut redundant memory
 * traffic; this carries that across the two layers of the block. The up
 * layer's branch input T is carried as a bf16 pair here (about 16 significant
 * bits, where a single forward holds it in bf16), because the bf16 rounding
 * of the up output decides the down layer's codes.
 * Kernels on `stream`: the up layer's activation kernel, the fused up GEMM, a
 * small fixed-order sum of the T partials, the down layer's GEMM.
 *   up, down  NVFP4 layers on the same device, up->N == down->K,
 *             down->K % 256 == 0, down rank (with adapters) 1..32
 *   X         device bf16 [M, K_up];  Y  device bf16 [M, N_down] (overwritten)
 *   workspace at least svdq_mlp_workspace_size(up, down, M) bytes, 256-byte
 *             aligned, no initialisation needed
 * Other layer pairs return SVDQ_ERR_UNSUPPORTED (run them as two forwards). */
SVDQ_API svdq_status svdq_mlp_workspace_size(svdq_layer_t up, svdq_layer_t down, int M, size_t* bytes);
SVDQ_API svdq_status svdq_mlp_forward(svdq_layer_t up, svdq_layer_t down, const void* X, int M, void* Y,
                                      void* workspace, size_t workspace_bytes, void* stream);
/* svdq_mlp_forward recording events[0..4] (cudaEvent_t) before the activation
 * kernel, after it, after the fused up GEMM, after the T sum and after the
 * down GEMM. */
/* Where a forward leaves the down layer's activations in the MLP workspace
 * (for inspection): offsets[0] codes, offsets[1] scales, offsets[2] T, in
 * bytes from the workspace start, in the layouts svdq_quantize_activations
 * documents for the down layer (M_pad = M rounded up to 128 rows). */
SVDQ_API svdq_status svdq_mlp_workspace_layout(svdq_layer_t up, svdq_layer_t down, int M, size_t* offsets);
SVDQ_API svdq_status svdq_mlp_forward_profiled(svdq_layer_t up, svdq_layer_t down, const void* X, int M, void* Y,
                                               void* workspace, size_t workspace_bytes, void* stream,
                                               void* const* events);

/* svdq_linear_forward for callers that cannot allocate device memory: hosts
 * whose device memory belongs to their own allocator and may not be grown
 * behind its back, or latency-critical loops where an allocation may
 * synchronize the device. The pages describe no such call; it exists for
 * these callers only. The workspace is a fixed 32 MiB scratch array inside
 * the library's device image (held by every GPU that loads the library until
 * the process exits); the caller passes only X and Y. Nothing is allocated
 * and nothing needs clearing: the first kernel overwrites every byte the
 * second one reads. Layers whose workspace for M rows exceeds 32 MiB are
 * refused with SVDQ_ERR_INVALID_ARG (svdq_workspace_size gives the need).
 * The first call on a device looks up the array's device address (set-up, once
 * per device, with that device current); make that first call before any
 * stream capture. All calls on a device share the array: calls whose work
 * overlaps on the GPU race, so issue them on one stream. */
SVDQ_API svdq_status svdq_linear_forward_noalloc(svdq_layer_t layer, const void* X, int M, void* Y, void* stream);

/* Attaches a LoRA adapter Y += scale X A B to the low-rank branch without
 * re-quantizing R (abstract: off-the-shelf LoRAs without re-quantization).
 * The branch sees X diag(s)^-1, so the adapter enters as the column block
 * [bf16(diag(s) A)] of L1' and the row block [bf16(scale B)] of L2'. The
 * residual codes and scales are untouched.
 * The adapter takes the lowest free of SVDQ_MAX_ADAPTERS slots, returned in
 * *slot_out (may be NULL). The branch is L1' = [L1 | F_a | F_b | ...],
 * L2' = [L2 ; G_a ; G_b ; ...] with the occupied slots in slot order, so by
 * default every adapter applies to every row (they accumulate); see
 * svdq_linear_forward_masked for per-row selection.
 *   A  device bf16 [K, r_l];  B  device bf16 [r_l, N];  rank + r_l <= 256.
 * On any failure the layer is unchanged and *slot_out is -1. Synchronizes
 * `stream` before freeing the previous branch buffers. */
SVDQ_API svdq_status svdq_attach_lora(svdq_layer_t layer, const void* A, const void* B, int r_l, float scale, void* stream,
                                      int* slot_out);

/* Removes the adapter in `slot`: the branch buffers become byte for byte what
 * they would be had the adapter never been attached (the remaining blocks are
 * re-laid out in slot order), and the residual is untouched. Returns
 * SVDQ_ERR_INVALID_ARG for an empty slot. Synchronizes `stream`. */
SVDQ_API svdq_status svdq_detach_lora(svdq_layer_t layer, int slot, void* stream);

/* svdq_linear_forward with per-row adapter selection (several requests with
 * different LoRAs in one batch): row m of X uses the base branch plus the
 * adapters whose slot bits are set in row_adapter_mask[m]; the branch columns
 * of the other adapters are zeroed in T for that row before the GEMM, so a
 * row gives exactly what a layer holding only its selected adapters would.
 *   row_adapter_mask  device uint32 [M], 4-byte aligned (bit a = slot a). */
SVDQ_API svdq_status svdq_linear_forward_masked(svdq_layer_t layer, const void* X, int M, void* Y, void* workspace,
                                                size_t workspace_bytes, const uint32_t* row_adapter_mask, void* stream);

/* The first kernel of the forward alone, into caller buffers, for inspection:
 *   codes   INT4: uint8 [M_pad, K], the E4M3 encoding of each integer code
 *                 (-8..7; exact). NVFP4: uint8 [M_pad, K/2], two E2M1 codes per
 *                 byte, element 2j in bits 3:0.
 *   scales  INT4: float [K/64][M_pad] (group scale amax/7, transposed).
 *           NVFP4: uint8 E4M3 in 512-byte atoms, atom (m/128)*(K/64) + k/64,
 *                  byte (m%32)*16 + ((m/32)%4)*4 + (k/16)%4.
 *   T       bf16 [M_pad, rank_pad] = t_scale * (x_hat L1) (columns >= rank are 0)
 * with M_pad = M rounded up to a multiple of 128 (rows >= M are zero codes).
 * This call allocates: the activation kernel splits K into shares whose float
 * partial products it sums in share order, and their scratch buffer is taken
 * with cudaMallocAsync on `stream` and freed (cudaFreeAsync) before the call
 * returns. The forward keeps that buffer in its workspace instead. */
SVDQ_API svdq_status svdq_quantize_activations(svdq_layer_t layer, const void* X, int M, void* codes, void* scales, void* T,
                                      void* stream);

/* Prepared weights in canonical layout, for checkpointing and inspection.
 * With blob == NULL only *bytes is set. Otherwise *bytes must be at least the
 * size and the blob (host memory) receives an svdq_blob_header followed by the
 * sections at the offsets it lists. Synchronizes `stream`. */
typedef struct {
  uint32_t magic;     /* 0x51445653 ("SVDQ") */
  uint32_t version;   /* 1 */
  int32_t fmt, K, N, rank;
  float alpha, g_x, g_w, reserved;
  uint64_t off_s;       /* float [K] */
  uint64_t off_inv_s;   /* float [K] */
  uint64_t off_L1;      /* bf16 [K, rank] */
  uint64_t off_L2;      /* bf16 [rank, N] */
  uint64_t off_codes;   /* uint8 [N, K/2]: two 4-bit codes per byte, element 2j in bits 3:0;
                           INT4 two's complement, NVFP4 E2M1 */
  uint64_t off_scales;  /* INT4 float [N, K/64]; NVFP4 uint8 E4M3 [N, K/16] */
  uint64_t off_bias;    /* bf16 [N] */
  uint64_t total;
} svdq_blob_header;

SVDQ_API svdq_status svdq_export_weights(svdq_layer_t layer, void* blob, size_t* bytes, void* stream);

SVDQ_API svdq_status svdq_layer_get_info(svdq_layer_t layer, svdq_layer_info* info);

/* Reads and clears the layer's device status word (synchronizes `stream`):
 * SVDQ_OK, or SVDQ_ERR_DEVICE_TIMEOUT if a kernel of this layer gave up a wait. */
SVDQ_API svdq_status svdq_device_status(svdq_layer_t layer, void* stream);

/* Frees the handle and its device buffers (synchronizes the device first). */
SVDQ_API svdq_status svdq_destroy(svdq_layer_t layer);

/* Thread-local message of the last failed call ("" if none). */
SVDQ_API const char* svdq_last_error(void);

/* ------------------------------------------------------------------------
 * The 4-bit weight-only baseline (W4A16) the SVDQuant abstract measures its
 * 3.0x speedup against. W is quantized alone (no smoothing, no low-rank
 * branch) with the same symmetric INT4 group-64 quantizer (scale = amax / 7
 * per output column and 64 consecutive k); activations stay bf16:
 *   Y = X bf16(fp32(q * scale))^T + b, fp32 accumulation, bf16 out.
 * The packed codes stay 4-bit in device memory and are dequantized on chip in
 * every forward. Same shape limits as the W4A4 layer (K % 128 == 0,
 * N % 16 == 0), same error conventions. */
typedef struct svdq_w4a16* svdq_w4a16_t;

/* W device bf16 [K, N]; bias device bf16 [N] or NULL. Synchronizes `stream`. */
SVDQ_API svdq_status svdq_w4a16_prepare(const void* W, const void* bias, int K, int N, void* stream,
                                        svdq_w4a16_t* out);
/* X device bf16 [M, K] -> Y device bf16 [M, N], one kernel on `stream`. */
SVDQ_API svdq_status svdq_w4a16_forward(svdq_w4a16_t layer, const void* X, int M, void* Y, void* stream);
/* The quantized weights, for inspection: codes host uint8 [N, K/2] (two's-
 * complement nibbles, element 2j in bits 3:0), scales host float [K/64, N].
 * Synchronizes `stream`. */
SVDQ_API svdq_status svdq_w4a16_export(svdq_w4a16_t layer, void* codes, void* scales, void* stream);
/* Frees the layer (synchronizes the device first). */
SVDQ_API svdq_status svdq_w4a16_destroy(svdq_w4a16_t layer);

/* Test hook for failure detection: the library's device allocation number
 * `index` (0 = the next one) fails with SVDQ_ERR_OOM as if the device were out
 * of memory, so that tests can check that every allocating call unwinds
 * cleanly (no leak, no handle). A negative index switches the hook off. */
SVDQ_API void svdq_debug_fail_allocation(long long index);

/* Failure-detection self-test: launches a kernel that waits on a barrier no
 * one arrives on, with the library's bounded wait shortened to limit_ns, and
 * returns SVDQ_ERR_DEVICE_TIMEOUT when the wait gave up as designed (the
 * context stays usable). Synchronizes `stream`. */
SVDQ_API svdq_status svdq_selftest_bounded_wait(unsigned long long limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
