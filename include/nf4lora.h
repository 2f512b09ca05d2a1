/*
 * nf4lora.h -- C ABI of the NF4-LoRA linear layer library (libnf4lora.so),
 * hand-written CUDA for NVIDIA B200 (sm_100a).
 *
 * The layer is the frozen-base linear of QLoRA:
 *
 *     Y  = X . W_hat^T + s . (X . A^T) . B^T,        s = alpha / r
 *     dX = dY . W_hat  + s . (dY . B) . A
 *     dA = s . (dY . B)^T . X
 *     dB = s . dY^T . (X . A^T)
 *
 * where W_hat is the bfloat16 dequantisation of a 4-bit NormalFloat (NF4)
 * encoding of the frozen weight W.  No gradient of W is ever formed.
 *
 * Sources: "第 04 篇：QLoRA 原理" (jupiter-lab.pages.dev), cited below as
 * [QP] with its section numbers; the compassingai.com QLoRA concept page,
 * cited as [CA] with its headings.
 *
 * Conventions common to every entry point
 * ---------------------------------------
 * Layout:     row-major.  W and W_hat are [d_out, d_in]; A is [r, d_in];
 *             B is [d_out, r]; X is [M, d_in]; Y and dY are [M, d_out]
 *             ([CA] "與原始 LoRA 的技術關係": B in R^{d x r}, A in R^{r x k}).
 * bfloat16:   passed as uint16_t bit patterns.
 * Pointers:   every array argument is a DEVICE pointer unless stated, at
 *             least 16-byte aligned.  The caller owns all memory; the library
 *             never allocates, frees or synchronises.
 * Streams:    `stream` is a cudaStream_t (NULL = legacy default stream).  All
 *             work is enqueued on it; NF4_OK means "enqueued".
 * Errors:     arguments are checked on the host before anything is enqueued;
 *             a failed check returns a negative nf4_status and enqueues
 *             nothing.  A failed launch returns NF4_ERR_CUDA.  The text of
 *             the last error of the calling thread is available from
 *             nf4lora_last_error_string().  Kernels bound every wait they
 *             perform; one that gives up records NF4_ERR_TIMEOUT in a device
 *             status word that nf4lora_device_status() returns.
 * Devices:    one device per call (the current one); the kernels are built
 *             for sm_100a only.
 */
#ifndef NF4LORA_H
#define NF4LORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NF4_OK = 0,
    NF4_ERR_INVALID_ARG = -1,       /* NULL pointer, negative size, bad r or s  */
    NF4_ERR_UNSUPPORTED_SHAPE = -2, /* d_in % 64 != 0, d_out % 8 != 0, ...     */
    NF4_ERR_MISALIGNED = -3,        /* a pointer not 16-byte aligned           */
    NF4_ERR_WORKSPACE = -4,         /* workspace NULL or smaller than required */
    NF4_ERR_CUDA = -5,              /* a CUDA runtime call or launch failed    */
    NF4_ERR_TIMEOUT = -6,           /* a kernel gave up a bounded wait         */
    NF4_ERR_DEVICE = -7             /* current device is not sm_100            */
} nf4_status;

/* Block sizes of the encoding: 64 weights share one first-level absmax scale
 * ([QP] §3.4, §5.1); 256 first-level scales share one second-level fp32 scale
 * ([QP] §5.2). */
#define NF4_BLOCK_SIZE 64
#define NF4_DQ_BLOCK_SIZE 256

/*
 * An NF4 + double-quantised weight ([QP] §2.1 "store the 4-bit indices, the
 * block scales or their second-level state, and the codebook"; §5.2).
 * All pointers are device pointers owned by the caller.
 *   codes       [d_out * d_in / 2] bytes.  Two 4-bit level indices per byte,
 *               row-major element order, the even element in the high nibble.
 *               Index j means the j-th NF4 level in ascending order (the table
 *               of [QP] §4.3: -1, -0.6961928, ..., 0, ..., 0.7229568, 1).
 *   qscale      [n_b] int8, n_b = d_out * d_in / 64.  Symmetric 8-bit code of
 *               (absmax_b - mean) / scale2_g, in [-127, 127].
 *   scale2      [n_g] fp32, n_g = ceil(n_b / 256).  Per group of 256 blocks,
 *               max |absmax_b - mean|.
 *   scale_mean  [1] fp32, the mean of all first-level absmax scales.
 * Restored block scale: s_b = fp32(qscale_b * fp32(scale2_g / 127)) + mean;
 * weight: w_hat = bf16_rne(fp32(level[code] * s_b))  ([QP] §6.1).
 *
 * The same codes with plain fp32 block scales (no double quantisation,
 * [QP] §5.1: one 32-bit scale per block of 64 weights, 0.5 bit per weight):
 *   absmax      [n_b] fp32, the absmax a_b of each block, stored as is.
 * A tensor with absmax != NULL is in this format: s_b = absmax_b, and qscale,
 * scale2 and scale_mean are not read (they may be NULL).  With absmax ==
 * NULL the double-quantised scales above are used.  Every entry point below
 * accepts either format.
 */
typedef struct {
    int64_t d_out;
    int64_t d_in;
    uint8_t* codes;
    int8_t* qscale;
    float* scale2;
    float* scale_mean;
    float* absmax;
} nf4_tensor;

/* ---------------------------------------------------------------- sizing */

/* Bytes of one encoded [d_out, d_in] weight when laid out by
 * nf4_tensor_from_buffer (each part padded to 256 bytes).  The unpadded
 * storage is n/2 + n_b + 4 n_g + 4 bytes, about 4.127 bits per weight
 * ([QP] §5.3, §8.1).  Returns 0 for invalid shapes.  Host only. */
size_t nf4_packed_bytes(int64_t d_out, int64_t d_in);

/* Fill `t` with pointers into one caller-owned device buffer `base` of
 * `bytes` >= nf4_packed_bytes(d_out, d_in) bytes (256-byte aligned); sets
 * t->absmax = NULL (the double-quantised format).  Host only; touches no
 * device memory.  Returns NF4_OK or an error status. */
int nf4_tensor_from_buffer(nf4_tensor* t, void* base, size_t bytes, int64_t d_out,
                           int64_t d_in);

/* The same for the fp32-block-scale format (no double quantisation): the
 * codes and one fp32 scale per block, each part padded to 256 bytes; the
 * unpadded storage is n/2 + 4 n_b bytes, 4.5 bits per weight ([QP] §5.1).
 * nf4_tensor_from_buffer_nodq sets qscale, scale2 and scale_mean to NULL. */
size_t nf4_packed_bytes_nodq(int64_t d_out, int64_t d_in);
int nf4_tensor_from_buffer_nodq(nf4_tensor* t, void* base, size_t bytes, int64_t d_out,
                                int64_t d_in);

/* Workspace (device bytes, 256-byte aligned) that each call needs. */
size_t nf4_quantize_workspace_bytes(int64_t d_out, int64_t d_in);
size_t qlora_fwd_workspace_bytes(int64_t M, int64_t d_out, int64_t d_in, int r);
size_t qlora_bwd_workspace_bytes(int64_t M, int64_t d_out, int64_t d_in, int r);

/* ---------------------------------------------------------------- encode */

/*
 * nf4_quantize -- encode the fp32 weight W [d_out, d_in] (device) into `out`
 * (whose pointers and d_out/d_in the caller set, e.g. by
 * nf4_tensor_from_buffer).
 *   1. per block of 64 consecutive weights, absmax a_b = max |w|
 *      ([QP] §3.4, §4.4; [CA] "NF4 量化機制詳解" steps 1-2);
 *   2. per weight, x = w / a_b (IEEE fp32 division) and the code = number of
 *      the 15 fp32 midpoints (level_j + level_{j+1}) / 2 strictly below x, i.e.
 *      the nearest level with ties to the lower one; an all-zero block codes
 *      every weight as the exact 0 (index 7) ([QP] §3.2, §4.3; [CA] step 3);
 *   3. pack two codes per byte ([QP] §2.1);
 *   4. mean = fp32(sum / n_b), the sum of all a_b in fp64 by a fixed pairwise
 *      tree (adjacent pairs, level by level) ([QP] §5.2);
 *   5. per group of 256 blocks, scale2 = max |a_b - mean| and
 *      qscale_b = rint((a_b - mean) / scale2 * 127) ([QP] §5.2, §3.3).
 * When out->absmax != NULL (the fp32-block-scale format) steps 4 and 5 are
 * skipped: a_b itself is written to out->absmax, and ws may be NULL.
 * Requirements: d_out >= 1, d_in >= 64, d_in % 64 == 0; W 16-byte aligned;
 * ws >= nf4_quantize_workspace_bytes(d_out, d_in) for the double-quantised
 * format.  Results are bit-identical to the stated arithmetic on every run.
 * Non-finite W is undefined.
 */
int nf4_quantize(const float* W, int64_t d_out, int64_t d_in, const nf4_tensor* out,
                 void* ws, size_t ws_bytes, void* stream);

/*
 * nf4_quantize_noalloc -- nf4_quantize without a workspace argument.  It
 * exists for callers that are not allowed to allocate device memory: for
 * example a plugin whose host framework owns every byte of device memory
 * and hands out only the tensors it manages, or code that runs where a
 * cudaMalloc would break a stream capture or a fixed memory budget.  The
 * pages describe no such entry point; it is an interface convenience only.
 *
 * The scratch the encoder needs (the fp32 absmax of every block and the fp64
 * tree partial sums) lives in a fixed array inside the library, sized for
 * at most 4,194,304 blocks of 64 weights (d_out * d_in <= 268,435,456); that
 * array (17 MiB) stays resident on every GPU that loads the library
 * until the process exits.  Larger weights return NF4_ERR_UNSUPPORTED_SHAPE.
 * The call allocates nothing; the caller still passes W and `out`.  An
 * `out` in the fp32-block-scale format (out->absmax != NULL) needs no scratch
 * and so has no such size limit.
 * Every call looks up the array's device address on the current device (a
 * host-side lookup, nothing is cached), so the call stays correct after a
 * cudaDeviceReset, which may place the array elsewhere.  The first call on a
 * device may load the library's device code there; make that first call
 * before any stream capture on the device.  Every call shares the one array,
 * so calls whose kernels overlap
 * on the GPU (different streams without ordering) race on it; calls on one
 * stream, or otherwise ordered, are safe.  Results are bit-identical to
 * nf4_quantize.  Returns NF4_OK or an error status (no message is recorded).
 */
int nf4_quantize_noalloc(const float* W, int64_t d_out, int64_t d_in, const nf4_tensor* out,
                         void* stream);

/*
 * nf4_dequantize -- W_hat [d_out, d_in] bfloat16 (device) from `w`, with the
 * bit-exact definition above ([QP] §6.1 double dequantisation, §6.2 BF16
 * compute dtype).  Materialises the whole weight; the layer calls below never
 * do.
 */
int nf4_dequantize(const nf4_tensor* w, uint16_t* W_hat, void* stream);

/* ---------------------------------------------------------------- layer */

/*
 * qlora_linear_fwd -- Y [M, d_out] = X . W_hat^T + (s X A^T) . B^T
 * ([QP] §2.2-§2.3, §6.1-§6.3; [CA] compute graph).
 *   A [r, d_in], B [d_out, r], X [M, d_in]: bfloat16, device.
 *   scaling: s (alpha / r, alpha / sqrt(r), ...).
 *   T_saved: NULL, or [M, r] fp32 (device) that receives T = s X A^T (fp32
 *            accumulation) for reuse by qlora_linear_bwd.
 * The weight is decoded tile by tile in on-chip memory and never written to
 * device memory; products accumulate in fp32; Y is rounded to bfloat16.  The
 * rank-r intermediate T enters the LoRA-up product as a pair of bfloat16
 * arrays hi = bf16(T), lo = bf16(T - hi) (about 16 significant bits), so the
 * adapter branch is not limited to bfloat16 precision ([QP] §6.3: the adapter
 * dtype may be wider than the base compute dtype).
 * Requirements: 0 <= M < 2^31, 1 <= r <= 256, d_in % 64 == 0,
 * d_out % 8 == 0, ws >= qlora_fwd_workspace_bytes(M, d_out, d_in, r).
 * A rank that is not a multiple of 8 runs as the next multiple of 8 on
 * zero-padded copies of A, B and T that the workspace holds (three more
 * small copy launches; the zero rows and columns contribute exact zeros).
 * M = 0 (an empty batch) does nothing and returns NF4_OK; X, Y and T_saved
 * may then be NULL.
 */
int qlora_linear_fwd(const nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r,
                     float scaling, const uint16_t* X, int64_t M, uint16_t* Y,
                     float* T_saved, void* ws, size_t ws_bytes, void* stream);

/*
 * qlora_linear_bwd -- gradients of the forward above ([QP] §2.4: the frozen
 * base passes the input gradient but no weight gradient is formed; §6.4:
 * only the adapters receive gradients):
 *   dX [M, d_in]  = dY W_hat + s (dY B) A
 *   dA [r, d_in]  = s (dY B)^T X
 *   dB [d_out, r] = dY^T T,    T = s X A^T   (fp32 T_saved, or recomputed
 *                                             from X when T_saved is NULL)
 * The rank-r intermediates T and V = s dY B enter the tensor-core products
 * as bfloat16 hi/lo pairs, as in the forward.
 * dX, dA or dB may be NULL to skip that output (X is then only needed for dA
 * and for recomputing T).  accumulate_grads = 1 adds the new dA / dB to the
 * values already in those buffers (gradient accumulation, [QP] §6.4) instead
 * of overwriting them.  Requirements as for the forward, and
 * ws >= qlora_bwd_workspace_bytes(M, d_out, d_in, r).
 * M = 0 (an empty batch): the gradients of an empty sum are zero, so dA and
 * dB are set to zero (left as they are with accumulate_grads = 1) and nothing
 * else happens; dY, X, T_saved and dX may then be NULL.
 */
int qlora_linear_bwd(const nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r,
                     float scaling, const uint16_t* X, const float* T_saved,
                     const uint16_t* dY, int64_t M, uint16_t* dX, uint16_t* dA,
                     uint16_t* dB, int accumulate_grads, void* ws, size_t ws_bytes,
                     void* stream);

/* ---------------------------------------------------------------- adapter merge */

/* Workspace (device bytes, 256-byte aligned) of nf4_merge_requantize: the
 * fp32 merged weight plus the encoder's scratch.  0 for invalid shapes. */
size_t nf4_merge_workspace_bytes(int64_t d_out, int64_t d_in);

/*
 * nf4_merge_lora -- the merged weight for deployment ([QP] §12.3: fold the
 * adapter into the base, W + s B A; §12.4: the effective weight is the
 * dequantised base plus the adapter):
 *   W_merged[n, k] = fp32( W_hat[n, k] + s * sum_j B[n, j] A[j, k] )
 * with W_hat the bf16 dequantisation of `w` (as nf4_dequantize), each
 * product of two bf16 values exact in fp64, the rank sum in fp64 in
 * ascending j (each addition rounded once), then one fp64 multiply by s, one
 * fp64 add and one rounding to fp32 (to nearest even): bit-identical to that
 * arithmetic on every run.  A [r, d_in], B [d_out, r] bf16; W_merged
 * [d_out, d_in] fp32 (device).  Requirements: 1 <= r <= 256 (any r), s
 * finite, the weight's shape rules.
 */
int nf4_merge_lora(const nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r, float scaling,
                   float* W_merged, void* stream);

/*
 * nf4_merge_requantize -- nf4_merge_lora followed by nf4_quantize of the
 * merged weight into `out` ([QP] §12.3: the last step rounds again, so the
 * merged 4-bit model is not exactly base + adapter).  `out` has the shape of
 * `w` and may be `w` itself (the merged weight is complete before encoding
 * starts).  ws >= nf4_merge_workspace_bytes(d_out, d_in).
 */
int nf4_merge_requantize(const nf4_tensor* w, const uint16_t* A, const uint16_t* B, int r,
                         float scaling, const nf4_tensor* out, void* ws, size_t ws_bytes,
                         void* stream);

/* ---------------------------------------------------------------- optimizer */

/*
 * One trainable adapter tensor (A or B) for lora_adamw_step.  Device
 * pointers, 16-byte aligned, n elements each, caller-owned:
 *   master  fp32 parameters, updated in place;
 *   param   the bf16 copy the layer reads, overwritten with bf16_rne(master),
 *           or NULL;
 *   grad    bf16 gradient (the dA or dB of qlora_linear_bwd), read only;
 *   m, v    fp32 first and second moments, updated in place (zero before
 *           the first step).
 */
typedef struct {
    float* master;
    uint16_t* param;
    const uint16_t* grad;
    float* m;
    float* v;
    int64_t n;
} lora_adamw_tensor;

typedef struct {
    float lr;
    float beta1;
    float beta2;
    float eps;
    float weight_decay;
    int64_t step; /* t, counted from 1 */
} lora_adamw_hparams;

/*
 * lora_adamw_step -- one AdamW update of `count` adapter tensors, the step
 * that follows the backward ([QP] §7.3: two fp32 moments per trainable
 * parameter; §8.3: an fp32 master copy beside a bf16 adapter; the frozen
 * base has no optimizer state).  The pages print no update rule; this is
 * decoupled-weight-decay AdamW with bias-corrected moments:
 *   p <- p (1 - lr wd);   m <- b1 m + (1 - b1) g;   v <- b2 v + (1 - b2) g^2;
 *   p <- p - lr / (1 - b1^t) * m / (sqrt(v) / sqrt(1 - b2^t) + eps)
 * computed per element in fp32; the constants 1 - lr wd, 1 - b1, 1 - b2,
 * lr / (1 - b1^t) and 1 / sqrt(1 - b2^t) are formed on the host in fp64 and
 * rounded once.  Requirements: 1 <= count <= 1024; n >= 0 (n = 0 tensors are
 * skipped and may have NULL pointers); step >= 1; 0 <= beta1, beta2 < 1;
 * eps > 0; lr >= 0; weight_decay >= 0; all finite.  Up to 8 tensors share
 * one launch.  The tensors must not overlap one another.
 */
int lora_adamw_step(const lora_adamw_tensor* tensors, int count, const lora_adamw_hparams* h,
                    void* stream);

/* ---------------------------------------------------------------- status */

/* Text of the last error returned to the calling host thread ("" if none). */
const char* nf4lora_last_error_string(void);

/* Reads (and clears) the device status word of the current device after
 * synchronising `stream`: NF4_OK, or NF4_ERR_TIMEOUT if a kernel gave up a
 * bounded wait since the last call.  Returns NF4_ERR_CUDA if the
 * synchronisation fails. */
int nf4lora_device_status(void* stream);

/*
 * nf4lora_check_bounded_wait -- self-check of the failure detector shared by
 * every kernel above (no counterpart in the pages: it guards the library, not
 * the method).  Enqueues one small kernel that, like a layer kernel, holds
 * tensor memory and has a bulk copy in flight, and then waits on a barrier
 * that nothing ever arrives on.  The wait gives up after limit_ns
 * nanoseconds (1e5 <= limit_ns <= 1e9), records NF4_ERR_TIMEOUT in the
 * device status word, drains the copy, frees the tensor memory and returns,
 * so the context stays usable.  A later nf4lora_device_status() returns
 * NF4_ERR_TIMEOUT once, then NF4_OK.  Allocates nothing.  Returns NF4_OK
 * (enqueued), NF4_ERR_INVALID_ARG, NF4_ERR_DEVICE or NF4_ERR_CUDA.
 */
int nf4lora_check_bounded_wait(int64_t limit_ns, void* stream);

/*
 * Debug build (no counterpart in the pages).  Built with NF4LORA_DEBUG
 * (python nf4_base_lora_b200/build.py --debug -> lib/libnf4lora_debug.so),
 * the kernels check the index and alignment of their memory accesses; the
 * first check that fails records (site << 16) | source line and that access
 * is skipped instead of faulting.  nf4lora_debug_site() synchronises
 * `stream`, stores that word (0 if every check passed) in *site and clears
 * it.  In a release build no check runs and the word stays 0.
 * nf4lora_debug_build() returns 1 in a debug build, 0 otherwise.
 */
int nf4lora_debug_site(void* stream, unsigned int* site);
int nf4lora_debug_build(void);

/* ---------------------------------------------------------------- tracing */

/* Start timing the library's own kernel launches (host-side tracing): each
 * launch from now on is bracketed by two CUDA events recorded on its stream;
 * inside a stream capture the records become graph nodes that every replay
 * refreshes.  The first max_launches launches get a record, later ones are
 * only counted.  Creates 2 * max_launches events (no device memory).
 * Returns NF4_OK, NF4_ERR_INVALID_ARG or NF4_ERR_CUDA. */
int nf4lora_trace_start(int max_launches);

/* Stop bracketing launches; the records stay readable. */
int nf4lora_trace_stop(void);

/* Launches counted since nf4lora_trace_start (recorded or not). */
int nf4lora_trace_count(void);

/* Kernel name and device time in ms of record i; waits for its stop event. */
int nf4lora_trace_get(int i, char* name, size_t name_len, float* ms);

/* Library version, e.g. "nf4lora 0.1.0 sm_100a". */
const char* nf4lora_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NF4LORA_H */
