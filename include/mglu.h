/*
 * mglu.h -- C ABI of libmglu.so, a B200 (sm_100a) forward pass of the Masked
 * Gated Linear Unit (MGLU, "Mixture of Element-wise Gating").
 *
 * The method ("Masked Gated Linear Unit", atlas.scime.ai summary of the MGLU
 * paper, "Approach"): one shared weight matrix W (d x h) and n_m learned
 * binary masks M_i over it.  Mask i splits W into complementary gate and value
 * parts; the layer sums the n_m gated products ("Measured effects": summing
 * all 4 masks is the default the routing ablations are measured against):
 *
 *     out[b,j] = sum_{i<n_m} act(g_i[b,j]) * v_i[b,j]
 *     g_i = x (M_i . W)          v_i = x ((1 - M_i) . W) = x W - g_i
 *
 * act is Swish (beta = 1, "SwiMGLU"), exact-erf GELU or ReLU ("Measured
 * effects" rows on the gating activation).  Which side of a mask is the gate
 * is not stated on the page; here a set bit marks a gate weight.  No biases.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    allocates no device memory on any call declared here except
 *    mglu_backward's first call (its cuBLAS handle); the little global
 *    scratch the decode kernel needs is a caller-provided buffer (see
 *    mglu_scratch_bytes).
 *  - Calls are asynchronous and ordered on `stream` (a cudaStream_t passed as
 *    void*; NULL = the legacy default stream).
 *  - Arguments are checked before anything is launched.  A negative return
 *    is an mglu_status; nothing was launched when it is INVALID, UNSUPPORTED
 *    or ALIGN.  MGLU_ERR_CUDA means a launch failed (cudaGetLastError is
 *    cleared and the text is available from mglu_last_cuda_error()).
 *  - Layouts (row-major, dense, no padding):
 *        x       [T][d]            activations
 *        W       [h][d]            W^T, i.e. nn.Linear(d, h).weight
 *        masks   [n_m][h][d]       uint8, 0 or 1 (unpacked form)
 *        packed  mglu_packed_bytes(n_m, d, h) bytes, see mglu_pack_masks
 *        out     [T][h]
 *        W_down  [d][h]            nn.Linear(h, d).weight
 *        y       [T][d]
 *  - bf16 path (dtype MGLU_BF16): x, W, out, W_down, y are bf16; every
 *    product x*W is exact and they accumulate in fp32, at any input scale
 *    within bf16's range (masks select or negate whole bf16 values, no
 *    rescaling); the result is rounded to bf16 once.
 *    Requirements (else MGLU_ERR_ALIGN): every pointer 16-byte aligned and
 *    d % 8 == 0 (a row of W then starts on 16 bytes, and each 8-weight piece
 *    owns whole bytes of mask bits).  The down-projection needs h % 8 == 0.
 *  - fp32 path (dtype MGLU_F32): x, W, out, W_down, y are float; plain fp32
 *    FMA on CUDA cores (never TF32); any d, h; 4-byte aligned pointers.
 *  - Supported n_m: 1, 2, 4, 8 (else MGLU_ERR_UNSUPPORTED).  T == 0 is a
 *    no-op that returns MGLU_OK.  Sizes are limited to d, h < 2^31 and
 *    T * max(d, h) < 2^62.
 */
#ifndef MGLU_H
#define MGLU_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MGLU_OK = 0,
    MGLU_ERR_INVALID = -1,     /* null pointer, negative size, bad act/dtype, small workspace */
    MGLU_ERR_UNSUPPORTED = -2, /* n_m not in {1,2,4,8}; T > 16 on the decode-only entry point */
    MGLU_ERR_ALIGN = -3,       /* a pointer or size alignment rule above is broken */
    MGLU_ERR_CUDA = -4,        /* a CUDA runtime call or a kernel launch failed */
    MGLU_ERR_TIMEOUT = -5      /* a device-side bounded wait gave up (see mglu_last_device_status) */
} mglu_status;

typedef enum { MGLU_ACT_SWISH = 0, MGLU_ACT_GELU = 1, MGLU_ACT_RELU = 2 } mglu_act;

/* OR into act for the dense-gate ablation ("Masked Gated Linear Unit",
 * "Measured effects", last row, "Remove the gate mask (dense gate)"): the
 * gate of every mask is the whole product x W, each value keeps its mask,
 *     out[b,j] = sum_{i<n_m} act((x W)[b,j]) * v_i[b,j].
 * Accepted wherever an act is (forward, FFN block, host and static calls). */
#define MGLU_GATE_DENSE 16
typedef enum { MGLU_BF16 = 0, MGLU_F32 = 1 } mglu_dtype;

/* Kernel families mglu_forward can launch (see mglu_forward_path). */
typedef enum { MGLU_PATH_DECODE = 0, MGLU_PATH_PREFILL = 1, MGLU_PATH_F32 = 2 } mglu_path;

/* Bytes of the packed mask stream: ceil(h * d * n_m / 8).  0 for bad input. */
size_t mglu_packed_bytes(int n_m, int64_t d, int64_t h);

/*
 * Pack n_m binary masks into the bit stream the forward reads ("Approach":
 * the masks are binary and are unpacked inside the fused kernel; the bit
 * format is this library's own).  Weight (j, k) owns the n_m consecutive bits
 * starting at bit (j*d + k)*n_m; bit i of that field is mask i; bits are
 * numbered from the least significant bit of each byte.  So for n_m = 8 byte
 * j*d+k holds the eight masks of weight (j, k); for n_m = 4 the low nibble of
 * a byte is weight k (even) and the high nibble weight k+1.  A row of W
 * (fixed j) and its mask bits are therefore tiled alike along k.
 *   masks   in : [n_m][h][d] uint8; any nonzero byte counts as 1.
 *   packed out : mglu_packed_bytes(n_m, d, h) bytes, every byte written
 *                (unused high bits of a partial last byte are 0).
 * Requirements: packed 16-byte aligned.  Any d and h are accepted; the bf16
 * forward additionally needs d % 8 == 0.
 * Errors: INVALID, UNSUPPORTED, ALIGN, CUDA.
 */
int mglu_pack_masks(const uint8_t *masks, int n_m, int64_t d, int64_t h,
                    uint8_t *packed, void *stream);

/*
 * Pack the masks straight from their training-time logits ("Masked Gated
 * Linear Unit", "Limitations": the masks are held as FP16 logits while
 * training, and binary in the forward): M_i[j,k] = 1 where the logit is
 * greater than zero, else 0.  +0, -0, negative values and NaN give 0;
 * positive subnormals and +infinity give 1.
 *   logits in  : [n_m][h][d] IEEE binary16 (uint16 bit patterns), device,
 *                2-byte aligned (16-byte aligned with (h*d) % 8 == 0 for
 *                vector loads).
 *   packed out : as mglu_pack_masks (same format, every byte written).
 * Errors: INVALID, UNSUPPORTED, ALIGN, CUDA.
 */
int mglu_pack_mask_logits(const void *logits, int n_m, int64_t d, int64_t h,
                          uint8_t *packed, void *stream);

/* Exact inverse of mglu_pack_masks: writes [n_m][h][d] bytes, each 0 or 1. */
int mglu_unpack_masks(const uint8_t *packed, int n_m, int64_t d, int64_t h,
                      uint8_t *masks, void *stream);

/*
 * Bytes of scratch the decode kernel needs for a product with `rows` output
 * rows (h for mglu_forward, d for mglu_down_proj): the partial sums of the
 * row blocks that several CTAs share, two slots per CTA of the grid (about
 * 6 MB, the same for every `rows`).  The scratch must be 16-byte aligned; its
 * contents need no initialization (every slot is written before it is read
 * within a call).  Calls that may run concurrently (other streams) need
 * separate scratch buffers.  Only the decode path touches it: when
 * mglu_forward_path(T, dtype) is not MGLU_PATH_DECODE it may be NULL.
 */
size_t mglu_scratch_bytes(int64_t rows);

/*
 * MGLU up-projection with the act-and-sum epilogue fused: out = MGLU(x)
 * ("Masked Gated Linear Unit", "Approach": one shared W, n_m binary masks
 * splitting it into gate and value parts, the gated products summed; and
 * "Problem": at decode the layer is bound by reading W, so the masks are
 * unpacked inside the kernel that reads it).
 * Reads each weight and its mask bits once per pass; for T up to the decode
 * limit (16 by default) one pass serves all tokens; above it a tensor-core
 * (tcgen05) kernel tiles tokens and weights.
 *   x [T][d], W [h][d], packed (from mglu_pack_masks with the same n_m, d, h),
 *   act in mglu_act (optionally | MGLU_GATE_DENSE), dtype in mglu_dtype,
 *   out [T][h],
 *   scratch / scratch_bytes: see mglu_scratch_bytes(h).
 * Errors: INVALID (also: scratch missing or too small on the decode path),
 * UNSUPPORTED, ALIGN, CUDA.
 */
int mglu_forward(const void *x, int64_t T, int64_t d, const void *W, int64_t h,
                 const uint8_t *packed, int n_m, int act, int dtype, void *out,
                 void *scratch, size_t scratch_bytes, void *stream);

/* Weightings of routed masks (see mglu_route_topk). */
typedef enum { MGLU_ROUTE_HARD = 0, MGLU_ROUTE_SOFTMAX = 1 } mglu_route_mode;

/*
 * Mask routing ("Masked Gated Linear Unit", "Measured effects": each token
 * routed to only 1, or 2, of its 4 masks instead of summing all of them).
 * The page defines no router; here one linear map scores the masks per
 * token, r[b,i] = sum_k x[b,k] W_r[i,k] (fp32 accumulation, no bias), the k
 * highest scores are kept (of equal scores the lower mask index; a NaN score
 * never beats a number), and the token's mask weights are written:
 *   MGLU_ROUTE_HARD:    1 for each kept mask, 0 otherwise;
 *   MGLU_ROUTE_SOFTMAX: the softmax of all n_m scores for each kept mask,
 *                       0 otherwise (as a mixture-of-experts router scales
 *                       an expert by its probability).
 *   x [T][d] and W_r [n_m][d] in dtype (MGLU_BF16 or MGLU_F32, aligned to
 *   their element size); weights [T][n_m] float (written); scores
 *   [T][n_m] float (written, may be NULL).  0 <= k <= n_m.
 * The weights feed mglu_forward_weighted.  Errors: INVALID, UNSUPPORTED,
 * ALIGN, CUDA.
 */
int mglu_route_topk(const void *x, int64_t T, int64_t d, const void *W_r,
                    int n_m, int k, int mode, int dtype, float *weights,
                    float *scores, void *stream);

/*
 * mglu_forward with per-token mask weights, the forward of routed masks:
 *     out[b,j] = sum_{i<n_m} w[b,i] act(g_i[b,j]) v_i[b,j]
 * (w = 1 everywhere is mglu_forward).  mask_weights: [T][n_m] float, device,
 * 4-byte aligned; any values.  On the decode kernel (T <= the decode limit)
 * a mask whose weight is 0 for every token of the call skips its products,
 * so top-k routing with k < n_m does less arithmetic (the weights and mask
 * bits are still read once).  Other arguments and errors as mglu_forward.
 */
int mglu_forward_weighted(const void *x, int64_t T, int64_t d, const void *W,
                          int64_t h, const uint8_t *packed, int n_m, int act,
                          int dtype, const float *mask_weights, void *out,
                          void *scratch, size_t scratch_bytes, void *stream);

/*
 * The routed forward in one call: the router of mglu_route_topk (same
 * scores, same selection, same weights, bit for bit), then
 * mglu_forward_weighted with those weights.  On the decode kernel (T up to
 * the decode limit, MGLU_BF16) the router runs inside the forward kernel:
 * every CTA routes the call's tokens itself while its first weight copies
 * are in flight, so the step is one launch (plus the row-block finisher)
 * instead of two; otherwise the two calls run in turn.
 *   W_r [n_m][d], k, mode: as mglu_route_topk;
 *   weights [T][n_m] float (required), scores [T][n_m] float (or NULL):
 *   written, as mglu_route_topk writes them;
 *   other arguments as mglu_forward_weighted.
 * Errors: as mglu_route_topk and mglu_forward_weighted.
 */
int mglu_forward_routed(const void *x, int64_t T, int64_t d, const void *W,
                        int64_t h, const uint8_t *packed, int n_m,
                        const void *W_r, int k, int mode, int act, int dtype,
                        float *weights, float *scores, void *out,
                        void *scratch, size_t scratch_bytes, void *stream);

/*
 * The partial sums behind mglu_forward's output, for checking the
 * decomposition ("Masked Gated Linear Unit", "Approach": each mask splits W
 * into a gate part M_i . W and a value part (1 - M_i) . W):
 *   D[b,j]   = sum_k x[b,k] W[j,k]
 *   g_i[b,j] = sum_k x[b,k] M_i[j,k] W[j,k]
 *   v_i[b,j] = sum_k x[b,k] (1 - M_i[j,k]) W[j,k]
 * computed by the decode kernel (fp32 accumulation, as mglu_forward) and
 * written unrounded as float32 planes partials[2*n_m + 1][T][h]: plane 0 is
 * D, plane 1 + 2i is g_i, plane 2 + 2i is v_i.  g_i + v_i equals D up to
 * float32 rounding.
 *   Arguments as mglu_forward with dtype MGLU_BF16 (alignment, d % 8);
 *   partials: device, 16-byte aligned.  T must be in 0..16 (the decode
 *   kernel), else MGLU_ERR_UNSUPPORTED.  scratch as for mglu_forward.
 */
int mglu_forward_partials(const void *x, int64_t T, int64_t d, const void *W,
                          int64_t h, const uint8_t *packed, int n_m,
                          float *partials, void *scratch, size_t scratch_bytes,
                          void *stream);

/*
 * The FFN down-projection alone, a dense product (MGLU replaces only the two
 * GLU projections; "Masked Gated Linear Unit", "Problem"):
 *   y[b,c] = sum_j hid[b,j] * W_down[c,j]
 *   hid [T][h], W_down [d][h], y [T][d], scratch: mglu_scratch_bytes(d).
 * bf16 requirements: 16-byte aligned pointers, h % 8 == 0.
 */
int mglu_down_proj(const void *hid, int64_t T, int64_t h, const void *W_down,
                   int64_t d, int dtype, void *y, void *scratch,
                   size_t scratch_bytes, void *stream);

/* Workspace bytes mglu_forward_down needs: the decode scratch for
 * max(d, h) rows (mglu_scratch_bytes) at the START of the workspace, then the
 * hidden activation [T][h] in the path's dtype (rounded up to 256 bytes).
 * The scratch's place does not depend on T, so one workspace serves calls of
 * any token count; like the scratch, it needs no initialization. */
size_t mglu_workspace_bytes(int64_t T, int64_t d, int64_t h, int n_m, int dtype);

/*
 * The FFN block: y = MGLU(x) W_down^T ("Masked Gated Linear Unit", "Problem":
 * the GLU is the gated half of a transformer FFN, followed by its dense
 * down-projection).  The hidden activation is written to
 * the workspace after the decode scratch (dtype of the path; bf16 rounding
 * happens once, as in mglu_forward) and then multiplied by W_down, both on
 * `stream`.  workspace: device, 16-byte aligned, workspace_bytes >=
 * mglu_workspace_bytes(...) (else INVALID / ALIGN).
 */
int mglu_forward_down(const void *x, int64_t T, int64_t d, const void *W,
                      int64_t h, const uint8_t *packed, int n_m, int act,
                      int dtype, const void *W_down, void *workspace,
                      size_t workspace_bytes, void *y, void *stream);

/* Most output rows mglu_forward_decode_static accepts. */
#define MGLU_STATIC_SCRATCH_MAX_ROWS 262144

/*
 * mglu_forward on the decode kernel, with the kernel's cross-CTA scratch
 * taken from a buffer built into the library (a static device array of
 * mglu_scratch_bytes(MGLU_STATIC_SCRATCH_MAX_ROWS) bytes, about 6 MB, which
 * the CUDA runtime places when it loads the library's device code) instead
 * of a caller buffer.  The paper has no counterpart: it is an interface
 * convenience of this library, not part of the method.
 *
 * It is meant for callers that cannot hand the library a scratch buffer: a
 * plain-C host that has no device allocator of its own, or a serving loop
 * with a fixed device-memory budget that must not allocate once it has
 * started.  No call allocates device memory: there is no cudaMalloc,
 * cudaFree or other allocating call on this path.
 *
 *   Arguments and layouts as mglu_forward with dtype MGLU_BF16 (same
 *   alignment and d % 8 rules).  T must be in 0..16 (T == 0 is a no-op),
 *   else MGLU_ERR_UNSUPPORTED.  h must be <= MGLU_STATIC_SCRATCH_MAX_ROWS,
 *   else MGLU_ERR_INVALID, with the limit stated in mglu_last_cuda_error().
 *   The decode kernel runs for every T in 1..16, whatever
 *   mglu_set_decode_max_tokens says.
 *
 * The first call on each device does the set-up: it looks up the array's
 * device address (cudaGetSymbolAddress, return code checked) and clears the
 * scratch on `stream`.  Make that first call before any stream capture.
 *
 * There is one such scratch per device, so calls that may overlap in time
 * (other streams, other host threads) race on it and give wrong results.
 * Order them on one stream.
 */
int mglu_forward_decode_static(const void *x, int64_t T, int64_t d,
                               const void *W, int64_t h, const uint8_t *packed,
                               int n_m, int act, void *out, void *stream);

/*
 * Device workspace mglu_forward_host needs: the decode scratch for max(d, h)
 * rows at its start (whether or not W_down is given, so its place never
 * moves), then a staging copy of x, the device result and, when
 * with_down != 0, the hidden activation.  0 for bad input.
 */
size_t mglu_host_workspace_bytes(int64_t T, int64_t d, int64_t h, int n_m,
                                 int dtype, int with_down);

/*
 * The forward (W_down == NULL) or the FFN block (W_down != NULL) on HOST
 * activations: copies x_host [T][d] to the device, runs mglu_forward or
 * mglu_forward_down, and copies the result back to result_host ([T][h], or
 * [T][d] with W_down), all in order on `stream` (cudaMemcpyAsync, then the
 * kernels, then cudaMemcpyAsync).  W, packed and W_down are device pointers
 * as for mglu_forward.  The call returns before the copies finish:
 * x_host must stay unchanged and result_host is written when the stream
 * reaches the end of the call (synchronize before reading it).  Pinned host
 * memory (cudaHostAlloc) makes both copies asynchronous; pageable memory
 * works but the copies then block the calling thread.
 *   workspace: device, 256-byte aligned, >= mglu_host_workspace_bytes(...)
 *   (it holds the decode scratch; no initialization needed).
 * Nothing is allocated.  Errors: as mglu_forward / mglu_forward_down, plus
 * INVALID for a missing or small workspace or a NULL host pointer.
 */
int mglu_forward_host(const void *x_host, int64_t T, int64_t d, const void *W,
                      int64_t h, const uint8_t *packed, int n_m, int act,
                      int dtype, const void *W_down, void *workspace,
                      size_t workspace_bytes, void *result_host, void *stream);

/* Device workspace mglu_backward needs (0 for bad input). */
size_t mglu_backward_workspace_bytes(int64_t T, int64_t d, int64_t h, int n_m);

/*
 * The training path's backward through out = MGLU(x) for a given loss
 * gradient dout = dL/dout ("Masked Gated Linear Unit", "Limitations": the
 * masks are learned, held as FP16 logits while training; its list of prior
 * work names the straight-through estimator).  The page gives no formula;
 * the reading: the gradients of x and W are the exact derivatives of the
 * forward with the binary masks held fixed (ReLU takes the subgradient 0 at
 * 0), and a mask logit receives the loss gradient of its binary mask entry
 * unchanged (straight through):
 *     a_i = dout act'(g_i) v_i,   c_i = dout act(g_i)
 *     dx      = sum_i a_i (M_i . W)^T-product + c_i ((1 - M_i) . W)
 *     dW      = sum_i M_i . (a_i^T x) + (1 - M_i) . (c_i^T x)
 *     dlogits_i = W . ((a_i - c_i)^T x)
 *   x [T][d], W [h][d], packed, dout [T][h]: bf16 device (as mglu_forward;
 *   act without MGLU_GATE_DENSE, else UNSUPPORTED).
 *   dx [T][d], dW [h][d], dlogits [n_m][h][d]: float device, 16-byte
 *   aligned, written; dlogits may be NULL (masks held fixed).
 *   workspace: device, 256-byte aligned, >= mglu_backward_workspace_bytes.
 * The g_i are recomputed on the tensor cores and the backward's coefficients
 * formed in that kernel's epilogue (rounded to bf16); the masked operand and
 * the final masked combination are this library's kernels; the two plain
 * products over the materialised operands run on cuBLAS, which is loaded on
 * the first call and, unlike the rest of this library, allocates its own
 * handle memory then.  Errors: as mglu_forward, plus CUDA if cuBLAS cannot
 * be loaded.
 */
int mglu_backward(const void *x, int64_t T, int64_t d, const void *W,
                  int64_t h, const uint8_t *packed, int n_m, int act,
                  const void *dout, float *dx, float *dW, float *dlogits,
                  void *workspace, size_t workspace_bytes, void *stream);

/* Which kernel family mglu_forward uses for T tokens of `dtype`. */
int mglu_forward_path(int64_t T, int dtype);

/* Largest T served by the decode kernel (the rest go to the tensor-core
 * kernel).  Accepts 0..16 (0 = always the tensor-core kernel); returns the
 * previous value, or MGLU_ERR_INVALID.  Process-wide setting. */
int mglu_set_decode_max_tokens(int t);

/*
 * Synchronizes `stream`, then reads and clears the library's device status
 * word for the current device.  Kernels whose bounded waits give up record
 * MGLU_ERR_TIMEOUT there instead of hanging.  Returns MGLU_OK, an error
 * recorded by a kernel, or MGLU_ERR_CUDA if the synchronization failed.
 */
int mglu_last_device_status(void *stream);

/* Text of the last CUDA error seen by the library on this thread ("" if none). */
const char *mglu_last_cuda_error(void);

/* Number of kernels this library has launched in this process, over all
 * threads and devices (a kernel recorded into a CUDA graph counts once, when
 * it is recorded).  For counting the launches of a call: read it before and
 * after.  Never fails. */
uint64_t mglu_kernel_launches(void);

/* Static text for an mglu_status value. */
const char *mglu_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MGLU_H */
