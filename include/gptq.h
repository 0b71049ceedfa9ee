/*
 * gptq.h -- C ABI of libgptq.so, the per-layer GPTQ quantizer for NVIDIA B200
 * (sm_100a).
 *
 * What it computes (GPTQ overview page, robocikowo.com/technologie-ai/gptq):
 *   "Jak działa"      each linear layer is quantized on its own: H = 2 X X^T
 *                     from the layer's input activations; weights quantized
 *                     column by column in a fixed order; after each column the
 *                     not-yet-quantized weights are corrected by the Optimal
 *                     Brain Surgeon rule through the inverse Hessian; block
 *                     updates; 4- or 3-bit weights with a scale per group.
 *   "Komponenty"      the Cholesky factorisation of the inverse Hessian.
 *   "Hiperparametry"  bit width, weights per scale, activation order, value
 *                     added to the Hessian diagonal.
 * and the calibration flow of the torchao issue "GPTQ implementation with
 * tensor subclasses" ("Background": gather the activations reaching a linear,
 * update its weight, use the updated weight for its outputs).
 *
 * Conventions shared by every call:
 *   - Pointers are DEVICE pointers unless a parameter says "host".  The caller
 *     owns every buffer.  No call allocates device memory for its data (the
 *     workspace is the caller's).  The only allocations are made by the CUDA
 *     runtime on the library's behalf: the module's static data (the device
 *     status word; the static scratch of gptq_quantize_static_scratch) when its
 *     device code is first loaded on a device, the instantiation of a cached
 *     CUDA graph the first time gptq_prepare / gptq_quantize /
 *     gptq_quantize_q4k meet a new set of arguments (at most 16 are kept),
 *     and one pinned host word (cudaMallocHost) per cached graph and per
 *     calling thread for the status gptq_prepare reads back.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are stream-ordered and asynchronous unless stated.
 *   - Matrices are row-major.  W is [d_out, d_in] (PyTorch Linear layout; a
 *     "column" is an input channel).  X is [n_tokens, d_in].
 *   - Arguments are validated on the host before any launch; an invalid
 *     argument returns GPTQ_ERR_INVALID_ARG and launches nothing.
 *   - A CUDA error returns GPTQ_ERR_CUDA; gptq_last_cuda_error() gives it.
 *   - Device-side waits are bounded; a wait that runs out records
 *     GPTQ_ERR_TIMEOUT in the device status word (see gptq_device_status()).
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GPTQ_OK = 0,
    GPTQ_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or option        */
    GPTQ_ERR_NOT_PD = 2,      /* damped Hessian not positive definite          */
    GPTQ_ERR_NONFINITE = 3,   /* NaN/Inf met in H                              */
    GPTQ_ERR_CUDA = 4,        /* a CUDA runtime call failed                    */
    GPTQ_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up            */
    GPTQ_ERR_WORKSPACE = 6,   /* workspace pointer NULL/misaligned or too small */
    GPTQ_ERR_UNSUPPORTED = 7, /* device is not sm_100                          */
    GPTQ_ERR_NO_MEMORY = 8    /* the static scratch could not be created (only
                                 gptq_quantize_static_scratch)                 */
} gptq_status;

/* Static English text for a status code.  Never NULL. */
const char *gptq_status_string(int status);

/* Text of the last CUDA error seen by this library in this thread ("" if none). */
const char *gptq_last_cuda_error(void);

/* ABI version: major * 10000 + minor * 100 + patch. */
int gptq_version(void);

/* Number of kernels this library has launched in this process (all devices,
 * all threads).  Lets callers count device work without a profiler. */
uint64_t gptq_launch_count(void);

/* Reads and clears the device status word of the current device: 0 or the
 * first gptq_status a kernel recorded (a timed-out wait, an invalid pivot).
 * Synchronises the current device. */
int gptq_device_status(void);

/* Bytes of workspace gptq_prepare (d_in) and gptq_quantize (d_out, d_in,
 * block_size, with or without an activation order) need for their fastest
 * path; the maximum of the two is safe for both.  The workspace must be
 * 256-byte aligned.  Returns 0 for invalid sizes. */
size_t gptq_workspace_bytes(int64_t d_out, int64_t d_in, int block_size);

/* The smallest workspace the two calls accept (same arguments and rules).
 * gptq_quantize with less than gptq_workspace_bytes but at least this much
 * forms the tf32 low parts of its lazy-batch operands inside the products
 * instead of keeping them in the workspace (same results, somewhat slower).
 * Returns 0 for invalid sizes. */
size_t gptq_workspace_min_bytes(int64_t d_out, int64_t d_in, int block_size);

/*
 * H += 2 * X^T X   ("Jak działa": H = 2 X X^T; "Złożoność obliczeniowa":
 * O(N_calib d^2)).  Call it once per calibration chunk; H accumulates across
 * calls, so a saved H is a resumable checkpoint.
 *
 *   H         float32 [d_in, d_in], IN/OUT, full symmetric matrix.  The caller
 *             zero-initialises it before the first chunk.  On return both
 *             triangles hold the sum (bitwise symmetric).  16-byte aligned.
 *             While the call runs, the strictly lower triangle is scratch
 *             (ordering counters); it is rewritten from the upper triangle
 *             before the call's work on `stream` ends.  The sums are added in
 *             a fixed order, so the same H and X give the same bits every run.
 *   X         bfloat16 bit patterns [n_tokens, d_in], row-major, 16-byte
 *             aligned.  Products of bf16 values are exact; sums are float32
 *             (tensor cores, tcgen05 kind::f16, accumulating in TMEM).
 *   n_tokens  >= 0 (0 is a no-op).
 *   d_in      > 0, multiple of 8 (TMA row pitch), <= 65536.
 */
int gptq_hessian_accumulate(float *H, const uint16_t *X, int64_t n_tokens, int64_t d_in,
                            void *stream);

/*
 * Same as gptq_hessian_accumulate with X in HOST memory: the rows are copied
 * in chunks of `chunk_tokens` through two caller-owned device staging buffers
 * while earlier chunks are accumulated, so the copy overlaps the tensor-core
 * work.  X_host should be page-locked for the copies to be asynchronous.
 * The copies run on a copy stream of the library.  When `staging` is the
 * buffer the previous call on the device used, they wait only for that
 * call's accumulations (the buffer's last readers), not for all earlier work
 * on `stream`: the uploads of one layer's activations overlap the previous
 * layer's factorisation and column loop.  With another buffer, or inside a
 * stream capture, they wait for the earlier work on `stream`.  The
 * accumulations into H stay in the order of `stream`.
 *
 *   X_host        host bf16 bit patterns [n_tokens, d_in].
 *   staging       device buffer of 2 * chunk_tokens * d_in uint16, 16-byte
 *                 aligned, used by nothing but this function while any of
 *                 its calls may be in flight.
 *   chunk_tokens  > 0.
 * Returns after all copies and kernels are enqueued; the host buffer must stay
 * valid until `stream` has finished them.
 */
int gptq_hessian_accumulate_host(float *H, const uint16_t *X_host, int64_t n_tokens,
                                 int64_t d_in, uint16_t *staging, int64_t chunk_tokens,
                                 void *stream);

/* Workspace bytes of gptq_hessian_accumulate_f32 for d_in and chunk_tokens
 * (0 for invalid sizes): 16 d_in^2 + 4 chunk_tokens d_in, rounded up. */
size_t gptq_hessian_f32_workspace_bytes(int64_t d_in, int64_t chunk_tokens);

/*
 * gptq_hessian_accumulate for float32 activations: H += 2 X^T X with X
 * float32 [n_tokens, d_in] on the device.  Each value is split into two bf16
 * parts, x = hi + lo + r with |r| <= 2^-18 |x|, and the bf16 tensor-core
 * Hessian of [hi | lo] (n_tokens x 2 d_in) gives every term of (hi + lo)^T
 * (hi + lo): products exact, sums in float32, so the result matches the
 * float64 2 X^T X to about 1e-5 relative (four times the tensor work of the
 * bf16 call).
 *   H             float32 [d_in, d_in], IN/OUT, symmetric; stays bitwise
 *                 symmetric.  16-byte aligned.
 *   X             float32 [n_tokens, d_in], 16-byte aligned.
 *   d_in          > 0, multiple of 8, <= 32768.
 *   chunk_tokens  tokens per pass through the workspace, 1 .. 2^30.
 *   workspace     >= gptq_hessian_f32_workspace_bytes(d_in, chunk_tokens)
 *                 bytes of device memory, 256-byte aligned, not used by
 *                 anything else until `stream` has finished this call.
 * Stream-ordered.  GPTQ_ERR_WORKSPACE when the workspace is missing or small.
 */
int gptq_hessian_accumulate_f32(float *H, const float *X, int64_t n_tokens, int64_t d_in,
                                int64_t chunk_tokens, void *workspace, size_t ws_bytes,
                                void *stream);

/*
 * Damping, activation order and the Cholesky factor of the inverse Hessian
 * ("Hiperparametry": value added to the diagonal, quantizing columns in order
 * of activation importance; "Komponenty": Cholesky of the inverse Hessian).
 *
 *   mu = mean(diag H);  H_d = H + damp * mu * I.
 *   act_order != 0: perm = order of descending diag(H) (undamped), equal keys
 *                   in increasing column index; otherwise perm = identity.
 *   U (Hinv_chol) = the upper-triangular factor with U^T U = (P^T H_d P)^{-1},
 *                   P the permutation, i.e. rows/columns in processing order.
 *                   Computed as M = chol_lower(J P^T H_d P J), U = J M^{-1} J
 *                   (J = index reversal), all in float32.
 *
 *   H          float32 [d_in, d_in] symmetric, read only.
 *   damp       >= 0 (0.01 typical).
 *   perm       int32 [d_in], OUT: perm[k] = original column processed k-th.
 *   Hinv_chol  float32 [d_in, d_in], OUT: U, entries below the diagonal 0.
 *   workspace  >= gptq_workspace_bytes(0, d_in, 1) bytes.
 * Synchronises `stream` once to read the factorisation status.  Returns
 * GPTQ_ERR_NOT_PD if mean(diag H) <= 0 or a pivot is not positive,
 * GPTQ_ERR_NONFINITE if H holds NaN/Inf on its diagonal.  Deterministic: the
 * same H gives the same bits.  One call runs at a time per device: calls of a
 * device share its internal side streams, so a concurrent call (another host
 * thread, another stream) waits inside the library until the first returns.
 */
int gptq_prepare(const float *H, int64_t d_in, float damp, int act_order, int32_t *perm,
                 float *Hinv_chol, void *workspace, size_t ws_bytes, void *stream);

/*
 * gptq_prepare without the wait: the same work, enqueued on `stream` (the
 * same cached graph), and the factorisation status (0, GPTQ_ERR_NOT_PD or
 * GPTQ_ERR_NONFINITE, as gptq_prepare returns it) written to *status when
 * the stream reaches the end of the call.  Returns as soon as the work is
 * enqueued, so the host can enqueue the column loop while the factorisation
 * runs.  The caller reads *status after synchronising the stream; U and perm
 * are meaningful only when it is 0.
 *   status   int32, device memory or pinned host memory, 4-byte aligned,
 *            owned by the caller; must stay valid until the stream passes
 *            the call.
 * Returns GPTQ_ERR_INVALID_ARG / GPTQ_ERR_WORKSPACE for bad arguments (before
 * any launch), else GPTQ_OK.  Concurrent calls are safe: the enqueue is
 * serialised per device and each call replays its own cached graph (two
 * calls with the same buffers replay the same graph, one after the other).
 * With graphs switched off (GPTQ_GRAPHS=0) the call waits for the stream like
 * gptq_prepare, since direct launches use the device's shared side streams;
 * inside a stream capture it only enqueues.
 */
int gptq_prepare_async(const float *H, int64_t d_in, float damp, int act_order, int32_t *perm,
                       float *Hinv_chol, void *workspace, size_t ws_bytes, int *status,
                       void *stream);

/*
 * GPTQ column loop ("Jak działa"): for columns c in processing order, with a
 * new per-row (scale, zero) at each group start taken from the row's current
 * values of the group's columns (range including 0; an all-zero range is
 * [-1, 1]):
 *     s = (max - min) / (2^bits - 1),  z = rint(-min / s)
 *     q = clamp(rint(w_c / s) + z, 0, 2^bits - 1),  w^_c = s (q - z)
 *     e = (w_c - w^_c) / U[c,c],   w[c+1:] -= e * U[c, c+1:]
 * with the correction of columns beyond the current block of `block_size`
 * columns applied once per block as W[:, j+B:] -= E_blk U[j:j+B, j+B:].
 * Grid choice and rounding are decided in float32; ties round to even.
 *
 *   W           float32 [d_out, d_in] IN/OUT, original column order.  On
 *               return it holds the dequantized weights W^ (original order).
 *   Hinv_chol   U from gptq_prepare (processing order).
 *   perm        int32 [d_in] from gptq_prepare, or NULL for identity.  It must
 *               be a permutation of 0 .. d_in-1; entries out of range or
 *               columns named twice are detected on the device (status word
 *               GPTQ_ERR_INVALID_ARG, see gptq_device_status()); the outputs
 *               are then unspecified, but every access stays in bounds.
 *   bits        1..8 (2, 3, 4 are the GPTQ widths; codes are one byte each).
 *   group_size  > 0 and dividing d_in, or -1 for one (scale, zero) per row
 *               from the original row.  group_size must divide block_size or
 *               be a multiple of it.
 *   block_size  1..128, the lazy-batch width.
 *   codes       uint8 [d_out, d_in] OUT (original column order) or NULL.
 *   scales      float32 [d_out, n_groups] OUT, groups in processing order;
 *               n_groups = d_in / group_size (1 when group_size = -1).
 *   zeros       float32 [d_out, n_groups] OUT, integer-valued.
 *   packed_int4 uint8 [d_out, d_in / 2] OUT or NULL; needs bits <= 4 and even
 *               d_in: column 2i in the low nibble, 2i + 1 in the high nibble.
 *   g_idx       int32 [d_in] OUT or NULL: group of each original column.
 *   err_sq      float32 [d_out] OUT or NULL: sum over columns of e^2.
 *   workspace   >= gptq_workspace_bytes(d_out, d_in, block_size) bytes.
 */
int gptq_quantize(float *W, const float *Hinv_chol, const int32_t *perm, int64_t d_out,
                  int64_t d_in, int bits, int group_size, int block_size, uint8_t *codes,
                  float *scales, float *zeros, uint8_t *packed_int4, int32_t *g_idx,
                  float *err_sq, void *workspace, size_t ws_bytes, void *stream);

/*
 * gptq_quantize onto the two-level Q4_K grid (torchao pull request "Add gguf
 * q4_k quantization": w = q * block_scale + block_min with a 4-bit q, 6-bit
 * block scales and mins, and super-block scales above them).  Blocks of 32
 * columns and super-blocks of 256, both in processing order:
 *     w^ = d sc q - dmin m,   q in 0..15,  sc in 1..63,  m in 0..63.
 * At a super-block's first column, from each row's current (compensated)
 * values of its 256 columns: per 32-column block the range [min(0, min),
 * max(0, max)] (an all-zero block takes [-1, 1]) gives a raw scale
 * (max - min) / 15 and offset -min; d = max raw scale / 63, dmin = max raw
 * offset / 63.  At each block's first column, from the current values of its
 * 32 columns: sc = clamp(rint(scale / d), 1, 63), m = clamp(rint(offset /
 * dmin), 0, 63) (0 when dmin = 0).  Per column q = clamp(rint((w + dmin m) /
 * (d sc)), 0, 15), then the usual error feedback (lazy batch of 128).
 * Arguments as gptq_quantize (bits 4, group 32, block 128 implied), and
 *   d_in     a multiple of 256.
 *   codes    uint8 [d_out, d_in] OUT or NULL (original column order).
 *   sc6, m6  uint8 [d_out, d_in / 32] OUT, blocks in processing order.
 *   dsup, dmin  float32 [d_out, d_in / 256] OUT, super-blocks in processing order.
 *   scales, offsets  float32 [d_out, d_in / 32] OUT: the block's d sc and
 *            dmin m (w^ = scales * q - offsets).
 *   packed_int4, g_idx (block of each original column), err_sq: as gptq_quantize.
 * W holds W^ on return.
 */
int gptq_quantize_q4k(float *W, const float *Hinv_chol, const int32_t *perm, int64_t d_out,
                      int64_t d_in, uint8_t *codes, uint8_t *sc6, uint8_t *m6, float *dsup,
                      float *dmin, float *scales, float *offsets, uint8_t *packed_int4,
                      int32_t *g_idx, float *err_sq, void *workspace, size_t ws_bytes,
                      void *stream);

/* Size of the fixed device array that gptq_quantize_static_scratch works in:
 * 128 MiB.  Every GPU on which the library's device code is loaded holds it
 * from then until the process exits. */
#define GPTQ_STATIC_SCRATCH_BYTES ((size_t)128 << 20)

/*
 * gptq_quantize with no workspace argument, for callers that cannot allocate
 * device memory: a plugin inside another engine that is handed only input and
 * output pointers and has no allocator to ask; a serving loop that must not
 * pay cudaMalloc's implicit device-wide synchronisation; a process that has
 * reserved the GPU's memory up front for its own pool.  The method has no
 * counterpart to this call; it exists only for such callers.
 *
 * Arguments, outputs and results are those of gptq_quantize.  The scratch is
 * a fixed array inside the library (GPTQ_STATIC_SCRATCH_BYTES), so the call
 * allocates nothing.  Limits and rules:
 *   - A layer whose working set exceeds the array (the minimum workspace of
 *     gptq_quantize: about 5 bytes per weight plus 4 KiB per output row;
 *     4096 x 4096 needs about 102 MiB and fits, 4096 x 11008 does not) is
 *     refused with GPTQ_ERR_WORKSPACE before the device is touched.  When the
 *     array also holds the optional low-part buffers (small layers) they are
 *     used.
 *   - The first call on each device looks up the array's device address with
 *     that device current (a one-time set-up); make that first call before any
 *     stream capture begins.  CUDA loads device code lazily, so that first
 *     lookup is also when the array is created on the device: a caller that
 *     reserves the GPU's memory up front must make its first call before
 *     reserving.  If the device has no room for it the call returns
 *     GPTQ_ERR_NO_MEMORY (and leaves no CUDA error pending).
 *   - All calls share the one array, and it keeps whatever the last call left
 *     in it.  Nothing in it needs to start at zero (each call writes every byte
 *     it later reads), but two calls whose work overlaps on the GPU (different
 *     streams, or different host threads) race on it: order them on one stream
 *     or otherwise make sure one finishes before the next starts.
 */
int gptq_quantize_static_scratch(float *W, const float *Hinv_chol, const int32_t *perm,
                                 int64_t d_out, int64_t d_in, int bits, int group_size,
                                 int block_size, uint8_t *codes, float *scales, float *zeros,
                                 uint8_t *packed_int4, int32_t *g_idx, float *err_sq,
                                 void *stream);

/* Diagnostic: gptq_quantize (same arguments, rules and results) enqueued
 * directly on `stream` in its production launch sequence (programmatic
 * dependent launches included); synchronises the stream.  The column-loop
 * kernels and the tensor-core lazy-batch products record their own spans
 * (device clock, ns): each launch from its first CTA passing its wait for the
 * previous kernel to its last CTA's end.  Returns the summed spans of the
 * column-loop kernels (*loop_ms) and of the lazy-batch products (*update_ms),
 * and the rest of the call's device time (*other_ms: layout, gathers,
 * unpermute/packing and launch gaps).  One timed call runs at a time in a
 * process (the spans live in one static device array). */
int gptq_quantize_timed(float* W, const float* Hinv_chol, const int32_t* perm, int64_t d_out,
                        int64_t d_in, int bits, int group_size, int block_size, uint8_t* codes,
                        float* scales, float* zeros, uint8_t* packed_int4, int32_t* g_idx,
                        float* err_sq, void* workspace, size_t ws_bytes, void* stream,
                        float* loop_ms, float* update_ms, float* other_ms);

/* Diagnostic of the bounded waits the tensor-core kernels use: launches one
 * warp that waits on an mbarrier nothing completes, with a limit of
 * `limit_cycles` SM clocks (0 < limit <= about 2e9), and returns what the
 * device status word then holds: GPTQ_ERR_TIMEOUT when the wait gave up as
 * designed.  The device stays usable afterwards.  Synchronises the device. */
int gptq_selftest_bounded_wait(int64_t limit_cycles);

/* Diagnostic of the column loop's division-free quotient (the rounding of
 * w / s that decides each code): evaluates it on n_pairs > 0 operand pairs
 * drawn from `seed` (log-uniform scales over 2^-40 .. 2^20, scales with
 * all-ones significands, and quotients within 4 ulps of a half-integer) and
 * stores in *mismatches how many differ from IEEE round-to-nearest division.
 * Expected 0.  Uses the default stream and synchronises the device. */
int gptq_selftest_quotient(int64_t n_pairs, uint64_t seed, int64_t* mismatches);

/* Paths of gptq_w4a16_gemm. */
enum { GPTQ_W4A16_AUTO = 0, GPTQ_W4A16_TENSOR_CORE = 1, GPTQ_W4A16_GENERAL = 2, GPTQ_W4A16_DECODE = 3 };

/*
 * Y = X W^T with W^ the dequantized 4-bit weights gptq_quantize writes: the
 * consumer of its packed format (AutoGPTQ page, "Mixed Precision Scheme":
 * 4-bit weights, 16-bit activations, dequantized on the fly inside the
 * product).  W^[n][k] = scales[n][g] * (q[n][k] - zeros[n][g]) with
 * g = g_idx[k] when g_idx is given, else k / group_size (0 for group_size
 * -1); q[n][k] is nibble k of row n of `packed`.
 *   Y           float32 [M, N] OUT, row-major.
 *   X           bf16 [M, K] row-major (uint16 bit patterns), 16-byte aligned.
 *   packed      uint8 [N, K / 2]: column 2i in the low nibble of byte i,
 *               2i + 1 in the high nibble; 16-byte aligned.
 *   scales      float32 [N, n_groups], zeros float32 [N, n_groups] with
 *               integer values 0..15; n_groups = K / group_size (1 for -1).
 *   g_idx       int32 [K] or NULL (groups contiguous along K).
 *   M >= 0, N >= 0, K > 0 with K % 8 == 0; group_size -1 or dividing K.
 *   path        GPTQ_W4A16_AUTO picks the decode path for M <= 4 when it
 *               applies (g_idx NULL, K % 32 == 0, group_size a multiple of
 *               32 or -1), else the tensor-core path when it applies: g_idx
 *               NULL, K % 32 == 0, group_size dividing 128 (a multiple of 16)
 *               or a multiple of 128 or -1.  GPTQ_W4A16_TENSOR_CORE and
 *               GPTQ_W4A16_DECODE ask for their path (GPTQ_ERR_INVALID_ARG
 *               when it does not apply); GPTQ_W4A16_GENERAL takes the SIMT
 *               path for any layout.
 * Tensor-core path: Y = sum_g s * (sum over the group's columns of
 * (q - z) x), the inner sums exact bf16 products accumulated in fp32 on
 * tcgen05 (q - z is exact in bf16), the scale applied per group; split-K
 * partial sums are added in a fixed order, so results are deterministic.
 * Decode path (M <= 4): the weights streamed once with 16-byte loads, per
 * 32-column chunk the fp32 sum of (q - z) x (exact q - z), scaled once.
 * General path: fp32 W^ = s * (q - z) and fp32 dot products.  All are
 * X W^T up to fp32 rounding of the sums.  Stream-ordered; allocates nothing.
 * Y must not overlap the inputs.
 */
int gptq_w4a16_gemm(float *Y, const uint16_t *X, const uint8_t *packed, const float *scales,
                    const float *zeros, const int32_t *g_idx, int64_t M, int64_t N, int64_t K,
                    int group_size, int path, void *stream);

/* dst[i] = (float) bf16 src[i] (exact widening), n >= 0 elements. */
int gptq_bf16_to_f32(float *dst, const uint16_t *src, int64_t n, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_H */
