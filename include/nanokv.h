/*
 * nanokv.h -- C ABI of the NanoKV compressed-history attention library
 * (libnanokv.so, CUDA, sm_100a).
 *
 * Source method: "NanoKV: High-Ratio KV Cache Compression for Autoregressive
 * Video Generation" (arXiv 2611.06377).  Historical keys and values are stored
 * per token as a cluster-center id plus INT4 joint head-channel residual
 * coefficients with a per-token scale, under a linear decoder (abstract;
 * Fig. 4(a,b)).  Attention of a new chunk's queries reads that history either
 * fully decoded (NanoKV) or, for history that a fixed policy routes to low
 * dimension, against the coefficients with reduced queries (NanoKV-Fast,
 * Fig. 4(d)); branch outputs are combined by log-sum-exp merging.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or retains them.  Scratch memory is passed in as
 *    `workspace` where needed.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and never synchronises.
 *  - Joint dimension J = H * d.  Head h owns joint columns [h*d, (h+1)*d).
 *  - Row-major layouts, no padding between rows.  Every pointer must be
 *    16-byte aligned.
 *  - Codes: r INT4 values per token packed two per byte, code 2i in the low
 *    nibble of byte i, two's complement; encode emits values in [-7, 7].
 *  - Return values are nanokv_status.  Argument errors return
 *    NANOKV_ERR_INVALID (nothing launched); shape/dtype combinations without a
 *    kernel return NANOKV_ERR_UNSUPPORTED (nothing launched); a launch failure
 *    returns NANOKV_ERR_CUDA.  nanokv_last_error() describes the last non-OK
 *    status of the calling thread.
 *  - Kernels never trap.  A kernel whose internal wait exceeds its iteration
 *    bound records that in a device error word and returns early;
 *    nanokv_check() reports it as NANOKV_ERR_TIMEOUT.
 */
#ifndef NANOKV_H
#define NANOKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  NANOKV_OK = 0,
  NANOKV_ERR_INVALID = -1,
  NANOKV_ERR_UNSUPPORTED = -2,
  NANOKV_ERR_CUDA = -3,
  NANOKV_ERR_TIMEOUT = -4
} nanokv_status;

typedef enum { NANOKV_F32 = 0, NANOKV_F16 = 1, NANOKV_BF16 = 2 } nanokv_dtype;

/*
 * One codec: per layer and per K or V branch (Table 5: rank per layer per K/V
 * branch; centers fitted separately for K and V).  All pointers are device
 * pointers in `param_dtype`.
 *   centers [C, J]  cluster centers (Fig. 4(a,b): shared content)
 *   D       [J, r]  linear decoder (Fig. 4(b): reconstructs the residual)
 *   E       [r, J]  linear encoder (Fig. 4(b): residual -> coefficients);
 *                   may be NULL for calls that do not encode.
 *   aux     optional device buffer of derived encode tables written by
 *           nanokv_codec_prepare (fp32 E c_j for every center and |c_j|^2);
 *           NULL is allowed.  nanokv_encode uses its tensor-core kernel only
 *           when aux is present, and the fp32 CUDA-core kernel otherwise.
 * Constraints: 1 <= C <= 256; r even, 2 <= r <= 512; d in {16, 32, 64, 128}.
 * Precision modes: param_dtype = scale_dtype = F32 (fp32 everywhere), or
 * param_dtype = BF16 with scale_dtype = F16.
 */
typedef struct {
  int32_t H, d, r, C;
  int32_t param_dtype; /* nanokv_dtype */
  int32_t scale_dtype; /* nanokv_dtype */
  const void *centers;
  const void *D;
  const void *E;
  const void *aux;
} nanokv_codec;

/* Bytes of the codec's derived encode tables (C*r + C fp32 values, padded). */
size_t nanokv_codec_aux_bytes(const nanokv_codec *c);

/*
 * nanokv_codec_prepare -- fill `aux` (device, 16-byte aligned, at least
 * nanokv_codec_aux_bytes bytes) with the tables the tensor-core encode reads:
 * EC[j][k] = sum_i E[k][i] c_j[i] (fp32, [C][r]) and |c_j|^2 (fp32, [C]).
 * The encode of Fig. 4(b) projects y = E (x - c_a); the tensor-core encode
 * forms it as E x - EC[a] and finds the nearest center through |c_j|^2 -
 * 2 x.c_j.  The tables depend on the codec only, so a caller prepares once
 * per codec and stores the pointer in nanokv_codec.aux; they are summed in a
 * fixed order, the same on every call.  Needs E.  Asynchronous on stream.
 */
int nanokv_codec_prepare(const nanokv_codec *c, void *aux, void *stream);

/* One branch of compressed history, T tokens in time order (oldest first).
 *   ids    [T]        uint8 center id (values >= C are read as C - 1)
 *   codes  [T, r/2]   packed INT4 coefficients
 *   scales [T]        per-token scale in the codec's scale_dtype            */
typedef struct {
  const uint8_t *ids;
  const uint8_t *codes;
  const void *scales;
} nanokv_hist;

/*
 * nanokv_encode -- compress T tokens of K and of V (Fig. 4(b); abstract).
 * For each token x (J values in x_dtype, which must equal the codec's
 * param_dtype):
 *   a = argmin_j |x - c_j|^2            (squared Euclidean, ties -> lowest j)
 *   y = E (x - c_a)                     (r coefficients)
 *   s = scale_dtype(max_i |y_i| / 7)    (round to nearest even)
 *   code_i = clamp(rint(y_i / s), -7, 7), all zero when s == 0
 * Inputs k, v [T, J]; outputs ids_* [T], codes_* [T, r/2], scales_* [T].
 * Either branch may be skipped by passing its codec as NULL (then its input
 * and outputs are ignored).  T = 0 is a no-op.
 * Kernels: bf16 codecs with aux, J a multiple of 64, C a multiple of 16
 * (16..256) and r a multiple of 64 up to 384 run on the tensor cores (a
 * 2-CTA kernel per 128 tokens for C <= 64 and r in {64, 128, 192}, a
 * multi-pass kernel otherwise); every other codec runs on the fp32 CUDA-core
 * kernel.  Both branches share one launch when their shapes agree.
 */
int nanokv_encode(const nanokv_codec *ck, const nanokv_codec *cv,
                  const void *k, const void *v, int32_t x_dtype, int64_t T,
                  uint8_t *ids_k, uint8_t *codes_k, void *scales_k,
                  uint8_t *ids_v, uint8_t *codes_v, void *scales_v,
                  void *stream);

/*
 * nanokv_attend -- attention of a query chunk over compressed history plus
 * the current uncompressed chunk (Fig. 4(a) full-dim decode-attention;
 * Fig. 4(d) fixed routing to full or low dimension and LSE merging).
 *   q      [Tq, H, d] in io_dtype (= codec param_dtype)
 *   hk, hv compressed history of T tokens.  Fixed routing policy: the most
 *          recent T_full tokens (indices [T - T_full, T)) use full-dim
 *          decode-attention, K_hat = c_K[a] + s D_K code, decoded on chip and
 *          never written to memory; the older T - T_full tokens use low-dim
 *          attention: per head h, scores tau (s (D_{K,h}^T q) . code +
 *          c_{K,a,h} . q), output (sum p c_{V,a,h} + D_{V,h} sum p s code) / sum p.
 *          The two forms compute the same attention (the low-dim one only
 *          reorders the contraction).  When the tensor-core kernels have no
 *          low-dim kernel for the codec shape (r > 192 or C > 64) but have the
 *          full-dim one, the low-dim tokens are attended with the full-dim
 *          kernel as well (kernel paths 0 and 2; path 1 keeps the routing).
 *   k_cur, v_cur [T_cur, H, d] current chunk in io_dtype (may be NULL if T_cur = 0)
 *   softmax_scale tau (callers normally pass 1/sqrt(d)); no mask.
 *   out    [Tq, H, d] in io_dtype.  lse_out [H, Tq] fp32 natural-log LSE, or NULL.
 *   Rows with no keys at all get out = 0 and lse = -inf.
 *   workspace: device scratch of at least nanokv_attend_workspace(...) bytes,
 *   16-byte aligned; contents on entry are ignored.
 * ck and cv must share H, d, param_dtype and scale_dtype; r and C may differ.
 */
int nanokv_attend(const void *q, int32_t io_dtype, int64_t Tq,
                  const nanokv_codec *ck, const nanokv_codec *cv,
                  const nanokv_hist *hk, const nanokv_hist *hv,
                  int64_t T, int64_t T_full,
                  const void *k_cur, const void *v_cur, int64_t T_cur,
                  float softmax_scale, void *out, float *lse_out,
                  void *workspace, size_t workspace_bytes, void *stream);

/*
 * nanokv_attend_static -- nanokv_attend without a workspace argument, for
 * callers that cannot allocate device memory: for example code that runs
 * where the CUDA allocator must not be entered (it can synchronise the device
 * and take process-wide locks), or a plug-in that is handed only its input and
 * output buffers by a host that owns the whole memory pool.  (The pages have no
 * counterpart; this is a property of the library, not of the method.)
 * Arguments and results are those of nanokv_attend.  The scratch lives in one
 * fixed device array of 32 MiB inside the library, which every GPU that loads
 * the library keeps until the process exits; calls whose
 * nanokv_attend_workspace(...) exceeds it return NANOKV_ERR_INVALID with a
 * message.  No allocation or free happens in this call.  The first call on a
 * device (and the first after a device reset, or under another CUDA context)
 * looks up the array's device address (cudaGetSymbolAddress) and caches it
 * with the context, so make that first call before any stream capture.  All calls share the
 * array: calls that may overlap on the GPU (other streams, other threads) race
 * on it and must be serialised by the caller.  Nothing in the array needs to be
 * zero on entry; it keeps the last call's partial results.
 */
int nanokv_attend_static(const void *q, int32_t io_dtype, int64_t Tq,
                         const nanokv_codec *ck, const nanokv_codec *cv,
                         const nanokv_hist *hk, const nanokv_hist *hv,
                         int64_t T, int64_t T_full,
                         const void *k_cur, const void *v_cur, int64_t T_cur,
                         float softmax_scale, void *out, float *lse_out, void *stream);

/*
 * nanokv_attend_partial -- nanokv_attend with its output in fp32: the
 * attention of the queries over THIS call's keys (its history, routed by
 * T_full, and the current chunk if given) as a partial result (O, LSE) for
 * an LSE merge with partials over other keys (nanokv_lse_merge; Fig. 4(d)).
 * A history held in several pieces -- e.g. sharded across GPUs, one (O, LSE)
 * exchange before the merge -- attends each piece with this call and merges
 * the partials; pass the current chunk to exactly one piece.
 *   out      device [Tq, H, d] fp32, 16-byte aligned
 *   lse_out  device [H, Tq] fp32, required
 * Everything else (arguments, workspace = nanokv_attend_workspace, errors)
 * is as for nanokv_attend.
 */
int nanokv_attend_partial(const void *q, int32_t io_dtype, int64_t Tq,
                          const nanokv_codec *ck, const nanokv_codec *cv,
                          const nanokv_hist *hk, const nanokv_hist *hv,
                          int64_t T, int64_t T_full,
                          const void *k_cur, const void *v_cur, int64_t T_cur,
                          float softmax_scale, float *out, float *lse_out,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * nanokv_attend_routed -- nanokv_attend under a general full-dim routing
 * policy instead of "the most recent T_full tokens" (NanoKV-Fast, Table 7:
 * full-dimensional routing by recent frames, periodic anchor frames, sink
 * frames, per-layer full fallback, and head-layer pairs kept at full
 * dimension; Fig. 4(d): a fixed policy routes history to full- or
 * low-dimensional attention, the branches are LSE-merged).
 *   full, n_full  HOST array of n_full (0 <= n_full <= NANOKV_MAX_RANGES)
 *                 history token ranges [start, start + count), sorted by start,
 *                 disjoint, inside [0, T): these tokens use full-dim
 *                 decode-attention, every other history token low-dim.  A
 *                 per-layer full fallback is the single range [0, T).
 *   full_heads    HOST array of H bytes or NULL: a head with a non-zero entry
 *                 attends ALL its history tokens full-dim (a sensitive head kept
 *                 at full dimension).  Heads of both kinds in one call need the
 *                 tensor-core kernels (NANOKV_ERR_UNSUPPORTED on the CUDA-core
 *                 path).
 *   lowdim        NULL, or the heads deployed at a reduced attention dimension
 *                 (nanokv_lowdim, prepared by nanokv_lowdim_prepare): a head
 *                 with d_h[h] > 0 that is not in full_heads reads its low-dim
 *                 tokens at dimension d_h[h] instead of in the coefficient
 *                 space.  Needs the tensor-core kernels (bf16 codecs, d = 128;
 *                 NANOKV_ERR_UNSUPPORTED otherwise).
 * Everything else (arguments, layouts, the current chunk, outputs, errors) is
 * as for nanokv_attend.  The routed tokens of each branch are first gathered
 * into contiguous compressed histories in the workspace (attention does not
 * depend on the order of its keys), so the result is the attention over the
 * same key set as nanokv_attend, up to rounding (and, for reduced heads, with
 * their low-dim tokens seen through the maps).
 */
#define NANOKV_MAX_RANGES 64
typedef struct {
  int64_t start, count;
} nanokv_range;

/*
 * Reduced attention dimension per head (NanoKV-Fast, Table 6: head-layer
 * pairs deployed at d_h in {32, 64, 96, 128}; Fig. 4(d): the low-dimensional
 * branch reduces the queries and restores the output dimension; Table 8:
 * low-dimensional maps).  Head h attends its low-dim tokens through
 * orthonormal maps U_h (queries and keys) and W_h (values and the output
 * restore), each [d, d_h]:
 *     q~ = U_h^T q,   k~_t = U_h^T c_K[a_t] + s_t (U_h^T D_K,h) code_t,
 *     v~_t likewise with W_h,   o~ = softmax(tau q~ k~^T) v~,   O = W_h o~.
 * The stored coefficients decode straight into d_h dimensions through the
 * mapped decoder rows and centers.  Fields (d = 128, bf16 codecs only):
 *   d_h   HOST array [H]: 0 (not reduced), 32, 64 or 96.  A head kept at the
 *         full 128 dimensions goes in full_heads instead.
 *   U, W  device [H, d, d] row-major bf16, 16-byte aligned, caller-owned:
 *         head h's map in columns [0, d_h[h]) of U[h] / W[h] (the leading
 *         columns, so maps ordered by importance serve every d_h).
 *   aux   device buffer of nanokv_lowdim_aux_bytes() bytes, 16-byte aligned,
 *         caller-owned: the mapped decoder rows and centers of both branches,
 *         written by nanokv_lowdim_prepare; valid while U, W and the codecs'
 *         D / centers are unchanged.
 */
typedef struct {
  const int32_t *d_h;
  const void *U, *W;
  void *aux;
} nanokv_lowdim;

/* Bytes of nanokv_lowdim.aux for these codecs (0 if they have no reduced
 * path: not bf16, d != 128, or K and V disagree on H or r). */
size_t nanokv_lowdim_aux_bytes(const nanokv_codec *ck, const nanokv_codec *cv);

/* Analytical maps (Table 8, "analytical initialization" of the
 * low-dimensional maps): maps[h] [d, d] row-major bf16 holds, as its columns,
 * the left singular vectors of the head's decoder rows D_h = rows
 * [h*d, (h+1)*d) of c->D, by decreasing singular value, so that its leading
 * d_h columns span the best rank-d_h approximation of D_h's column space
 * (Eckart-Young).  Pass ck for U and cv for W.  Computed on the GPU as the
 * eigenvectors of D_h D_h^T (cyclic Jacobi, fp32); the sign of each column
 * is arbitrary (attention does not depend on it).  maps: device, H*d*d bf16,
 * 16-byte aligned, caller-owned.  bf16 codecs with d = 128 only. */
int nanokv_lowdim_analytic(const nanokv_codec *c, void *maps, void *stream);

/*
 * nanokv_calibrate -- fit one branch's codec on a calibration chunk, the step
 * before encode (Table 5: centers fitted separately for K and V; Table 2:
 * joint PCA with INT4 coefficients, then shared centers; Fig. 3(a): joint
 * head-channel PCA retains the most KV variance at matched compression).
 *   1. `rounds` Lloyd k-means rounds from init_centers: every token to its
 *      nearest center (squared Euclidean over the joint J = H*d channels,
 *      ties to the lowest index), every center to the mean of its tokens (a
 *      center without tokens stays); then the final assignment (ids_out).
 *   2. D = the r leading eigenvectors, by decreasing eigenvalue, of the
 *      residual second moment (1/N) sum_t rho_t rho_t^T, rho_t = x_t -
 *      c_{a_t}; each column's largest-magnitude entry positive; E = D^T.
 *   x             device [N, J] in dtype (F32 or BF16), 16-byte aligned
 *   init_centers  device [C, J] fp32 (the caller's choice, e.g. C tokens)
 *   centers_out   device [C, J], D_out [J, r], E_out [r, J], in dtype
 *   ids_out       device [N] u8 or NULL; eigenvalues_out device [r] fp32 or NULL
 *   workspace     device, nanokv_calibrate_workspace(N, J, C) bytes
 * J a multiple of 32 up to 3072, C <= 256, 1 <= r <= J.  All work is fp32
 * on the GPU: k-means kernels, a tiled second-moment kernel and cyclic
 * Jacobi rotations (three launches per round of J/2 disjoint pairs).  The
 * call synchronises `stream` once per Jacobi sweep to test convergence (so
 * it cannot be captured in a CUDA graph) and returns when the work is done.
 * Eigenvectors of (nearly) equal eigenvalues are determined only as a
 * subspace.  Errors: NANOKV_ERR_INVALID / _UNSUPPORTED before any launch,
 * NANOKV_ERR_CUDA on a CUDA error.
 */
size_t nanokv_calibrate_workspace(int64_t N, int32_t J, int32_t C);
int nanokv_calibrate(const void *x, int32_t dtype, int64_t N, int32_t J, int32_t C, int32_t r,
                     const float *init_centers, int32_t rounds, void *centers_out, void *D_out,
                     void *E_out, uint8_t *ids_out, float *eigenvalues_out, void *workspace,
                     size_t workspace_bytes, void *stream);

/* Writes ld->aux from the maps and the codecs (all d mapped rows of every
 * head, so any d_h can use them): asynchronous on `stream`; NANOKV_OK, or
 * NANOKV_ERR_INVALID / NANOKV_ERR_UNSUPPORTED before anything is launched. */
int nanokv_lowdim_prepare(const nanokv_codec *ck, const nanokv_codec *cv, const nanokv_lowdim *ld,
                          void *stream);

int nanokv_attend_routed(const void *q, int32_t io_dtype, int64_t Tq,
                         const nanokv_codec *ck, const nanokv_codec *cv,
                         const nanokv_hist *hk, const nanokv_hist *hv, int64_t T,
                         const nanokv_range *full, int32_t n_full, const uint8_t *full_heads,
                         const nanokv_lowdim *lowdim,
                         const void *k_cur, const void *v_cur, int64_t T_cur,
                         float softmax_scale, void *out, float *lse_out,
                         void *workspace, size_t workspace_bytes, void *stream);

/* Workspace bytes nanokv_attend_routed needs (0 for invalid arguments). */
size_t nanokv_attend_routed_workspace(int64_t Tq, const nanokv_codec *ck, const nanokv_codec *cv,
                                      int64_t T, const nanokv_range *full, int32_t n_full,
                                      const uint8_t *full_heads, const nanokv_lowdim *lowdim,
                                      int64_t T_cur);

/* Workspace bytes nanokv_attend needs for these sizes (0 is possible). */
size_t nanokv_attend_workspace(int64_t Tq, const nanokv_codec *ck, const nanokv_codec *cv,
                               int64_t T, int64_t T_full, int64_t T_cur);

/*
 * nanokv_lse_merge -- merge n partial attention results over disjoint key sets
 * (Fig. 4(d): LSE merging):  LSE = log sum_i exp(LSE_i),
 * O = sum_i exp(LSE_i - LSE) O_i.  Parts with LSE_i = -inf contribute nothing;
 * rows where every part is -inf get O = 0, LSE = -inf.
 *   o_parts[i]   device [Tq, H, d] fp32      lse_parts[i] device [H, Tq] fp32
 *   o_parts / lse_parts are HOST arrays of n device pointers, 1 <= n <= 8.
 *   out [Tq, H, d] in out_dtype (F32 or BF16); lse_out [H, Tq] fp32 or NULL.
 */
int nanokv_lse_merge(int32_t n, const float *const *o_parts, const float *const *lse_parts,
                     int64_t Tq, int32_t H, int32_t d, void *out, int32_t out_dtype,
                     float *lse_out, void *stream);

/* Kernel family selection: 0 = automatic (tensor-core kernels where the shape
 * has one, fp32 CUDA-core kernels otherwise), 1 = fp32 CUDA-core kernels only,
 * 2 = tensor-core kernels only (NANOKV_ERR_UNSUPPORTED where none exists).
 * Process-wide; returns the previous value, or -1 for an invalid argument. */
int nanokv_set_kernel_path(int32_t path);

/* Reads (and clears) the device error word after synchronising `stream`:
 * NANOKV_OK, NANOKV_ERR_TIMEOUT if a kernel gave up on a bounded wait, or
 * NANOKV_ERR_CUDA if the stream reports an error. */
int nanokv_check(void *stream);

/* Number of history tokens nanokv_attend attends on the full-dim path for
 * these codecs under the current kernel path (T_full as given, or T when the
 * low-dim tokens are attended with the full-dim kernel; see nanokv_attend).
 * For work accounting and planning; -1 for invalid arguments. */
int64_t nanokv_attend_full_tokens(const nanokv_codec *ck, const nanokv_codec *cv, int64_t T,
                                  int64_t T_full);

/* Failure-detection self-test (diagnostic; the method has no counterpart).
 * Launches one small kernel on `stream` that waits on an mbarrier nothing
 * arrives on, gives up after about `limit_ns` nanoseconds (clamped to
 * [1e6, 2e9]) exactly as every pipeline wait of the attention and encode
 * kernels does on expiry, records the timeout in the device error word and
 * returns.  The next nanokv_check() on that stream then reports
 * NANOKV_ERR_TIMEOUT and clears the word; the CUDA context stays usable.
 * Returns NANOKV_OK once launched, NANOKV_ERR_CUDA on a launch error. */
int nanokv_selftest_wait(uint64_t limit_ns, void *stream);

/* Message for the calling thread's last non-OK status ("" if none). */
const char *nanokv_last_error(void);

/* Kernel identities for the diagnostics below. */
typedef enum {
  NANOKV_K_ENCODE = 0,   /* encode (one launch per K or V branch)           */
  NANOKV_K_FULL = 1,     /* full-dim decode-attention                       */
  NANOKV_K_LOW = 2,      /* low-dim attention (incl. its query prep)        */
  NANOKV_K_DENSE = 3,    /* attention over the current uncompressed chunk   */
  NANOKV_K_MERGE = 4,    /* LSE merge                                       */
  NANOKV_K_COUNT = 8
} nanokv_kernel_id;

/* Diagnostics.  nanokv_timing_enable(1) makes every later kernel launch record
 * a pair of CUDA events on its own stream (the library creates and reuses the
 * events; no device memory).  nanokv_timing_read() waits for the recorded
 * events, writes per-kernel total milliseconds and launch counts into the
 * caller's arrays of NANOKV_K_COUNT entries (either may be NULL), and clears
 * the record.  Launch counts are kept even when timing is off. */
int nanokv_timing_enable(int32_t on);
int nanokv_timing_read(double *ms_total, int64_t *launches);

/* Library version string. */
const char *nanokv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NANOKV_H */
