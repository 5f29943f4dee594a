/*
 * admmq.h -- C ABI of the B200 (sm_100a) ADMM-Q layer solve.
 *
 * The method (ADMM-Q technical summary, gist.science 2605.11222, Methodology):
 * for one linear layer with pre-trained weights W_hat (d_in x d_out) and
 * calibration activations X (n x d_in), minimise
 *     1/2 Tr((W - W_hat)^T H (W - W_hat))   s.t.  W on a per-group integer grid,
 * with H = X^T X + lambda I (section 1).  The solve scales by
 * Sigma = Diag(H)^(-1/2), eigendecomposes the scaled Hessian once, and runs
 * ADMM under rho_t = rho0 * gamma^t: an eigenbasis W-update, a D-update that
 * projects onto a per-group asymmetric grid refreshed from the current iterate,
 * and the dual update V += W - D (section 2).
 *
 * Conventions for every entry point:
 *   - Pointers named *_dev are DEVICE pointers owned by the caller; the
 *     library never frees them and keeps no reference after the call returns,
 *     except the context, which keeps the workspace pointer and the W_hat
 *     pointer given to admmq_prepare() until admmq_destroy().
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy default
 *     stream.  Calls are asynchronous on that stream unless stated otherwise.
 *   - Matrices are row-major.  W_hat and codes use the torch nn.Linear layout
 *     [d_out][d_in] (the pages' d_in x d_out matrix stored column-major).
 *     A quantization group is `group` consecutive input channels of one output
 *     row; scale/zero are [d_out][d_in / group].
 *   - Return value: ADMMQ_OK (0) or a negative ADMMQ_ERR_* code.  Nothing is
 *     launched when an argument check fails.  No exception crosses the ABI.
 *   - Sizes: d_in a multiple of 32 and of `group`; group in {32, 64, 128};
 *     bits in 1..8; d_out >= 1; n >= 0.
 */
#ifndef ADMMQ_H_
#define ADMMQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  ADMMQ_OK = 0,
  ADMMQ_ERR_INVALID_ARG = -1, /* a size, pointer or parameter is out of range   */
  ADMMQ_ERR_CUDA = -2,        /* a CUDA runtime call or kernel launch failed      */
  ADMMQ_ERR_EIG = -3,         /* the eigensolver reported failure (info != 0)    */
  ADMMQ_ERR_NOT_PD = -4,      /* a diagonal entry of H is not positive           */
  ADMMQ_ERR_NONFINITE = -5,   /* NaN/Inf found in H's diagonal or the eigenvalues */
  ADMMQ_ERR_TIMEOUT = -6,     /* a kernel's bounded pipeline wait gave up        */
  ADMMQ_ERR_WORKSPACE = -7,   /* the workspace is smaller than required          */
  ADMMQ_ERR_UNSUPPORTED = -8, /* device is not sm_100 or a shape is unsupported  */
  ADMMQ_ERR_RANGE = -9        /* an fp16-split operand left fp16's range          */
};

/* Grid refresh used by the D-update (the pages do not fix the fit). */
enum {
  ADMMQ_GRID_MINMAX = 0, /* scale/zero from the group's min/max, 0 included    */
  ADMMQ_GRID_LSQ = 1,    /* weighted least-squares refit, weights diag(H); its
                            float32 sums are taken per 32-column block in
                            element order and the block sums added pairwise */
  ADMMQ_GRID_FROZEN = 2, /* keep the start grid (RTN grid of W_hat)             */
  ADMMQ_GRID_MSE = 3     /* MSE clipping search: the min/max grid of the range
                            clipped by a = (32 - k) / 32, k < 16, whose float32
                            squared error (summed in element order) is the
                            first smallest (ADMM-Q technical summary,
                            Methodology section 3: clipping heuristics)       */
};

enum { ADMMQ_DTYPE_F32 = 0, ADMMQ_DTYPE_BF16 = 1 };

/* Split precision of the eigenbasis GEMMs (fp32-accurate products on tf32 /
 * bf16 tensor cores; see "operand encoding" below). */
enum {
  ADMMQ_SPLIT_AUTO = 0,   /* fp16 x3 from d_in >= 2048, else 3xTF32               */
  ADMMQ_SPLIT_3XTF32 = 1, /* hi.hi + hi.lo + lo.hi, three tf32 products           */
  ADMMQ_SPLIT_MIXED = 2,  /* tf32 hi.hi + one bf16 product for hi.lo + lo.hi      */
  ADMMQ_SPLIT_F16 = 3     /* hi.hi + hi.lo + lo.hi, three fp16 products on
                             power-of-two scaled operands (22 bits like 3xTF32,
                             at the full 16-bit rate)                           */
};

/* How admmq_iterate launches the iterations.  Every step of an iteration acts
 * on rows, so GEMM 1 and GEMM 2 of all the iterations of one admmq_iterate
 * call can run in one persistent launch whose tiles wait until the row block
 * they read is complete (the default: one launch and one tail per call); or
 * GEMM 1 and GEMM 2 of each iteration are launched separately.  Both give the
 * same bits.  The fused launch hands out its tiles in order from a counter
 * to whichever CTAs are running, so it needs no particular number of them
 * resident and may share the GPU with other work. */
enum {
  ADMMQ_SCHEDULE_FUSED = 0,   /* every iteration of a call in one launch      */
  ADMMQ_SCHEDULE_PER_GEMM = 1 /* two launches per iteration                   */
};

typedef struct admmq_params {
  int bits;         /* b: codes in [0, 2^b - 1]                                  */
  int group;        /* g: input channels per quantization group                 */
  int iters;        /* T: ADMM iterations                                        */
  float rho0;       /* penalty at t = 0                                          */
  float gamma;      /* penalty growth: rho_t = rho0 * gamma^t                    */
  float lambda_rel; /* damping: lambda = lambda_rel * mean(diag(X^T X))          */
  int grid_mode;    /* ADMMQ_GRID_*                                              */
  int split_mode;   /* ADMMQ_SPLIT_*                                             */
  int no_scaling;   /* 1: Sigma = I, the unscaled ablation ([ADMM-Q] Methodology
                       section 2 reports what removing the scaling costs); 0 */
  int schedule;     /* ADMMQ_SCHEDULE_*                                          */
  int rescale_dual; /* 1: after each iteration V~ *= rho_t / rho_{t+1}, so that the
                       unscaled dual rho V~ carries over when the penalty grows
                       (the pages say nothing on it; a variant for study); 0
                       (default): V~ += W~ - D~ only                             */
  int fit_on_w;     /* 1: refresh the grid from Sigma W~ and round Sigma (W~ + V~)
                       onto it (the pages' "current continuous iterate" read as
                       W~; a variant for study); 0 (default): fit the grid on
                       the point being projected, Sigma (W~ + V~)               */
} admmq_params;

typedef struct admmq_ctx admmq_ctx; /* opaque; host memory owned by the library */

/* Status code -> static English string (never NULL). */
const char* admmq_status_string(int status);

/* Library ABI version (major * 100 + minor). */
int admmq_version(void);

/* Number of CUDA kernels this library has launched in this process (all
 * devices, all contexts); cuSOLVER's own kernels are not counted. */
int64_t admmq_launch_count(void);

/* ---------------------------------------------------------------- Hessian --
 * Gram of the calibration activations, H = X^T X  (ADMM-Q summary, Methodology
 * section 1: H = X^T X + lambda I; damping is added later by admmq_prepare).
 *   X_dev      bf16 [n][d_in], row-major (token-major), 16-byte aligned.
 *   H_dev      fp32 [d_in][d_in]; written in full (both triangles), or, with
 *              accumulate != 0, the Gram of this chunk is added to its contents
 *              (so X may be streamed in chunks of tokens).
 *   ws_dev     scratch of at least admmq_gram_workspace_bytes(n, d_in) bytes.
 * bf16 products are exact in fp32; sums are fp32 (tensor cores), combined in a
 * fixed order, so the result is deterministic for a given device and shape.
 * Failure: the Gram kernel's pipeline waits are bounded; one that gives up
 * sets the int32 status word at the start of ws_dev (non-zero) and the Gram
 * writes NaN on the diagonal of H, so admmq_prepare() on that H returns
 * ADMMQ_ERR_NONFINITE. */
size_t admmq_gram_workspace_bytes(int64_t n, int d_in);
int admmq_build_hessian(const void* X_dev, int64_t n, int d_in, float* H_dev, int accumulate,
                        void* ws_dev, size_t ws_bytes, void* stream);

/* No-allocation variant of admmq_build_hessian (the pages have no counterpart:
 * this is an interface for callers, not a step of the method).
 * Some callers cannot allocate device memory at the moment they need the
 * Hessian: a serving or training framework that has already reserved all
 * device memory for its own pool, or code on a latency-bound path that must
 * not call cudaMalloc (which can synchronise the whole device).  This entry
 * point takes no workspace: its scratch (the k-split
 * partial sums and a status word) lives in one file-scope device array of
 * ADMMQ_STATIC_SCRATCH_BYTES, which every GPU that loads the library holds
 * until the process exits.  It computes the same X^T X as
 * admmq_build_hessian (same kernels; the k-split count may be smaller so that
 * the partials fit, which only changes the order of fp32 additions).
 *   Limit: 256 + d_in * d_in * 4 bytes must fit in ADMMQ_STATIC_SCRATCH_BYTES
 *   (d_in <= 4096); larger d_in returns ADMMQ_ERR_WORKSPACE before anything
 *   is launched.
 *   The first call on a device looks the array's device address up
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  The address belongs to the device's current
 *   CUDA context: after cudaDeviceReset, or any other teardown and re-creation
 *   of that context, the next call looks it up again (and counts as a first
 *   call once more).  Nothing is allocated, here or later.
 *   Failure: the status word lives in the library's array, out of the
 *   caller's reach; a Gram whose bounded waits gave up is reported by NaN on
 *   the diagonal of H, which admmq_prepare() turns into ADMMQ_ERR_NONFINITE.
 *   Speed: the partial sums of the k-split must fit the array, so from
 *   d_in = 2048 up the split count falls (to 1 at d_in = 4096) and such a
 *   call can be slower than admmq_build_hessian on the same input.
 *   All calls share the array and it keeps the last call's contents (the
 *   status word is cleared at the start of every call): calls that overlap on
 *   the GPU -- on different streams, or from different threads -- race on it
 *   and must be serialised by the caller. */
#define ADMMQ_STATIC_SCRATCH_BYTES ((size_t)64 * 1024 * 1024 + 256)
int admmq_build_hessian_static(const void* X_dev, int64_t n, int d_in, float* H_dev,
                               int accumulate, void* stream);

/* ---------------------------------------------------------------- context --
 * One context per layer solve.  ws_dev (caller-allocated device memory of at
 * least admmq_workspace_bytes() bytes) holds all solver state; the context
 * only stores pointers into it.  admmq_create() validates the parameters and
 * creates the eigensolver handle; it launches nothing. */
size_t admmq_workspace_bytes(int d_in, int d_out, const admmq_params* p);
int admmq_create(admmq_ctx** ctx, int d_in, int d_out, const admmq_params* p, void* ws_dev,
                 size_t ws_bytes);
void admmq_destroy(admmq_ctx* ctx);

/* Damping and diagonal scaling (Methodology section 1 and section 2,
 * "diagonal scaling"): lambda = lambda_rel * mean(diag G), H = G + lambda I,
 * sigma_i = H_ii^(-1/2) (1 with params.no_scaling), H~ = Sigma H Sigma
 * (float64, into the workspace) and
 * the scaled weights W^~ = Sigma^-1 W_hat as split-precision operand planes
 * (see "operand encoding" below).
 *   G_dev      fp32 [d_in][d_in], X^T X WITHOUT damping (admmq_build_hessian).
 *   W_hat_dev  [d_out][d_in], fp32 or bf16 (w_dtype); must stay valid until
 *              admmq_destroy (the objective reads it).
 * Returns ADMMQ_ERR_NOT_PD / _NONFINITE after a host sync if diag(H) is bad. */
int admmq_prepare(admmq_ctx* ctx, const float* G_dev, const void* W_hat_dev, int w_dtype,
                  void* stream);

/* One-time eigendecomposition H~ = Q Lambda Q^T (Methodology section 2,
 * W-update) with cuSOLVER's float64 divide-and-conquer solver, then the
 * split-precision operand planes of Q^T and Q.  Synchronises the stream once
 * to read the solver's info (ADMMQ_ERR_EIG if non-zero). */
int admmq_eigh(admmq_ctx* ctx, void* stream);

/* admmq_prepare + admmq_eigh. */
int admmq_setup(admmq_ctx** ctx_out, const float* G_dev, const void* W_hat_dev, int w_dtype,
                int d_in, int d_out, const admmq_params* p, void* ws_dev, size_t ws_bytes,
                void* stream);

/* Start of the iteration: C0' = Lambda Q^T W^~ (so that Q^T H~ W^~ = C0') and
 * the RTN start D_0 = RTN(W_hat) on its min/max grid, V~_0 = 0.
 *   codes_dev  u8 [d_out][d_in], 32-byte aligned (the epilogues move 32 codes
 *              per 256-bit access); scale_dev, zero_dev fp32 [d_out][d_in/group].
 * A misaligned codes_dev returns ADMMQ_ERR_INVALID_ARG (also for iterate). */
int admmq_init(admmq_ctx* ctx, uint8_t* codes_dev, float* scale_dev, float* zero_dev,
               void* stream);

/* ADMM iterations t = t0 .. t0+count-1 with rho_t = rho0 gamma^t:
 *   T  = diag(1/(Lambda+rho)) (C0' + rho Q^T (D~ - V~))          (GEMM 1)
 *   W~ = Q T;  D = grid projection of Sigma (W~ + V~);  V~ += W~ - D~  (GEMM 2
 *        with the projection, the dual update and residual sums fused)
 * codes/scale/zero are updated in place (they hold D).  t0 + count <= iters.
 * With ADMMQ_SCHEDULE_FUSED the count iterations are one kernel launch.  Its
 * waits for other units are bounded like the pipeline waits: one that gives up
 * sets the kernel status word (ADMMQ_BUF_STATUS[0] = 1, "timed out") and the
 * launch ends. */
int admmq_iterate(admmq_ctx* ctx, int t0, int count, uint8_t* codes_dev, float* scale_dev,
                  float* zero_dev, void* stream);

/* After the last iteration: the objective 1/2 Tr((D - W_hat)^T H (D - W_hat))
 * (H with damping) and the residual history.
 *   resid_dev   optional fp64 [iters][2]: ||W~_t - D~_t||_F and
 *               rho_t ||D~_t - D~_{t-1}||_F (scaled coordinates); NULL to skip.
 *   objective_dev optional fp64 [1] (device); NULL to skip. */
int admmq_finish(admmq_ctx* ctx, const uint8_t* codes_dev, const float* scale_dev,
                 const float* zero_dev, double* resid_dev, double* objective_dev, void* stream);

/* admmq_init + admmq_iterate(0, iters) + admmq_finish. */
int admmq_solve(admmq_ctx* ctx, uint8_t* codes_dev, float* scale_dev, float* zero_dev,
                double* resid_dev, double* objective_dev, void* stream);

/* Pack codes u8 [d_out][d_in] into a little-endian b-bit stream per row:
 * code k of a row occupies bits [b k, b k + b) of the row, in uint32 words;
 * packed_dev is uint32 [d_out][d_in * bits / 32].  Codes must be < 2^bits.
 * (Our reading of "same format as GPTQ", ADMM-Q summary, Experimental results
 * section 3; the pages do not define the bit layout.) */
int admmq_pack(const uint8_t* codes_dev, int d_in, int d_out, int bits, uint32_t* packed_dev,
               void* stream);

/* ------------------------------------------------------------ inspection --
 * Device buffers inside the workspace, for tests and diagnostics.
 * Operand encoding of the eigenbasis GEMMs (fp32-accurate split precision,
 * per admmq_split_mode): a matrix x [rows][K] is stored as planes HI and LO:
 *   ADMMQ_SPLIT_3XTF32: HI fp32 [rows][K] with hi = tf32(x); LO fp32
 *     [rows][K], lo = tf32(x - hi);
 *   ADMMQ_SPLIT_MIXED: HI as for 3XTF32; LO u16 [rows][2K] of bfloat16 bit
 *     patterns: per 32 columns c0..c0+31 of a row, for operands on the A side
 *     (W^~, P, T, Delta~) the 32 values bf16(hi) then the 32 values
 *     bf16(x - hi); on the B side (Q^T, Q) the two halves swapped;
 *   ADMMQ_SPLIT_F16: HI and LO u16 [rows][K] of IEEE fp16 bit patterns,
 *     hi = fp16(x s), lo = fp16(x s - hi), with s = 2^14 on the B side
 *     (|entries| <= 1) and s = ADMMQ_BUF_ROW_IN[row] on the A side: a power
 *     of two with s ||W^~_row|| in [2^9, 2^10).  A scaled A-side value at or
 *     beyond 65504 sets status word 3 (admmq_check: ADMMQ_ERR_RANGE).
 * All roundings nearest-even.  Every encoding fits 4 bytes per element per
 * plane.
 * Layouts:
 *   ADMMQ_BUF_SIGMA, _RSIG, _HDIAG, _LAMBDA : fp32 [d_in]
 *   ADMMQ_BUF_V      fp32 [d_out][d_in]  scaled dual V~
 *   ADMMQ_BUF_C0     fp32 [d_out][d_in]  C0' = Lambda Q^T W^~ (row j, column k)
 *   ADMMQ_BUF_P_HI/_P_LO  P = D~ - V~, encoded planes (A side)
 *   ADMMQ_BUF_T_HI/_T_LO  GEMM-1 output T, encoded planes (A side)
 *   ADMMQ_BUF_E_HI/_E_LO  E = Q^T (row k = k-th eigenvector of H~), encoded
 *                         planes (B side)
 *   ADMMQ_BUF_HT     fp64 [d_in][d_in]   H~ before admmq_eigh, Q^T after
 *   ADMMQ_BUF_STATUS int32 [4]           kernel status words (0 = ok): [0]
 *                    a bounded wait gave up, [1] setup, [2] eigenvalues,
 *                    [3] fp16-split range
 *   ADMMQ_BUF_ROW_IN fp32 [d_out]        A-side operand scale per row
 *                                        (1 unless ADMMQ_SPLIT_F16)
 *   ADMMQ_BUF_ROW_OUT fp32 [d_out]       factor that unscales a GEMM result
 *                                        row (1 / (ROW_IN 2^14) for fp16) */
enum {
  ADMMQ_BUF_SIGMA = 0, ADMMQ_BUF_RSIG, ADMMQ_BUF_HDIAG, ADMMQ_BUF_LAMBDA, ADMMQ_BUF_V,
  ADMMQ_BUF_C0, ADMMQ_BUF_P_HI, ADMMQ_BUF_P_LO, ADMMQ_BUF_T_HI, ADMMQ_BUF_T_LO,
  ADMMQ_BUF_E_HI, ADMMQ_BUF_E_LO, ADMMQ_BUF_HT, ADMMQ_BUF_STATUS, ADMMQ_BUF_ROW_IN,
  ADMMQ_BUF_ROW_OUT, ADMMQ_BUF_COUNT
};
int admmq_get_buffer(admmq_ctx* ctx, int which, void** ptr_dev, size_t* bytes);

/* When wtilde_dev is non-NULL, the next GEMM-2 launches also write the raw
 * fp32 product W~ [d_out][d_in] there (tests compare the fused projection with
 * its float32 specification on exactly these values).  NULL turns it off;
 * a pointer that is not 32-byte aligned returns ADMMQ_ERR_INVALID_ARG. */
int admmq_debug_dump_wtilde(admmq_ctx* ctx, float* wtilde_dev);

/* Per-kernel timing with CUDA events recorded on the launch stream around
 * every GEMM launch of admmq_iterate.  enable != 0 clears and starts it.
 * admmq_get_timing returns the summed milliseconds and launch counts of
 * GEMM 1 (index 0) and GEMM 2 (index 1), or, with ADMMQ_SCHEDULE_FUSED, of
 * the fused launches (index 0; index 1 is zero); iters_timed (optional)
 * receives the number of iterations those launches ran.  It synchronises on
 * the events. */
int admmq_set_timing(admmq_ctx* ctx, int enable);
int admmq_get_timing(admmq_ctx* ctx, double ms[2], int launches[2], int* iters_timed);

/* Standalone projection kernel (the fused GEMM-2 epilogue reading W~ from
 * memory instead of tensor memory); same per-element float32 arithmetic.
 * All pointers device; V_dev is updated in place; P is written in the
 * eigenbasis GEMMs' operand encoding of `split_mode` (ADMMQ_SPLIT_3XTF32,
 * ADMMQ_SPLIT_MIXED or ADMMQ_SPLIT_F16, A side; see "operand encoding"):
 * P_hi_dev / P_lo_dev as that encoding lays them out; row_scale_dev
 * (optional, fp32 [d_out]) is the fp16 split's per-row scale (1 when NULL);
 * range_flag_dev (optional, int32) is set to 1 when a scaled value leaves
 * fp16's range; codes/scale/zero hold the previous D on entry and the new D
 * on exit; resid_dev fp64 [2] receives the two residual sums of squares;
 * dual_scale multiplies the new V~ (rho_t / rho_{t+1} under
 * admmq_params.rescale_dual; 1 otherwise; must be positive and finite);
 * fit_on_w = 1 refreshes the grid from sigma W~ alone (admmq_params.fit_on_w),
 * 0 from sigma (W~ + V~).
 * V_dev, codes_dev, P_hi_dev, P_lo_dev, sigma_dev, rsig_dev and hdiag_dev
 * must be 32-byte aligned, wtilde_dev 16-byte aligned, row_scale_dev and
 * range_flag_dev 4-byte aligned (ADMMQ_ERR_INVALID_ARG otherwise). */
int admmq_project(const float* wtilde_dev, float* V_dev, const float* sigma_dev,
                  const float* rsig_dev, const float* hdiag_dev, int d_in, int d_out, int bits,
                  int group, int grid_mode, int split_mode, uint8_t* codes_dev, float* scale_dev,
                  float* zero_dev, void* P_hi_dev, void* P_lo_dev, const float* row_scale_dev,
                  int* range_flag_dev, double* resid_dev, float dual_scale, int fit_on_w,
                  void* stream);

/* The split precision a context runs its eigenbasis GEMMs in
 * (ADMMQ_SPLIT_3XTF32, ADMMQ_SPLIT_MIXED or ADMMQ_SPLIT_F16; ADMMQ_SPLIT_AUTO
 * resolved by d_in), which fixes the encoding of its P/T/E buffers;
 * ADMMQ_ERR_INVALID_ARG for a NULL context. */
int admmq_split_mode(const admmq_ctx* ctx);

/* Synchronises the stream and reads the kernel status words: ADMMQ_OK,
 * ADMMQ_ERR_TIMEOUT (a bounded wait gave up) or ADMMQ_ERR_RANGE (an fp16-split
 * operand left fp16's range: the solve's result is not valid; switch the
 * context with admmq_set_split and solve again). */
int admmq_check(admmq_ctx* ctx, void* stream);

/* Switch a context whose eigendecomposition is done (admmq_eigh) to another
 * split precision (ADMMQ_SPLIT_3XTF32, _MIXED or _F16; not _AUTO): the
 * eigenvector planes are encoded again from the float64 eigenvectors kept in
 * the workspace and the scaled weights from W_hat, in the same buffers, and
 * the timeout and range status words are cleared.  The iterate is not
 * converted: admmq_init (or admmq_solve) must come next; admmq_iterate and
 * admmq_finish return ADMMQ_ERR_INVALID_ARG until then.  A solve after the
 * switch gives the same bits as a context created with that split.
 * The fp16 split's operands carry 64x headroom over each row's scaled weight
 * norm; a row whose iterate grows past it (seen on layers where the min/max
 * grid refresh lets a row drift) sets the range word.  The recovery is this
 * call with ADMMQ_SPLIT_MIXED, then the solve again.
 * Asynchronous on `stream`; nothing is allocated. */
int admmq_set_split(admmq_ctx* ctx, int split_mode, void* stream);

/* Test hook for the failure path: pretend `iterations` more iterations have
 * been counted, so that the next fused launch's GEMM-2 tiles wait for GEMM-1
 * tiles that never finish.  Their bounded waits run out (about a second),
 * the launch ends and admmq_check reports ADMMQ_ERR_TIMEOUT; admmq_prepare
 * clears the status words and admmq_init the counters, after which the
 * context solves normally.  No fault, trap or endless loop is involved. */
int admmq_debug_skew_ready(admmq_ctx* ctx, int iterations);

/* The projection's quotient rounding on its own (tests): out[i] =
 * rint(y[i] / s[i / 8]) with the quotient correctly rounded first, computed
 * as the projection does (a reciprocal product, exact division only near a
 * rounding tie).  Device pointers; n a multiple of 8. */
int admmq_debug_rint_div(const float* y_dev, const float* s_dev, long long n, float* out_dev,
                         void* stream);

/* ---------------------------------------------------------------- GPTQ ----
 * The baseline the ADMM-Q objective is reported against: GPTQ, Algorithm 1
 * of "GPTQ: Accurate Post-Training Quantization for Generative Pre-trained
 * Transformers" (sections 2-3), on a fixed grid (the min/max grid of W_hat
 * per output row and group, the RTN grid), columns in natural order, blocks
 * of `block` columns, float64 arithmetic.  R is the upper Cholesky factor of
 * H^-1 with H = G + lambda I and lambda = lambda_rel * mean(diag G), the same
 * damping as admmq_prepare.
 *
 * admmq_gptq_workspace_bytes: bytes of device workspace for d_in x d_out with
 * that block size (block in {32, 64, 128}); 0 for invalid sizes.
 *
 * admmq_gptq:
 *   G_dev       fp32 [d_in][d_in] Gram X^T X (read only).
 *   W_hat_dev   [d_out][d_in], fp32 or bf16 per w_dtype (read only).
 *   codes_dev   u8 [d_out][d_in] out; scale_dev, zero_dev fp32
 *               [d_out][d_in/group] out (the fixed grid).
 *   ws_dev      workspace, 256-byte aligned, ws_bytes >= the size above.
 * Synchronises the stream three times (status words and factorisation info).
 * ADMMQ_ERR_NOT_PD when H or H^-1 is not positive definite,
 * ADMMQ_ERR_NONFINITE for a non-finite diagonal, ADMMQ_ERR_WORKSPACE when
 * ws_bytes is too small. */
size_t admmq_gptq_workspace_bytes(int d_in, int d_out, int block);
int admmq_gptq(const float* G_dev, const void* W_hat_dev, int w_dtype, int d_in, int d_out,
               int bits, int group, float lambda_rel, int block, uint8_t* codes_dev,
               float* scale_dev, float* zero_dev, void* ws_dev, size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* ADMMQ_H_ */
