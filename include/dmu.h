/*
 * dmu.h -- C ABI of libdmu: the owner-side Muon update on one B200 GPU.
 *
 * The update, per weight matrix W (rows x cols, row-major, contiguous):
 *
 *   1. momentum        M <- beta * M + G
 *   2. orientation     X = M if rows <= cols, else X = M^T   (m = min, n = max)
 *   3. normalisation   X0 = X / (||M||_F + eps)
 *   4. Gram recursion  G0 = X0 X0^T, P0 = I;  K times:
 *                        Q = a I + b G + c G^2,  G <- Q G Q,  P <- Q P
 *   5. update          O = P X0 (in W's orientation);
 *                      W <- W - lr * sqrt(max(1, rows / cols)) * O
 *
 * Sources (page title and section):
 *   - "DMuon: Efficient Distributed Muon Training with Near-Adam Overhead",
 *     technical summary, section 1: Muon applies Newton-Schulz to the
 *     momentum-accumulated gradient of each weight matrix (steps 1, 4, 5).
 *   - same page, section 2.2: the recursion runs in the m x m Gram space
 *     G = X X^T, the symmetric products take a SYRK-style path, and
 *     similar-shape matrices are batched (steps 2, 4; the batching below).
 *   - same page, section 2.4: per-shape kernel schedules are tuned and
 *     cached (the per-plan schedule choice).
 *   - "DeMuon" technical summary, Method 1: the target of the iteration is
 *     the matrix sign msgn(X) = U V^T.
 *   - "Dion3: Full-Stack Orthogonal Updates" review, sections 1 and 3:
 *     Gram Newton-Schulz and a symmetric GEMM kernel.
 * The pages give no coefficients, step count, eps, momentum form or scale
 * rule; the defaults here are (a,b,c) = (3.4445, -4.7750, 2.0315), K = 5,
 * eps = 1e-7, the plain accumulation above and sqrt(max(1, rows/cols)).
 *
 * Conventions for every call:
 *   - Ownership: the caller owns all device memory -- gradients, momenta,
 *     weights and the workspace (dmu_set_workspace).  The library owns only
 *     its host-side plan and a small pinned staging buffer for pointer
 *     tables.  Pointer arrays are HOST arrays of DEVICE pointers; the
 *     library copies them to the workspace when they differ from the last
 *     call's (stream-ordered), so steady-state steps upload nothing.
 *   - Asynchrony: compute calls enqueue work on `stream` (a cudaStream_t,
 *     passed as void*; NULL = legacy default stream) and return without
 *     synchronising.  Only dmu_read_status and dmu_debug_gram synchronise.
 *   - Errors: every call returns a dmu_status.  Argument errors are
 *     detected before any launch.  CUDA errors map to DMU_ERR_CUDA.
 *     dmu_last_error() returns the message of the calling thread's last
 *     error.  There are no device traps: device-side faults of the data
 *     (non-finite norms) and bounded-wait timeouts set bits of a device
 *     status word that dmu_read_status returns.
 *   - Layout: every matrix i is contiguous row-major with the shape given
 *     to dmu_plan_create.  Device pointers must be 16-byte aligned for the
 *     vectorised paths (misaligned pointers take a scalar path).
 *   - Threads: a plan must not be used by two host threads at once.
 *   - Schedule: tensor-core launches run on CTA pairs (256 x 256 tiles,
 *     tcgen05.mma.cta_group::2) by default.  Two single-CTA schedules
 *     exist: 128 x 256 tiles, and 128 x 128 tiles for many small matrices.
 *     dmu_autotune picks one by measurement.  At plan creation the
 *     environment variable DMU_SCHEDULE=0|1|2|4|5|6 (0 = 128 x 256 single
 *     CTAs, 1 = CTA pairs, 2 = 128 x 128 single CTAs, 4-6 as in
 *     dmu_get_gram_schedule) overrides the default, and so does
 *     DMU_CTA_PAIR=0|1.  Every schedule accumulates each element over K in
 *     the same order, so all give bitwise-equal results.
 */
#ifndef DMU_H
#define DMU_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DMU_VERSION 100

#if defined(__GNUC__)
#define DMU_API __attribute__((visibility("default")))
#else
#define DMU_API
#endif

typedef enum {
  DMU_OK = 0,
  DMU_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, count mismatch   */
  DMU_ERR_UNSUPPORTED = 2,  /* device is not sm_100, or a mode not built */
  DMU_ERR_WORKSPACE = 3,    /* workspace missing, too small, misaligned  */
  DMU_ERR_CUDA = 4,         /* a CUDA runtime or driver call failed       */
  DMU_ERR_NONFINITE = 5,    /* a momentum norm was NaN or Inf             */
  DMU_ERR_NOT_PLANNED = 6,  /* shapes differ from the plan, or call order */
  DMU_ERR_TIMEOUT = 7       /* a bounded device-side wait gave up         */
} dmu_status;

typedef enum {
  DMU_BF16 = 0, /* gradients and weights bf16; tensor-core (tcgen05) path */
  DMU_F32 = 1   /* gradients and weights fp32; exact fp32 FFMA path        */
} dmu_dtype;

/* Precision of the Gram-space products on the bf16 path.  Gram-space
 * matrices are stored as a 16-bit pair (hi, lo = round(x - hi)).  The image
 * of M that the Gram matrix and the final product read is fp16(2^e M) at a
 * power-of-two scale 2^e per matrix (for bf16 gradients and a first step,
 * exactly M); the final P X0 product multiplies it by P as one
 * fp16 operand (F16 classes) or as an fp16 hi/lo pair (other classes).
 * Each symmetric
 * product is computed on its upper-triangle tiles and mirrored, which
 * turns the antisymmetric part of the operand rounding error into a
 * symmetric one; with one bf16 MMA per product that error shifts the small
 * eigenvalues of G enough to miss 2e-2 on spiked inputs, so:
 *   FAST   : one bf16 MMA per product (hi x hi)        -- low precision:
 *            misses the 2e-2 bound on spiked inputs (measured 0.07-0.17
 *            relative error on rank-8 spiked 128x512 .. 512x2048);
 *   SPLIT2 : two MMAs per product (hi x hi + lo x hi)  -- low precision:
 *            misses 2e-2 on the same inputs (0.06-0.14);
 *   SPLIT3 : three MMAs per product (hi x hi + hi x lo + lo x hi);
 *   TF32   : Gram-space state in fp32, one kind::tf32 MMA per product
 *            (half the bf16 rate; 10-bit operand mantissa);
 *   F16    : Gram-space state as fp16 hi/lo pairs pre-scaled by powers of
 *            two, one fp16 MMA per product at the full rate, with the same
 *            10-bit operand mantissa as TF32;
 *   AUTO   : F16 for m >= 1024, SPLIT3 below (per Gram class). */
typedef enum {
  DMU_PREC_AUTO = 0,
  DMU_PREC_FAST = 1,
  DMU_PREC_SPLIT2 = 2,
  DMU_PREC_SPLIT3 = 3,
  DMU_PREC_TF32 = 4,
  DMU_PREC_F16 = 5
} dmu_prec;

/* Bits of the device status word (dmu_read_status). */
#define DMU_FLAG_NONFINITE 0x1u /* a Frobenius norm was not finite  */
#define DMU_FLAG_TIMEOUT 0x2u   /* a device wait hit its time limit */

typedef struct {
  int64_t rows; /* W.shape[0] (out_features) */
  int64_t cols; /* W.shape[1] (in_features)  */
} dmu_shape;

typedef struct dmu_plan_s* dmu_plan;

/* Build a plan for `count` matrices with these shapes on CUDA `device`.
 * Matrices are grouped into buckets of equal (rows, cols) and, for the
 * Gram-space recursion, into classes of equal m = min(rows, cols); tall
 * matrices are handled by logical transposition (no copy).  No device
 * memory is allocated.  Errors: INVALID_ARG (count <= 0, a non-positive
 * extent, out == NULL), UNSUPPORTED (device not compute capability 10.x
 * for DMU_BF16), CUDA. */
DMU_API dmu_status dmu_plan_create(const dmu_shape* shapes, int count, dmu_dtype dtype,
                           dmu_prec prec, int device, dmu_plan* out);

/* Bytes of device workspace the plan needs (0 for an invalid plan). */
DMU_API size_t dmu_workspace_bytes(dmu_plan plan);

/* Give the plan its workspace: `bytes` >= dmu_workspace_bytes, 256-byte
 * aligned, on the plan's device, owned by the caller and kept alive while
 * the plan is used.  Uploads the plan's tables (synchronous) and encodes
 * the TMA tensor maps.  Errors: WORKSPACE, INVALID_ARG, CUDA. */
DMU_API dmu_status dmu_set_workspace(dmu_plan plan, void* dev_ptr, size_t bytes);

/* Step 1 + the norm of step 3, for all matrices of the plan.
 *   grads[i]   : device pointer, rows*cols elements of the plan dtype.
 *   momenta[i] : device pointer, rows*cols fp32, updated in place
 *                (M <- beta*M + grad_scale*G).  momenta == NULL means "no
 *                state": M = grad_scale*G and nothing is written back.
 *   grad_scale : factor on the gradient, applied in the same pass (1 for
 *                the plain update; 1/N turns the sum of N data-parallel
 *                gradients into their mean without a separate pass).
 * Errors: INVALID_ARG for a NULL grads array or pointer, eps < 0, or a
 * non-finite beta or grad_scale; WORKSPACE; CUDA.
 * Writes the bf16 (or fp32) image of M and 1/(||M||_F + eps) for every
 * matrix into the workspace.  Source: DMuon page, section 1. */
DMU_API dmu_status dmu_momentum_normalize(dmu_plan plan, const void* const* grads,
                                  float* const* momenta, float beta, float grad_scale,
                                  float eps, void* stream);

/* Steps 2-4: the Gram Newton-Schulz recursion, batched over all matrices.
 *   ptrs   : NULL to use the matrices left by dmu_momentum_normalize; or
 *            device pointers to `count` matrices (plan dtype) to
 *            orthogonalise directly (they are normalised first, with the
 *            eps of the last dmu_momentum_normalize call, 1e-7 if none).
 *   shapes, count : must equal the plan's (else NOT_PLANNED).
 *   coeffs : (a, b, c);  steps : K >= 0 (K = 0 gives P = I).
 * Result: P_K per matrix, kept in the workspace for dmu_apply_update.
 * Sources: DMuon page, section 2.2; Dion3 review, sections 1 and 3. */
DMU_API dmu_status dmu_gram_ns_batched(dmu_plan plan, const void* const* ptrs,
                               const dmu_shape* shapes, int count,
                               const float coeffs[3], int steps, void* stream);

/* Step 5: O = P X0 fused with W <- W - lr * sqrt(max(1, rows/cols)) * O.
 *   weights[i] : device pointer, rows*cols of the plan dtype, updated in
 *                place; weights == NULL skips the update.
 *   out_o[i]   : optional fp32 device buffers (rows*cols) that receive O
 *                in W's orientation; out_o == NULL skips them all, a NULL
 *                entry skips that matrix.
 * Requires a completed dmu_gram_ns_batched (else NOT_PLANNED). */
DMU_API dmu_status dmu_apply_update(dmu_plan plan, void* const* weights, float lr,
                            float* const* out_o, void* stream);

/* Synchronise the plan's device, read and clear the status word.
 * Returns NONFINITE or TIMEOUT when the matching bit was set. */
DMU_API dmu_status dmu_read_status(dmu_plan plan, uint32_t* flags);

/* Test hook: write one workspace quantity as fp32 into `out` (device).
 *   which 0..4 : Gram-space matrix G, R, T, P(buffer A), P(buffer B) of
 *                matrix `index` (m*m floats, hi + lo combined);
 *   which 5    : the input image of matrix `index` (rows*cols floats, in
 *                M's units): on the bf16 path fp16(2^e M), read back with
 *                the power-of-two scale 2^e of which 9;
 *   which 6    : 1/(||M||_F + eps) of every matrix (count floats);
 *   which 7    : the final P of matrix `index` (m*m floats);
 *   which 8    : bounded-wait self-test, writes nothing to `out`: a kernel
 *                waits `index` microseconds (1..1e6) on a barrier that
 *                nothing completes, gives up, and sets DMU_FLAG_TIMEOUT
 *                (read it with dmu_read_status);
 *   which 9    : bf16 plans: the scale 2^e of every matrix's fp16 image
 *                (count floats).  A matrix keeps its scale from call to
 *                call while 2^e ||M||_F stays in (2^9, 2^15]; otherwise
 *                (and on the plan's first call) a new one puts it in
 *                (2^11, 2^12].
 * Synchronises `stream`. */
DMU_API dmu_status dmu_debug_gram(dmu_plan plan, int which, int index, float* out, void* stream);

/* Pick the fastest schedule per shape by measurement (DMuon page, section
 * 2.4: per-shape kernel configurations are tuned once and cached).
 *   - Every Gram class (all matrices with one m) is timed alone over the
 *     whole quintic recursion (K = 5) with CTA pairs (256 x 256 tiles),
 *     single CTAs (128 x 256 and 128 x 128 tiles), for scaled-fp16 classes
 *     CTA pairs with 2 and 1 K atoms per stage, and for split-bf16 classes
 *     with m <= 128 the on-chip recursion; CTA pairs win ties.
 *   - Every shape bucket's final GEMM + update is then timed alone with the
 *     three tile schedules.  Its weight writes go to the class's free
 *     Gram-space scratch, never to the caller's weights (buckets whose
 *     weights do not fit there are timed on the first matrices that do).
 * Times run on the data left by dmu_momentum_normalize.  Each choice is
 * appended to the text file `cache_path` (may be NULL: no cache) as one
 * line "<key> <schedule> <times...>"; the key names the device, the
 * precision and the shapes of the class or bucket, so any plan with the
 * same class or bucket reuses the entry without timing.  Synchronises
 * `stream`; overwrites the plan's Gram-space state and leaves P_K of the
 * quintic K = 5 recursion for dmu_apply_update.  Errors: NOT_PLANNED (no
 * dmu_momentum_normalize yet), CUDA. */
DMU_API dmu_status dmu_autotune(dmu_plan plan, const char* cache_path, void* stream);

/* The plan's default tile schedule: 1 = CTA pairs (256 x 256), 0 = single
 * CTAs (128 x 256), 2 = single CTAs (128 x 128); -1 for a NULL plan.
 * Classes and buckets that dmu_autotune (or DMU_ONCHIP) gave their own
 * schedule report it through the two calls below. */
DMU_API int dmu_get_schedule(dmu_plan plan);

/* Schedule of the Gram recursion of matrix `index`'s class (all matrices
 * with its m): 0, 1, 2 as above; 3 = the whole recursion on chip (one CTA
 * per matrix, m <= 128, split-bf16 precision); 4 and 5 = CTA pairs whose
 * one-MMA-per-slice fp16 kernels stage 2 and 1 K atoms of 64 (three and six
 * stages) instead of 3 (two stages); 6 = CTA pairs with 256 x 512 tiles
 * (two N = 256 MMAs per K slice share the A operand; scaled-fp16 launches
 * only, the others of a class on schedule 6 run as schedule 1).  -1 for a
 * bad argument. */
DMU_API int dmu_get_gram_schedule(dmu_plan plan, int index);

/* Tile schedule (0, 1 or 2) of the final GEMM of matrix `index`'s bucket.
 * -1 for a bad argument. */
DMU_API int dmu_get_final_schedule(dmu_plan plan, int index);

/* Schedule of the SYRK (G0 = s^2 X X^T) of matrix `index`'s bucket: its
 * class's tile schedule unless dmu_autotune measured another one faster
 * for that bucket's SYRK alone (candidates 0, 4 and 6 besides the class's;
 * its K is the long side n); 3 when the class runs on chip.  -1 for a bad
 * argument. */
DMU_API int dmu_get_syrk_schedule(dmu_plan plan, int index);

/* Number of kernel launches the last compute call enqueued. */
DMU_API int dmu_last_launch_count(dmu_plan plan);

/* Message for the calling thread's last error ("" if none). */
DMU_API const char* dmu_last_error(void);

/* Library version (DMU_VERSION). */
DMU_API int dmu_version(void);

/* Free the host-side plan.  Does not touch the caller's device memory. */
DMU_API void dmu_plan_destroy(dmu_plan plan);

/* Momentum + Frobenius norm of ONE matrix without allocating anything.
 * The pages describe no such call; it exists for callers that cannot
 * allocate device memory themselves -- a process whose device memory
 * belongs to another framework's pool, a plugin that may not call the CUDA
 * allocator, or a hot loop where cudaMalloc/cudaFree would synchronise.
 * It computes what dmu_momentum_normalize computes for one matrix, with
 * its scratch (one partial sum per 16384 elements) in a fixed 64 KB
 * __device__ array inside the library instead of a workspace:
 *   grad         : device, rows*cols elements of `dtype`;
 *   momentum     : device fp32 rows*cols, updated in place (M <- beta*M + G);
 *                  NULL means M = G and nothing is written back;
 *   image_out    : device, rows*cols of `dtype` receiving M rounded to the
 *                  dtype (bf16 image for DMU_BF16); may be NULL;
 *   inv_norm_out : device, one float, receives 1/(||M||_F + eps).
 * Limit: rows*cols <= 2^28 (268435456); larger returns DMU_ERR_UNSUPPORTED
 * before any launch.  Every call looks up the array's device address in
 * the current device's context (the lookup allocates nothing); the first
 * call on a device may load the library's device code, so make that first
 * call before any stream capture.  Every call on a device shares the array:
 * calls that overlap on the GPU race and must be ordered by the caller.
 * The array needs no clearing (each call writes every slot it reads).
 * Allocates nothing (no cudaMalloc, cudaFree or allocating library call). */
DMU_API dmu_status dmu_momentum_norm_static(const void* grad, float* momentum, void* image_out,
                                            int64_t rows, int64_t cols, dmu_dtype dtype, float beta,
                                            float eps, float* inv_norm_out, void* stream);

/* ---------------------------------------------------------------- DeMuon
 * Decentralised Muon over a communication graph of N agents (DeMuon
 * technical summary, "Methodology", 1. DeMuon: local momentum, gradient
 * tracking, and iterates updated from the neighbours' msgn steps).  Each
 * agent i keeps, per weight matrix, a momentum estimate M_i, a tracked
 * gradient V_i and an iterate X_i.  One iteration with mixing weights w_ij:
 *
 *   M_i' = (1 - theta) M_i + theta G_i          dmu_demuon_track
 *   V_i' = sum_j w_ij V_j + M_i' - M_i          dmu_demuon_track
 *   O_j  = msgn(bf16(V_j'))                     a plan over all agents' matrices:
 *                                               dmu_momentum_normalize (beta 0),
 *                                               dmu_gram_ns_batched,
 *                                               dmu_apply_update (out_o only)
 *   X_i' = sum_j w_ij (X_j - eta O_j)           dmu_demuon_mix
 *
 * The page names these sequences and operations but prints no formulas; the
 * recursions above are the plain gradient-tracking reading.
 *
 * Layout: every agent's state for all its matrices is one flat array of
 * `numel` elements (fp32 for M, V, X, O; bf16 for G and the msgn input),
 * the same element order in every agent; the kernels treat it as a vector.
 * `mix` is a HOST array of n_agents x n_agents fp32 weights, row-major, row
 * i holding the weights agent i applies to every agent's values.  The
 * pointer arguments are HOST arrays of n_agents DEVICE pointers, each
 * 16-byte aligned.  Outputs must not alias inputs of another role (every
 * output element reads all agents' inputs): v_out vs v_in, x_out vs x_in
 * and o; v_out, v_bf16 and momenta are distinct arrays, and v_bf16 does
 * not alias grads (momenta are updated in place).  Sums over agents run
 * in agent order, so results are deterministic.  Errors: n_agents outside
 * [1, DMU_DEMUON_MAX_AGENTS], a null or misaligned pointer, aliasing,
 * non-finite weights, theta outside [0, 1] or a non-finite eta return
 * DMU_ERR_INVALID_ARG before any launch.
 * Both calls are stream-ordered and do not synchronise. */
#define DMU_DEMUON_MAX_AGENTS 16

DMU_API dmu_status dmu_demuon_track(int n_agents, int64_t numel, const float* mix, float theta,
                                    const void* const* grads, float* const* momenta,
                                    const float* const* v_in, float* const* v_out, void* const* v_bf16,
                                    void* stream);

DMU_API dmu_status dmu_demuon_mix(int n_agents, int64_t numel, const float* mix, float eta,
                                  const float* const* x_in, const float* const* o, float* const* x_out,
                                  void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DMU_H */
