/*
 * fs.h -- C ABI of the streaming log-domain Sinkhorn library (libfs.so, sm_100a).
 *
 * Entropic optimal transport between two weighted point clouds under the squared
 * Euclidean ground cost C_ij = |x_i - y_j|^2 (SinkSLOT README, "Tensor Contract").
 * The N x M cost or kernel matrix is never stored: every pass recomputes the cost
 * tile by tile on chip and reduces it with an online log-sum-exp (FlashSinkhorn
 * summary, Methodology sections 1-2: attention-form reformulation, online LSE,
 * fusion, row-stationary traversal).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Array arguments are DEVICE pointers to contiguous float32 data, row-major for
 *    the (n, d) and (m, d) clouds, unless an entry point says otherwise. The caller
 *    owns every buffer; the library never allocates device memory. Scratch space is
 *    passed in as `ws` (ws_bytes >= fs_workspace_bytes(problem), 256-byte aligned);
 *    its contents need not be initialised and are not preserved between calls.
 *  - Every call is ordered on `stream` (NULL = the legacy default stream) and is
 *    blocking: it returns after its work has finished, having read back the input
 *    validation and the kernels' error word. Outputs are complete on return.
 *  - Weights a, b are used exactly as given, not normalised; NULL means uniform 1/n
 *    (resp. 1/m). They must be finite and >= 0, zero entries are legal, and their
 *    sums (accumulated in float64) must agree to 1e-5 relative and be positive
 *    (SinkSLOT README, "Tensor Contract": sums must match, zero entries legal).
 *  - n != m is allowed; 1 <= d <= FS_MAX_D; eps must be finite and > 0.
 *  - Potentials are in cost units (f, g), not divided by eps.
 *  - Errors are returned as fs_status; on error the outputs are unspecified and no
 *    GPU state is left behind (the call has drained its own work on `stream`).
 *
 * Thread safety: calls may run concurrently from several host threads on different
 * streams and workspaces. Kernel timing (fs_timing_*) is process-wide.
 */
#ifndef FS_H_
#define FS_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FS_API __attribute__((visibility("default")))
#else
#define FS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL selects the legacy default stream. */
typedef struct CUstream_st* fs_stream_t;

/* Widest points: d <= 16 runs on the FMA path, 16 < d <= 64 on the tensor cores with the
 * operand images resident, 64 < d <= 1024 on the tensor cores in 64-coordinate K-chunks. */
#define FS_MAX_D 1024

/* One OT problem. Pointer fields are device pointers (host pointers for fs_solve_host). */
typedef struct {
  const float* x; /* (n, d) source points */
  const float* y; /* (m, d) target points */
  const float* a; /* (n,) source weights, or NULL for uniform 1/n */
  const float* b; /* (m,) target weights, or NULL for uniform 1/m */
  int64_t n;      /* number of source points, >= 1 */
  int64_t m;      /* number of target points, >= 1 */
  int32_t d;      /* dimension, 1..FS_MAX_D */
  float eps;      /* entropic regularisation, finite and > 0, in cost units */
  int32_t cost;   /* fs_cost_kind; 0 (the default of a zeroed struct) is squared Euclidean */
} fs_problem;

/*
 * Ground costs. FS_COST_SQEUCLIDEAN: C_ij = |x_i - y_j|^2. FS_COST_COSINE:
 * C_ij = 1 - cos(x_i, y_j) = |x_i/|x_i| - y_j/|y_j||^2 / 2 (FlashSinkhorn summary: the cosine
 * distance after normalisation is the other cost of this structure); the library
 * normalises the points (scaled by sqrt(1/2)) into its workspace, so every pass is the
 * squared-Euclidean one, and fs_grad_x applies the normalisation's Jacobian. A zero vector
 * has no direction: FS_ERR_NONFINITE_INPUT. fs_hvp supports the squared-Euclidean cost only.
 */
typedef enum { FS_COST_SQEUCLIDEAN = 0, FS_COST_COSINE = 1 } fs_cost_kind;

typedef enum {
  FS_OK = 0,
  FS_ERR_NULL = 1,             /* a required pointer is NULL */
  FS_ERR_SHAPE = 2,            /* n < 1, m < 1, d < 1, or sizes overflow */
  FS_ERR_EPS = 3,              /* eps not finite or <= 0 */
  FS_ERR_ITERS = 4,            /* n_iters < 1 */
  FS_ERR_NEGATIVE_WEIGHT = 5,  /* a weight is negative or not finite */
  FS_ERR_NONFINITE_INPUT = 6,  /* a coordinate (or a given potential) is not finite, or a
                                  point is zero under the cosine cost */
  FS_ERR_MASS_MISMATCH = 7,    /* |sum a - sum b| > 1e-5 * max(sum a, sum b) */
  FS_ERR_ZERO_MASS = 8,        /* sum a == 0 (so every weight is zero) */
  FS_ERR_UNSUPPORTED_D = 9,    /* d > FS_MAX_D */
  FS_ERR_WORKSPACE = 10,       /* ws NULL, misaligned or smaller than required */
  FS_ERR_TIMEOUT = 11,         /* a kernel's bounded wait expired; outputs invalid */
  FS_ERR_CUDA = 12,            /* a CUDA runtime call failed (see fs_last_cuda_error) */
  FS_ERR_ALIGNMENT = 13,       /* a device pointer is not 4-byte aligned */
  FS_ERR_OPTION = 14,          /* an fs_solve_options field is out of range */
  FS_ERR_DEVICE_MEMORY = 15    /* the device could not commit the static scratch array of
                                  fs_potentials_noalloc when its module was loaded */
} fs_status;

/* Human-readable name of a status code (static storage, never NULL). */
FS_API const char* fs_status_string(fs_status s);

/* Text of the last CUDA error seen by this host thread inside the library, or "". */
FS_API const char* fs_last_cuda_error(void);

/*
 * Bytes of scratch space every entry point below needs for `p` (pointer fields of
 * `p` are not read). Returns 0 when the shape (n, m, d) is invalid. The size depends
 * on the current device's SM count, so query it with the device current that the
 * calls will use. It is not monotone in n and m (fewer rows get more column splits, and
 * so more partial sums), so a workspace shared by several problems takes the largest of
 * their sizes.
 */
FS_API size_t fs_workspace_bytes(const fs_problem* p);

/*
 * What a workspace carries from one call to the next. Every call on sorted clouds (d <= 16)
 * puts both clouds in Morton order; the workspace keeps that order and a record of it (the
 * shapes, a 64-bit fingerprint of each cloud's coordinates, the sort's frame and where the
 * order lies). A later call with the same workspace whose record matches reuses the order
 * instead of sorting again: fs_potentials, fs_grad_x, fs_marginal_residual and fs_cost on
 * the same clouds sort once. A stale or colliding record cannot make results wrong, only
 * screening less effective, since every pass is correct under any order.
 * fs_workspace_invalidate (ws: device, 256-byte aligned, ws_bytes >= 2048, else
 * FS_ERR_WORKSPACE; stream: as for the other calls) drops the record, so the next call
 * sorts; enqueued on `stream`, FS_ERR_CUDA if that fails.
 */
FS_API fs_status fs_workspace_invalidate(void* ws, size_t ws_bytes, fs_stream_t stream);

/*
 * Fixed-count alternating Sinkhorn (SinkSLOT README, API Reference: variant
 * "alternating", stop_mode "fixed"; FlashSinkhorn summary, section 1 for the update):
 *   g <- g_init (or 0 when g_init is NULL)
 *   repeat n_iters times:
 *     f_i <- -eps * LSE_j[(g_j - C_ij)/eps + log b_j]       (one fused streaming pass)
 *     g_j <- -eps * LSE_i[(f_i - C_ij)/eps + log a_i]       (one fused streaming pass)
 * Outputs: f (n floats) and g (m floats), the iterate after the last g-update.
 * g_init (m floats, device) may alias g.
 * From the third iteration on, the iterations of a fixed-count solve (this call, and
 * fs_solve with stop_mode FS_STOP_FIXED) are captured once as a CUDA graph and replayed on
 * `stream`. The capture runs on a non-blocking stream the library creates once per device
 * and keeps until exit (so `stream` may be the legacy default stream); a capture that
 * fails falls back to plain launches. Per-kernel timing (fs_timing_enable) turns it off,
 * and fs_potentials_noalloc never uses it (instantiating a graph may allocate). The call
 * returns once the replays have finished.
 * Problems of at most 2^22 pairs with d <= 16 whose two clouds fit in 200 KB of shared
 * memory (this call, and fs_solve with the alternating variant and FS_STOP_FIXED) run every
 * iteration in one kernel launch on a thread-block cluster of 16 CTAs (8, 4, 2 or 1 where
 * the device cannot co-schedule 16), the biases exchanged through distributed shared
 * memory; the update is the same, in the direct-difference form.
 */
FS_API fs_status fs_potentials(const fs_problem* p, int32_t n_iters, const float* g_init, float* f,
                        float* g, void* ws, size_t ws_bytes, fs_stream_t stream);

/*
 * The general solve (SinkSLOT README, API Reference: variant, alpha, stop_mode,
 * stop_max_iter, stop_tol, stop_check_every; the result's iters_run, converged and
 * final_viol).
 *   variant FS_VARIANT_ALTERNATING (Gauss-Seidel): the schedule of fs_potentials.
 *   variant FS_VARIANT_SYMMETRIC (Jacobi): from f = 0 and g = g_init (or 0), both updates
 *     come from the previous iterate and are blended:
 *       f <- (1 - alpha) f + alpha F(g),   g <- (1 - alpha) g + alpha G(f).
 *   stop_mode FS_STOP_FIXED: exactly n_iters iterations, no check.
 *   stop_mode FS_STOP_MARGINAL: at most stop_max_iter iterations; after every
 *     stop_check_every-th one (and after the last allowed one) the plan's marginal
 *     violation max(|P1 - a|_inf, |P^T 1 - b|_inf) is computed (two extra passes) and
 *     the solve stops once it is <= stop_tol.
 *   stop_mode FS_STOP_POTENTIAL: the same cadence; stops once
 *     max(|f - f_prev|_inf, |g - g_prev|_inf) < stop_tol, the previous values being those of
 *     the last check (of the start for the first one). This is eps * max |delta phi| for
 *     the absorbed potentials phi = f / eps.
 * Each check reads one scalar back to the host (a stream synchronisation).
 * report (host, may be NULL): iters_run; converged (1 or 0; -1 under FS_STOP_FIXED);
 * final_viol (the last check's value; NaN under FS_STOP_FIXED).
 * Errors as fs_potentials (FS_ERR_ITERS for n_iters < 1 under FS_STOP_FIXED), plus
 * FS_ERR_NULL for a NULL opt and FS_ERR_OPTION for an option out of range: an unknown
 * variant or stop mode, alpha outside (0, 1] for the symmetric variant, and under the
 * checked modes stop_max_iter < 1, stop_check_every < 1 or stop_tol < 0 (or NaN).
 */
typedef enum { FS_VARIANT_ALTERNATING = 0, FS_VARIANT_SYMMETRIC = 1 } fs_variant;
typedef enum { FS_STOP_FIXED = 0, FS_STOP_MARGINAL = 1, FS_STOP_POTENTIAL = 2 } fs_stop_mode;

typedef struct {
  int32_t n_iters;          /* iterations under FS_STOP_FIXED */
  int32_t variant;          /* fs_variant */
  float alpha;              /* blend weight of the symmetric variant */
  int32_t stop_mode;        /* fs_stop_mode */
  int32_t stop_max_iter;    /* iteration cap of the checked modes */
  int32_t stop_check_every; /* iterations between checks */
  double stop_tol;          /* threshold of the checks */
  const float* g_init;      /* initial g (m floats, device; may alias g) or NULL */
} fs_solve_options;

typedef struct {
  int32_t iters_run;
  int32_t converged;
  double final_viol;
} fs_solve_report;

FS_API fs_status fs_solve(const fs_problem* p, const fs_solve_options* opt, float* f, float* g,
                          fs_solve_report* report, void* ws, size_t ws_bytes,
                          fs_stream_t stream);

/*
 * Coarse-to-fine solve (FlashSinkhorn 2 abstract, the coarse stage), squared-Euclidean cost
 * and d <= 16 (FS_ERR_OPTION / FS_ERR_UNSUPPORTED_D otherwise). Each cloud is cut into cells
 * of cell_points (1 to 256) points consecutive in its Morton order; a cell is its weighted
 * centroid with its total mass. Rounds of coarse_iters alternating iterations run on the cell problem; after
 * each round its potentials are lifted to every point of y (g_j = G(f_cells)(y_j), one pass
 * of the fine y against the cells) and checked: one fine iteration from the lift and the
 * marginal violation max(|P1 - a|_inf, |P^T 1 - b|_inf) after it. The lift is accepted when
 * that violation is <= lift_tol, when a round shrank it by less than the factor lift_shrink,
 * or after max_rounds rounds; otherwise the coarse iterations continue. The fine stage is
 * then fs_solve with opt from the accepted lift (opt->g_init is ignored). Workspace:
 * fs_multiscale_workspace_bytes(p, cell_points). report (host, may be NULL): rounds, coarse iterations,
 * the accepted lift's violation and the fine solve's report.
 */
typedef struct {
  int32_t cell_points;   /* points per cell, 1..256 */
  int32_t coarse_iters;  /* coarse iterations per round, >= 1 */
  int32_t max_rounds;    /* >= 1 */
  double lift_tol;       /* >= 0 */
  double lift_shrink;    /* in (0, 1] */
} fs_multiscale_options;

typedef struct {
  int32_t rounds;
  int32_t coarse_iters;
  double lift_viol;
  fs_solve_report fine;
} fs_multiscale_report;

FS_API size_t fs_multiscale_workspace_bytes(const fs_problem* p, int32_t cell_points);
FS_API fs_status fs_solve_multiscale(const fs_problem* p, const fs_solve_options* opt,
                                     const fs_multiscale_options* mo, float* f, float* g,
                                     fs_multiscale_report* report, void* ws, size_t ws_bytes,
                                     fs_stream_t stream);

/*
 * Debiased (Sinkhorn) divergence S = OT(a, b) - OT(a, a)/2 - OT(b, b)/2 (the "divergence"
 * the pages' losses report): three fs_solve runs with the same options (g_init ignored) and
 * their dual objectives, value (device, one double) = S. grad_x (n x d) and grad_y (m x d),
 * device or NULL, receive grad_x S = grad_x OT(x, y) - (G1 + G2)/2 with G1, G2 the envelope
 * gradients of OT(x, x) from its two sides (they coincide at convergence), and the same for
 * y. Workspace: fs_divergence_workspace_bytes(p) (the largest of the three problems' plus
 * the divergence's own vectors). Errors as fs_solve.
 */
FS_API size_t fs_divergence_workspace_bytes(const fs_problem* p);
FS_API fs_status fs_divergence(const fs_problem* p, const fs_solve_options* opt, double* value,
                               float* grad_x, float* grad_y, void* ws, size_t ws_bytes,
                               fs_stream_t stream);

/*
 * Transport products and the Hessian-vector product (FlashSinkhorn summary, section 3:
 * transport-matrix application; an HVP decomposed into transport-vector and
 * transport-matrix products), for every d <= FS_MAX_D. Both stream the plan
 * P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps) like the potential passes and never store it.
 * For d <= 16 the passes run on the FMA path in float32 (and screen the plan the same way
 * as the potential passes). For d > 16 they run on the tensor cores: a first pass takes
 * each row's log-sum-exp, a second forms the weights p_ij = P_ij / (P 1)_i <= 1, stores
 * them as fp16 (2^-11 relative rounding each) and multiplies them by the payload (a [hi |
 * lo] fp16 pair, ~2^-22 relative) with fp32 accumulation, and divides by the sum of the
 * same rounded weights; the HVP's difference pass also takes v_i.y_j on the tensor cores.
 *
 * Their workspace is fs_transport_workspace_bytes(p) (0 for an invalid shape or
 * d > FS_MAX_D), larger than fs_workspace_bytes(p): payload keys or images with up to 16
 * channels and the HVP's vectors.
 */
FS_API size_t fs_transport_workspace_bytes(const fs_problem* p);

/*
 * transpose == 0: out (n x k) = P u for u (m x k); transpose == 1: out (m x k) = P^T u for
 * u (n x k); row-major, device, 4-byte aligned. P is the plan of the given (f, g). k >= 1
 * (FS_ERR_OPTION otherwise); channels are streamed 16 at a time.
 */
FS_API fs_status fs_transport_apply(const fs_problem* p, const float* f, const float* g,
                                    int32_t transpose, int32_t k, const float* u, float* out,
                                    void* ws, size_t ws_bytes, fs_stream_t stream);

/*
 * Hessian-vector product of the loss L(x) = OT_eps at the plan of (F(g), g) (exact at a
 * converged g), for one vector v_i per point x_i (v and out: n x d, row-major, device);
 * d <= 64 (FS_ERR_UNSUPPORTED_D above: its difference pass has no K-chunked form):
 *   (H v)_i = 2 a_i v_i + (2/eps) sum_j P_ij (x_i - y_j)(df_i + dg_j - 2 (x_i - y_j).v_i),
 * where (df, dg) solves [diag(P1) P; P^T diag(P^T 1)] (df, dg) = (r, s) with
 * r_i = sum_j P_ij 2 (x_i - y_j).v_i, s_j = sum_i P_ij 2 (x_i - y_j).v_i: the derivative of
 * the gradient 2 (a_i x_i - sum_j P_ij y_j) when the potentials follow x through the
 * marginal constraints. The system (positive semi-definite, singular along the gauge
 * direction (1, -1)) is solved by conjugate gradients on the device, two transport passes
 * and one host read-back per iteration. opt may be NULL (cg_max_iter 200, cg_tol 1e-6, a
 * relative residual). The iteration runs in fp32 and returns the iterate with the smallest
 * residual it has seen; it also stops after 50 iterations without a new smallest residual
 * (a tolerance below fp32 rounding is never reached, and past that point the recurrence
 * only drifts). report (host, may be NULL) receives the iterations run and the relative
 * residual of the returned iterate.
 */
typedef struct {
  int32_t cg_max_iter;  /* >= 1 */
  double cg_tol;        /* >= 0: stop once |residual| <= cg_tol |right-hand side| */
} fs_hvp_options;

typedef struct {
  int32_t cg_iters;
  double cg_rel_residual;
} fs_hvp_report;

FS_API fs_status fs_hvp(const fs_problem* p, const float* g, const float* v, float* out,
                        const fs_hvp_options* opt, fs_hvp_report* report, void* ws,
                        size_t ws_bytes, fs_stream_t stream);

/*
 * Dual objective at (f, g):
 *   D(f, g) = <f, a> + <g, b> - eps * (sum_ij P_ij - m_a * m_b),
 *   P_ij = a_i b_j exp((f_i + g_j - C_ij)/eps),  m_a = sum a, m_b = sum b.
 * sum_ij P_ij is evaluated exactly by one streaming column pass, so any (f, g) is
 * accepted; right after fs_potentials (P^T 1 = b) it equals
 * <f,a> + <g,b> - eps*m*(1 - m). Writes one double to `out` (device).
 */
FS_API fs_status fs_cost(const fs_problem* p, const float* f, const float* g, double* out, void* ws,
                  size_t ws_bytes, fs_stream_t stream);

/*
 * Envelope gradient of the cost with respect to x (FlashSinkhorn summary, section 3:
 * transport-matrix application without materialising P). For d > 16 it runs on the tensor
 * cores as two streaming passes (the rows' log-sum-exp, then sum_j Pt_ij y_j with the
 * weights in fp16 as for the transport products):
 *   ft = F(g) (a fresh f-update, fused into the same pass), Pt_ij = a_i b_j
 *   exp((ft_i + g_j - C_ij)/eps), so sum_j Pt_ij = a_i and
 *   grad_x[i, :] = 2 * (a_i x_i - sum_j Pt_ij y_j) = 2 a_i (x_i - T_i),
 * T_i the barycentric projection of x_i. Only g is needed. Writes (n, d) floats.
 */
FS_API fs_status fs_grad_x(const fs_problem* p, const float* g, float* grad_x, void* ws,
                    size_t ws_bytes, fs_stream_t stream);

/*
 * Marginal residuals of the plan of (f, g) (SinkSLOT README, stop_mode "marginal";
 * FlashSinkhorn 2 abstract, "marginal residual"):
 *   r_i = sum_j P_ij = a_i exp((f_i - F(g)_i)/eps)   (one streaming row pass)
 *   c_j = sum_i P_ij = b_j exp((g_j - G(f)_j)/eps)   (one streaming column pass)
 * Writes 4 doubles to `out` (device): [sum|r - a|, max|r - a|, sum|c - b|, max|c - b|].
 * row_marg (n floats) and col_marg (m floats), when not NULL, receive r and c.
 */
FS_API fs_status fs_marginal_residual(const fs_problem* p, const float* f, const float* g, double* out,
                               float* row_marg, float* col_marg, void* ws, size_t ws_bytes,
                               fs_stream_t stream);

/*
 * fs_potentials for callers that cannot allocate device memory. The pages have no
 * counterpart to this entry point; it exists for the library's users.
 *
 * Some callers may not call cudaMalloc or cudaFree at all: a host application whose
 * device memory is owned entirely by its own pool allocator, or a latency-critical loop
 * that must not hit the implicit device synchronisation those calls can cause. They pass
 * only their inputs and outputs (same meaning, layout and ownership as fs_potentials);
 * the scratch space comes from a fixed array of FS_NOALLOC_SCRATCH_BYTES bytes in device
 * global memory that the library declares statically. Every device that loads the
 * library holds that array until the process exits.
 *
 *  - Problems whose fs_workspace_bytes() exceeds FS_NOALLOC_SCRATCH_BYTES are rejected
 *    with FS_ERR_WORKSPACE before any device work. At d = 3 every problem with
 *    n, m <= 80000 fits; larger d needs more scratch per point.
 *  - Every call looks up the array's device address (cudaGetSymbolAddress) in the context
 *    current on the calling thread; nothing is cached, so the call stays correct after
 *    cudaDeviceReset or under a context of the caller's own.
 *  - When that memory is committed depends on the CUDA module loading mode. Under lazy
 *    loading (CUDA_MODULE_LOADING=LAZY, the default since CUDA 12.2) the FIRST call in a
 *    context loads the module that holds the array: that call commits
 *    FS_NOALLOC_SCRATCH_BYTES of device memory (plus the module's code) and may
 *    synchronise the device. Make it during initialisation, before a pool allocator
 *    reserves the device's memory and before any stream capture. If the device cannot
 *    provide the memory the call returns FS_ERR_DEVICE_MEMORY (other failures of the
 *    lookup: FS_ERR_CUDA). Under eager loading the array is committed when the context is
 *    created. Later calls commit nothing.
 *  - No call allocates or frees device memory (no cudaMalloc, cudaFree or allocating
 *    library routine).
 *  - All calls on a device share the one array and it keeps what the last call wrote:
 *    calls that overlap on the GPU (two streams or host threads at once) race and give
 *    wrong results. Serialise them.
 * Other errors are those of fs_potentials.
 */
#define FS_NOALLOC_SCRATCH_BYTES (20u << 20)
FS_API fs_status fs_potentials_noalloc(const fs_problem* p, int32_t n_iters, const float* g_init,
                                       float* f, float* g, fs_stream_t stream);

/*
 * Checks of the error path (SinkSLOT README, "Tensor Contract": bad states raise rather than
 * return wrong results). Every pass kernel bounds its waits (2 s of %globaltimer) and, when
 * one expires, sets a bit in the call's device error word, waits (bounded) for its own
 * copies in flight and returns; the entry point then returns FS_ERR_TIMEOUT.
 *
 * fs_inject_error_word arms a one-shot injection: the next entry point call (any host
 * thread) that reads its kernels' error word first ORs `bits` into that word on the device,
 * by a kernel launched on the call's stream after its passes, where an expired wait would
 * have set it. That call then returns FS_ERR_TIMEOUT (for any non-zero bits) and its
 * outputs are invalid; the injection is disarmed, and later calls are unaffected
 * (0 disarms without injecting). Process-wide, for tests of the error path.
 *
 * fs_check_bounded_wait runs the bounded mbarrier wait of the pass kernels, with a limit of
 * limit_ns (1e3 .. 2e9 ns, else FS_ERR_OPTION), on a barrier that nothing arrives at, with
 * no copy or MMA in flight. The wait expires, the kernel sets the error word (held in `ws`:
 * device, 256-byte aligned, >= 2048 bytes, else FS_ERR_WORKSPACE) and returns, so the call
 * returns FS_ERR_TIMEOUT after about limit_ns, the context still usable. FS_OK would mean a
 * wait that ended although nothing arrived.
 */
FS_API void fs_inject_error_word(unsigned bits);
FS_API fs_status fs_check_bounded_wait(int64_t limit_ns, void* ws, size_t ws_bytes,
                                       fs_stream_t stream);

/*
 * One call for callers whose data live in HOST memory: copies x, y, a, b (and nothing
 * else) to the device, runs fs_potentials, fs_grad_x, fs_marginal_residual and
 * fs_cost, and copies f, g, grad_x, the cost and the four residual norms back.
 * Pointer fields of `p` and every array argument are HOST pointers (page-locked
 * memory makes the copies asynchronous; pageable memory works but is slower);
 * grad_x, cost and residual may be NULL to skip those steps. `ws` is device scratch
 * of at least fs_solve_host_workspace_bytes(p) bytes.
 */
FS_API size_t fs_solve_host_workspace_bytes(const fs_problem* p);
FS_API fs_status fs_solve_host(const fs_problem* p, int32_t n_iters, float* f, float* g, float* grad_x,
                        double* cost, double* residual, void* ws, size_t ws_bytes,
                        fs_stream_t stream);

/*
 * Kernel timing, off by default. When on, every launch of the streaming passes is
 * bracketed by CUDA events recorded on the stream it runs on, and each entry point
 * adds the measured durations before returning. Process-wide; not for concurrent use.
 */
typedef struct {
  int64_t launches; /* launches measured since the last reset */
  double total_ms;  /* their summed device durations */
  double pairs;     /* (row, column) pairs the problem defines for them: N * M per pass */
  double evaluated; /* pairs actually evaluated (exponentials issued, padding included)
                       after block screening; filled for passes on sorted clouds (d <= 16) */
} fs_timing_entry;

typedef struct {
  fs_timing_entry lse_pass;  /* potential-update passes (f and g half-iterations) */
  fs_timing_entry grad_pass; /* gradient passes */
  fs_timing_entry marg_pass; /* marginal / plan-mass passes (residual and cost) */
  fs_timing_entry combine;   /* second-level merges of split or unit partials */
  fs_timing_entry screen;    /* block screening and unit planning on sorted clouds */
} fs_timing;

FS_API void fs_timing_enable(int on);
FS_API void fs_timing_reset(void);
FS_API void fs_timing_get(fs_timing* out);

/* Number of CUDA kernels this library has launched in this process (all entry points,
 * all devices), counted at each launch site. */
FS_API int64_t fs_launch_count(void);

/*
 * Block screening, on by default (point clouds with d <= 16, which the library puts in a
 * spatial order). A pass skips a 256-point key tile when a bound shows that each of its
 * terms is below 2^-(24 + log2 M) times the largest term of every row it meets, and for
 * d <= 3 a group of 16 consecutive keys of a tile it keeps by the same bound, so that the
 * omitted part of each row's sum is below 2^-24 of the sum (FlashSinkhorn 2 abstract,
 * block-sparse screening, here with a provable bound). fs_screening_enable(0) makes every
 * later call evaluate all N x M pairs; the results agree to fp32 rounding either way.
 * Process-wide; takes effect at the next call.
 */
FS_API void fs_screening_enable(int on);

#ifdef __cplusplus
}
#endif

#endif /* FS_H_ */
