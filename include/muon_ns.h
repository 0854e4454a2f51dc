/*
 * muon_ns.h -- C ABI of the B200 (sm_100a) Muon optimizer step.
 *
 * One Muon step on a set of 2D weight matrices, entirely in hand-written
 * CUDA kernels:
 *   1. momentum m' = beta*m + (1-beta)*g, Nesterov blend u = g + beta*(m'-g),
 *      per-matrix sum of squares of u and the bf16 cast of u (one kernel);
 *   2. the quintic Newton-Schulz iteration on the short side,
 *      A = X X^T, B = bA + cA^2, X <- aX + BX, with X = u / (||u||_F + 1e-7)
 *      (tensor-core GEMMs, one launch per phase for all matrices; in bf16
 *      the polynomial's epilogue forms aI + bA + cA^2, rounded once, and the
 *      combine is the product of that with X);
 *   3. p' = p*(1 - lr*wd) - lr*scale(m, n)*O: in the last combine's epilogue
 *      (blocks of p moved by bulk copies; see muon_config.fused_apply), or
 *      one separate kernel.
 *
 * Sources (web pages, cited by title and section):
 *   "About Muon: Why Not Adam": "The whole thing, in about forty lines"
 *     (step order, eps, transpose rule, lerp forms, defaults, Moonlight
 *     scale); "The lemma that makes it possible"; "The iteration does not
 *     converge, and that is deliberate" (coefficients); "How Do We Turn It
 *     Into a Real Optimizer?" (Jordan and Moonlight multipliers,
 *     (m, n) = (fan-out, fan-in) = p.shape); "The spectral ball gives UV^T"
 *     (Bernstein multiplier).
 *   "Por que AdamW para entrenar modelos de lenguaje, y que esta cambiando",
 *     "Momentum: recordar el paso anterior" (Muon uses Nesterov).
 *   "The Optimizer Wars: How Muon Is Replacing Adam in Frontier AI
 *     Training", "What is Muon? Momentum orthogonalized by Newton-Schulz"
 *     (five quintic steps in bf16 on tensor cores).
 *   "Why Muon Works", section 6 configuration block (scale mode, extra
 *     scale factor, number of NS steps, Nesterov flag).
 *
 * Conventions for every entry point:
 *   - Return value: a muon_status code; MUON_OK (0) on success. No C++
 *     exception crosses this boundary. muon_last_error() returns a
 *     thread-local description of the last failure on the calling thread.
 *   - "Device pointer" means memory of the handle's device; "host array"
 *     means an ordinary host array read during the call only.
 *   - Matrices are row-major m x n with (m, n) = (fan-out, fan-in), i.e. the
 *     PyTorch layout of a weight p of shape (m, n). The shape table is a
 *     host int32 array shapes[count][3] = {m, n, flags}; m, n >= 1;
 *     flags bit 0 (MUON_FLAG_GRAD_BF16) says the gradient is bf16 (else
 *     fp32). Other flag bits must be zero.
 *   - Parameters and momenta are fp32, densely packed (row stride n).
 *     Gradients are fp32 or bf16 per the flag, densely packed. Every
 *     caller pointer must be 16-byte aligned; params, grads and momenta of
 *     one matrix must not overlap.
 *   - "X layout": a bf16 (fp32 in the fp32 debug mode) row-major m x ldx
 *     buffer with ldx = round_up(n, 8); columns n..ldx-1 are ignored on
 *     input and left unspecified on output.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously; the call does not wait for the GPU
 *     unless documented. The caller keeps every buffer alive until the
 *     stream has reached the end of the enqueued work.
 *   - The handle is not thread-safe: one thread at a time per handle.
 */
#ifndef MUON_NS_H
#define MUON_NS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes. */
enum muon_status {
  MUON_OK = 0,
  MUON_ERR_INVALID_ARG = 1, /* bad shape, count, pointer, alignment, flag   */
  MUON_ERR_CUDA = 2,        /* a CUDA runtime/driver call failed           */
  MUON_ERR_OOM = 3,         /* workspace above the configured cap, or a
                               device allocation failed                     */
  MUON_ERR_TIMEOUT = 4,     /* a bounded device-side wait expired; the
                               kernel stopped early and results are invalid */
  MUON_ERR_NONFINITE = 5,   /* reported by muon_get_status only            */
  MUON_ERR_NO_DEVICE = 6,   /* no usable CUDA device                       */
  MUON_ERR_UNSUPPORTED = 7  /* device is not sm_100                        */
};

/* Update-scale families, (m, n) = (fan-out, fan-in). */
enum muon_scale_mode {
  MUON_SCALE_MOONLIGHT = 0, /* 0.2*sqrt(max(m,n)): "About Muon: Why Not
                               Adam", "How Do We Turn It Into a Real
                               Optimizer?" and the program in "The whole
                               thing, in about forty lines"               */
  MUON_SCALE_JORDAN = 1,    /* sqrt(max(1, m/n)): same section            */
  MUON_SCALE_BERNSTEIN = 2, /* sqrt(m/n) = sqrt(fan-out/fan-in):
                               "The spectral ball gives UV^T"             */
  MUON_SCALE_NONE = 3       /* 1                                          */
};

/* Newton-Schulz arithmetic. */
enum muon_ns_precision {
  MUON_NS_BF16 = 0, /* bf16 operands, fp32 tensor-core accumulation,
                       one round-to-nearest-even per GEMM output (default) */
  MUON_NS_FP32 = 1  /* debug: fp32 operands and FFMA accumulation          */
};

/* Form of the Newton-Schulz iteration. */
enum muon_ns_algorithm {
  MUON_NS_STANDARD = 0, /* X <- aX + (bA + cA^2)X, A = X X^T, each step
                           ("About Muon: Why Not Adam", "The whole thing,
                           in about forty lines")                          */
  MUON_NS_GRAM = 1      /* the same polynomial iterated on the s x s Gram
                           ("About Muon: Why Not Adam", "Gram
                           Newton-Schulz"), in segments of two steps: a
                           fresh Gram every second step; equal in exact
                           arithmetic, fewer FLOPs when max(m,n) >> min(m,n).
                           bf16 and single-CTA tiles only; matrices on the
                           on-chip small path keep the standard form       */
};

#define MUON_FLAG_GRAD_BF16 1

typedef struct muon_config {
  int scale_mode;             /* enum muon_scale_mode; default MOONLIGHT    */
  float extra_scale;          /* multiplies the scale; default 1.0
                                 ("Why Muon Works", configuration block)   */
  int ns_precision;           /* enum muon_ns_precision; default BF16      */
  int check_nonfinite;        /* 1: count non-finite u entries; read back
                                 with muon_get_status. Default 0           */
  int num_sms;                /* persistent-grid width; 0 = all SMs        */
  size_t workspace_cap_bytes; /* 0 = no cap. With a cap below the
                                 workspace of a shape table, consecutive
                                 matrices are packed into groups whose
                                 workspace fits and the step runs the groups
                                 one after another through one shared
                                 workspace (muon_plan_groups gives the
                                 partition); a matrix that alone exceeds the
                                 cap fails with MUON_ERR_OOM               */
  double wait_timeout_s;      /* limit of every device-side wait; a wait
                                 that runs out sets the error word and the
                                 kernel returns. Default 2.0 seconds       */
  int small_path;             /* 1: matrices with min(m,n) <= 128 and
                                 max(m,n) <= 512 run all iterations in one
                                 on-chip kernel (one CTA each); 0: every
                                 matrix uses the tiled phases. Default 1   */
  int ns_algorithm;           /* enum muon_ns_algorithm; default STANDARD  */
  int deterministic;          /* 1: the per-matrix sum of squares is added
                                 in a fixed order (per-block partials, then
                                 one more launch), so repeated steps on the
                                 same inputs are bitwise identical; 0
                                 (default): one double atomic per block    */
  int cta_pair;               /* 1: tiled phases use 256 x 256 tiles on CTA
                                 pairs (tcgen05 cta_group::2); 0: 128 x 256
                                 tiles on single CTAs. Default 0 (the
                                 single-CTA tiles measured 2-10% faster on
                                 the Llama-shaped set under the power cap) */
  int fused_apply;            /* 1 (default): in muon_step and
                                 muon_step_host, with bf16 Newton-Schulz in
                                 the standard form on single-CTA tiles,
                                 ns_steps >= 1, no active matrix on the
                                 small path and every parameter's rows
                                 16-byte aligned (n % 4 == 0, aligned base),
                                 the last combine's epilogue writes
                                 p' = p (1 - lr wd) - lr scale O itself
                                 (O rounded to bf16 first, so p' is bitwise
                                 the same as with 0; p moved by bulk copies)
                                 and O is not stored. 0, or any other step:
                                 O is stored in the workspace buffer
                                 muon_plan_query names and a separate pass
                                 applies it                                 */
} muon_config;

/* plan_flags of muon_plan_query */
#define MUON_PLAN_SMALL_PATH 1
#define MUON_PLAN_CTA_PAIR 2

typedef struct muon_handle muon_handle;

/* Fill *cfg with the defaults listed above. Returns MUON_ERR_INVALID_ARG if
 * cfg is NULL. Needs no GPU. */
int muon_config_init(muon_config* cfg);

/* Create a handle on CUDA device `device`. cfg may be NULL (defaults).
 * Allocates nothing large: the workspace is allocated on the first step of
 * a given shape table and reused while the table is unchanged. Fails with
 * MUON_ERR_NO_DEVICE / MUON_ERR_UNSUPPORTED when the device is missing or
 * not sm_100. *out is set only on success. */
int muon_init(int device, const muon_config* cfg, muon_handle** out);

/* Wait for the handle's work, free its workspace and the handle.
 * NULL is accepted and ignored. */
int muon_destroy(muon_handle* h);

/* One Muon step over `count` matrices ("About Muon: Why Not Adam", "The
 * whole thing, in about forty lines").
 *   params[i]  : device pointer, fp32 m x n, updated in place.
 *   grads[i]   : device pointer, fp32 or bf16 m x n (shapes flag); NULL
 *                skips matrix i entirely (its param and momentum are left
 *                unchanged), like a parameter without a gradient.
 *   momenta[i] : device pointer, fp32 m x n, updated in place; the caller
 *                zero-initialises it before the first step.
 *   params, grads, momenta are HOST arrays of `count` device pointers.
 *   shapes     : host int32[count][3], see the conventions above.
 *   lr, beta, wd : learning rate, momentum (0 <= beta < 1), decoupled
 *                weight decay (p is multiplied by 1 - lr*wd).
 *   nesterov   : 1 = u = g + beta*(m' - g); 0 = u = m'.
 *   ns_steps   : number of quintic iterations, 0..64 (0 returns the
 *                normalised u).
 *   coeffs     : host float[3] = (a, b, c); NULL = (3.4445, -4.7750, 2.0315).
 *   stream     : cudaStream_t.
 * Scale mode, extra scale and precision come from the handle's config.
 * The first call for a shape table builds the plan and the workspace
 * (device allocation and a host-to-device copy of the tables; do it before
 * any stream capture). The per-call pointer tables live in a ring of eight
 * device slots made with the plan: a call with pointers seen recently reuses
 * its slot; a call with new pointers (fresh tensors every step are fine)
 * takes the least recently used slot and uploads with one cudaMemcpyAsync on
 * `stream` from pinned staging, without allocating or synchronising the
 * device. Calls with the same shape table and pointers as an earlier
 * uncaptured call only enqueue kernels and may be captured in a CUDA graph;
 * the slots such a capture uses are kept for the graph (never overwritten)
 * until the shape table changes or the handle is destroyed. A call with new
 * pointers on a stream being captured fails with MUON_ERR_INVALID_ARG (the
 * upload cannot be captured). Matrices with a NULL gradient drop out of the
 * Newton-Schulz launches (their tiles are not listed). */
int muon_step(muon_handle* h, float* const* params, const void* const* grads,
              float* const* momenta, const int32_t* shapes, int count,
              float lr, float beta, int nesterov, float wd, int ns_steps,
              const float* coeffs, void* stream);

/* muon_step with a coefficient schedule: coeff_table is a host array of
 * table_rows x 3 floats (a, b, c); table_rows = 1 applies one triple to every
 * iteration, table_rows = ns_steps gives iteration t its own row. A sequence
 * of odd polynomials still acts on the singular values only ("About Muon:
 * Why Not Adam", "The lemma that makes it possible"); the pages name
 * Chebyshev-type compositions ("Gram Newton-Schulz" section) but print no
 * coefficients, so none are built in. Otherwise identical to muon_step. */
int muon_step_schedule(muon_handle* h, float* const* params,
                       const void* const* grads, float* const* momenta,
                       const int32_t* shapes, int count, float lr, float beta,
                       int nesterov, float wd, int ns_steps,
                       const float* coeff_table, int table_rows, void* stream);

/* QK-Clip after a Muon step ("The Optimizer Wars", MuonClip): for every
 * weight i (fp32 W_q or W_k, device pointer, rows x cols, updated in place)
 * with shapes[i] = {rows, cols, head_rows} (rows a multiple of head_rows),
 * the rows of head h are multiplied by sqrt(tau / s_max[i][h]) when
 * s_max[i][h] > tau (gamma_h = min(1, tau / S_max^h) applied as
 * sqrt(gamma_h) to each of W_q^h and W_k^h), else left unchanged (NaN
 * included). s_max is a host array of device float arrays, one per weight,
 * rows / head_rows entries each: the largest attention logit per head seen
 * in the step, tracked by the caller's forward pass. tau > 0 (the pages use
 * 100). One kernel per weight. */
int muon_qk_clip(muon_handle* h, float* const* weights, const int32_t* shapes,
                 const float* const* s_max, int count, float tau, void* stream);

/* Same step with every tensor in HOST memory. The matrices are split into
 * up to 32 chunks of consecutive matrices with about equal element counts;
 * while chunk c is computed, chunk c+1 is copied in and chunk c-1 copied
 * out, on three library streams (copy-in, compute, copy-out) that start
 * after the work already queued on `stream`; `stream` waits for the last
 * copy-out. Pinned host memory is needed for the copies to overlap. Only
 * matrices with a gradient are copied. The host buffers must stay valid and
 * untouched until `stream` reaches that point, and calls on one handle must
 * be ordered by the caller (one stream). Staging (three chunk slots, 12
 * bytes per element of the largest chunk) is allocated on first use per
 * shape table, in addition to the workspace: the workspace cap does not
 * bound it. Under a cap that splits the set into groups, the chunks are
 * those groups. */
int muon_step_host(muon_handle* h, float* const* params,
                   const void* const* grads, float* const* momenta,
                   const int32_t* shapes, int count, float lr, float beta,
                   int nesterov, float wd, int ns_steps, const float* coeffs,
                   void* stream);

/* ---- Stage entry points (each a row of the step; used by the tests and
 *      the NS-only sweep). Same validation and conventions. ---- */

/* Stage 1 (momentum, Nesterov, norm, cast). For each matrix with a
 * non-NULL grad: momenta[i] <- beta*m + (1-beta)*g (in place);
 * u = nesterov ? g + beta*(m' - g) : m'; y[i] <- cast(u) in X layout
 * (bf16 round-to-nearest-even, or fp32 in the fp32 mode);
 * sumsq[i] <- sum of u^2 (fp64, device array of count doubles, overwritten;
 * left unchanged for skipped matrices). */
int muon_momentum_norm(muon_handle* h, const void* const* grads,
                       float* const* momenta, void* const* y, double* sumsq,
                       const int32_t* shapes, int count, float beta,
                       int nesterov, void* stream);

/* Stage 2 (Newton-Schulz). For each matrix: X0 = x_in[i] * alpha with
 * alpha = 1/(sqrt(sumsq[i]) + 1e-7) when sumsq (device array) is non-NULL,
 * else alpha = 1; if m > n the iteration runs on the transpose (through
 * operand layout, no transposed copy); ns_steps iterations with `coeffs`;
 * result in x_out[i]. x_in and x_out are device pointers in X layout and
 * must not overlap; x_in is not modified. ns_steps = 0 copies alpha*x_in
 * (rounded to the storage type) to x_out. */
int muon_newton_schulz(muon_handle* h, const void* const* x_in,
                       void* const* x_out, const double* sumsq,
                       const int32_t* shapes, int count, int ns_steps,
                       const float* coeffs, void* stream);

/* Stage 3 (apply). params[i] <- params[i]*(1 - lr*wd) - lr*scale*o_scale*O
 * with O = o[i] (X layout, upcast exactly to fp32), scale from the handle's
 * scale mode and extra scale, o_scale = 1/(sqrt(sumsq[i]) + 1e-7) when
 * sumsq (device array) is non-NULL, else 1. A NULL o[i] skips matrix i. */
int muon_apply(muon_handle* h, float* const* params, const void* const* o,
               const double* sumsq, const int32_t* shapes, int count,
               float lr, float wd, void* stream);

/* ---- Plan, workspace and status ---- */

/* Integer plan tables for a shape table, computed on the host (needs no
 * GPU). plan_flags: MUON_PLAN_SMALL_PATH and MUON_PLAN_CTA_PAIR, as the
 * small_path and cta_pair fields of muon_config. Any output pointer may be
 * NULL.
 *   ws_bytes      : total workspace bytes for `ns_precision`.
 *   region_offsets: int64[count][4], byte offsets of X0, X1, A, B.
 *   ntiles        : int32[4], tile counts of the Gram, polynomial and
 *                   combine phases, and the number of small-path matrices.
 *   tiles         : int32[ntiles[0]+...+ntiles[3]][3] =
 *                   {matrix, row tile, column tile} for the three phases,
 *                   one after the other, then {matrix, 0, 0} for each
 *                   small-path matrix.
 *   chunk_prefix  : int64[count+1], elementwise chunks before matrix i.
 * Call once with tiles = NULL to learn ntiles. */
int muon_plan_query(const int32_t* shapes, int count, int ns_precision,
                    int plan_flags, int64_t* ws_bytes, int64_t* region_offsets,
                    int32_t* ntiles, int32_t* tiles, int64_t* chunk_prefix);

/* Matrix groups of a shape table under a workspace cap (needs no GPU). The
 * workspace holds one double per matrix, then per group the X0, X1, A and B
 * regions of its matrices; groups run one after another and share it. With
 * cap = 0, or when everything fits under the cap, there is one group.
 *   ngroups       : number of groups.
 *   group_bounds  : int32[count + 1]; group g is matrices
 *                   group_bounds[g] .. group_bounds[g+1]-1 (entries past
 *                   ngroups are not written).
 *   region_offsets: int64[count][4], byte offsets of X0, X1, A, B.
 *   ws_bytes      : workspace bytes (sum-of-squares block + largest group).
 * plan_flags as for muon_plan_query. A matrix whose regions alone exceed the
 * cap is MUON_ERR_OOM; bad shapes are MUON_ERR_INVALID_ARG. Any output
 * pointer may be NULL. */
int muon_plan_groups(const int32_t* shapes, int count, int ns_precision,
                     int plan_flags, size_t cap, int32_t* ngroups,
                     int32_t* group_bounds, int64_t* region_offsets,
                     int64_t* ws_bytes);

/* Workspace bytes the handle would allocate for this shape table
 * (excluding muon_step_host staging; under the handle's cap, the grouped
 * workspace). */
int muon_workspace_size(muon_handle* h, const int32_t* shapes, int count,
                        size_t* bytes);

/* Device base address and size of the current workspace (for inspection by
 * tests; the layout is given by muon_plan_query). */
int muon_workspace_ptr(muon_handle* h, void** base, size_t* bytes);

/* Wait for `stream`, then report the device error word (0 = none, else the
 * code of the first expired wait) and the non-finite count, and clear both.
 * Returns MUON_ERR_TIMEOUT if the error word was set, MUON_ERR_NONFINITE if
 * only the counter was non-zero, else MUON_OK. Either output may be NULL. */
int muon_get_status(muon_handle* h, void* stream, int32_t* error_word,
                    uint64_t* nonfinite_count);

/* Number of kernels the last muon_step / stage call enqueued. */
int muon_last_launch_count(muon_handle* h, int32_t* launches);

/* Kernel kinds reported by muon_profile_read. */
enum muon_kernel_kind {
  MUON_KERNEL_MOMENTUM_NORM = 0, /* stage 1                                  */
  MUON_KERNEL_NS_GRAM = 1,       /* tensor-core Gram phase, all matrices      */
  MUON_KERNEL_NS_POLY = 2,       /* tensor-core polynomial phase              */
  MUON_KERNEL_NS_COMB = 3,       /* tensor-core combine phase                 */
  MUON_KERNEL_APPLY = 4,         /* stage 3                                   */
  MUON_KERNEL_SCALE_COPY = 5,    /* zero-iteration Newton-Schulz stage        */
  MUON_KERNEL_NS_FP32 = 6,       /* fp32 debug phase (one matrix)             */
  MUON_KERNEL_NS_SMALL = 7,      /* on-chip small-matrix path, all iterations */
  MUON_KERNEL_NORM_REDUCE = 8,   /* fixed-order norm sum (deterministic mode) */
  MUON_KERNEL_NS_SYM = 9         /* symmetric-product phase of the Gram form  */
};

/* Per-launch timing for measurements. With max_calls > 0, each of the next
 * max_calls step / stage calls records a CUDA event on its stream before and
 * after every kernel it enqueues (at most 256 kernels per call); events are
 * created here, so call this outside stream capture. max_calls = 0 stops
 * recording and frees the events. Recording adds two event records per
 * kernel and nothing else. */
int muon_profile_enable(muon_handle* h, int max_calls);

/* Wait for the recorded events and return, in launch order, the kind
 * (enum muon_kernel_kind) and duration in milliseconds of up to `max`
 * recorded kernels; *n receives the number written. Clears the record so
 * the next calls start from an empty record (max_calls calls again). */
int muon_profile_read(muon_handle* h, int32_t* kinds, float* ms, int max, int32_t* n);

/* Thread-local text of the last error ("" if none). Never NULL. */
const char* muon_last_error(void);

/* Library version string. */
const char* muon_version(void);

/* ---- Allocation-free Newton-Schulz stage ----
 *
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory when they run the stage: a process
 * whose device memory belongs to its own fixed-budget pool allocator (a
 * cudaMalloc from outside the pool fails or takes memory the pool counts
 * on), or a serving process that reserved its memory at start-up and must
 * keep its device footprint fixed while it runs.
 *
 * Same computation and the same tensor-core kernels as muon_newton_schulz,
 * in bf16, on the CURRENT device, with no handle. All scratch (X ping-pong
 * buffers, Gram and polynomial matrices, tile lists, tensor maps, status
 * word) lives in one static device array of MUON_NOALLOC_SCRATCH_BYTES that
 * every GPU which loads this library holds until the process exits. The call
 * allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *
 *   x_in, x_out : host arrays of `count` device pointers in X layout (bf16),
 *                 owned by the caller; x_in is read only; they must not
 *                 overlap.
 *   sumsq       : device array of count doubles or NULL (as in
 *                 muon_newton_schulz).
 *   shapes, count, ns_steps (0..64), coeffs (NULL = default): as in
 *                 muon_newton_schulz.
 *   error_word  : device int32 or NULL; receives 0, or the code of a
 *                 device-side wait that ran out (results then invalid).
 *   stream      : cudaStream_t.
 * Errors (MUON_ERR_INVALID_ARG, message in muon_last_error): NULL, unaligned
 * or overlapping matrices, a matrix that is not device memory of the
 * current device, non-finite coefficients, and a call on a stream that is
 * being captured (each call writes its tables from host memory that lives
 * only during the call).
 * A shape table whose scratch (tables plus the workspace muon_plan_query
 * reports) exceeds MUON_NOALLOC_SCRATCH_BYTES is rejected with
 * MUON_ERR_INVALID_ARG and a message giving both sizes.
 * The first call on a device looks up the array's device address there
 * (cudaGetSymbolAddress) and the device's properties; make that first call
 * before any stream capture. Every call reuses the same array and leaves the
 * previous call's contents in it (the status word is cleared at the start
 * of each call, the tables are rewritten): calls whose work overlaps on the
 * GPU (different streams, different host threads) race on it; calls on one
 * stream are ordered. */
#define MUON_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
int muon_newton_schulz_noalloc(const void* const* x_in, void* const* x_out, const double* sumsq,
                               const int32_t* shapes, int count, int ns_steps, const float* coeffs,
                               int32_t* error_word, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MUON_NS_H */
