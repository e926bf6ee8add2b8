/*
 * muon.h -- C ABI of the B200 (sm_100a) Muon optimizer step.
 *
 * One call performs one Muon step over a grouped list of hidden-layer 2D weight
 * matrices, as the page "Muon: An optimizer for hidden layers in neural networks"
 * (papers.chlience.com synthesis note) defines it in section 4 "Muon 的算法定义":
 *
 *   B <- mu*B + G                                     (eq. 1, momentum)
 *   U <- G + mu*B   (Nesterov)   or   U <- B          (section 4: the Nesterov variant)
 *   X <- U, or U^T when rows > cols                   (section 4: smaller Gram)
 *   X <- X / (||X||_F + eps)                          (section 4: Frobenius normalisation)
 *   5 x  X <- aX + b(XX^T)X + c(XX^T)^2 X             (eqs. 4, 5: (a,b,c) = (3.4445,-4.7750,2.0315))
 *   O <- X, or X^T when transposed
 *   W <- W - lr*wd*W - lr*s*O                         (eq. 3; "关键实验/定理" result 2: decoupled
 *                                                      weight decay and a per-shape scale s)
 *
 * Every step runs in hand-written CUDA kernels on one GPU; there is no CPU
 * fallback.  No type of any framework appears in these signatures: pointers are
 * plain host or device addresses, sizes are ints, streams are cudaStream_t
 * passed as void*.
 *
 * Conventions for every entry point
 *  - Matrices are row-major, densely packed (row stride = cols elements).
 *  - "device pointer" means memory of the handle's device (cudaMalloc / torch
 *    CUDA tensors); "host pointer" means ordinary or pinned host memory.
 *  - Pointer arrays inside descriptors (W, G, B, ...) are HOST arrays of
 *    `count` pointers; the library reads them only during the call.
 *  - Work is enqueued on `stream` and returns before it completes.  The caller
 *    keeps every buffer alive, and unmodified by other work, until the stream
 *    reaches that point.  Errors detected on the host are returned before any
 *    launch, with no state touched; launch failures return MUON_ERR_CUDA.
 *  - Non-finite values in G propagate to W and B as NaN/Inf; they are not an
 *    error.
 *  - A handle is not thread-safe: one host thread at a time per handle.
 */
#ifndef MUON_B200_H
#define MUON_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MUON_ABI_VERSION 1

typedef enum {
    MUON_OK = 0,
    MUON_ERR_INVALID = 1,        /* bad argument: null pointer, size <= 0, bad enum, ...      */
    MUON_ERR_UNSUPPORTED = 2,    /* device is not sm_100, or a layout the kernels do not take  */
    MUON_ERR_OOM = 3,            /* device buffer allocation failed, or would pass the cap set
                                    by muon_set_memory_limit                                  */
    MUON_ERR_CUDA = 4,           /* a CUDA runtime call or kernel launch failed                */
    MUON_ERR_DEVICE_TIMEOUT = 5  /* a kernel gave up a bounded wait (reported by muon_sync)    */
} muon_status;

typedef enum { MUON_BF16 = 0, MUON_FP32 = 1 } muon_dtype;

/* MUON_PREC_BF16: tensor-core GEMMs with bf16 operands and fp32 accumulation; the
 *   iterate X is carried as a pair of bf16 arrays X = hi + lo (about 16 significant
 *   bits) so that the aX term keeps that precision (the timed path).
 * MUON_PREC_FP32_DEBUG: every Newton-Schulz GEMM in fp32 FFMA (no TF32). */
typedef enum { MUON_PREC_BF16 = 0, MUON_PREC_FP32_DEBUG = 1 } muon_precision;

/* Per-shape update scale s ("关键实验/定理" result 2; the page prints no formula):
 *   NONE: s = 1.   MATCH_RMS: s = rms_target * sqrt(max(rows, cols)), which gives a
 *   full-rank semi-orthogonal O the update RMS rms_target.   CUSTOM: s = group.scale. */
typedef enum { MUON_SCALE_NONE = 0, MUON_SCALE_MATCH_RMS = 1, MUON_SCALE_CUSTOM = 2 } muon_scale_mode;

typedef struct {
    float lr;            /* eta in eq. 3                                      */
    float momentum;      /* mu in eq. 1, 0 <= mu < 1                          */
    float weight_decay;  /* lambda: W <- W - lr*lambda*W - lr*s*O             */
    float eps;           /* X / (||X||_F + eps); the pages give none; 1e-7    */
    float rms_target;    /* MATCH_RMS only                                    */
    int nesterov;        /* 1: U = G + mu*B, 0: U = B                         */
    int ns_steps;        /* Newton-Schulz iterations, 0..16; 5 on the pages   */
    float ns_a, ns_b, ns_c;
    int scale_mode;      /* muon_scale_mode */
    int precision;       /* muon_precision  */
} muon_config;

/* Same-shape matrices.  W: fp32 rows x cols (updated in place); G: gradient,
 * bf16 or fp32 (read only); B: fp32 momentum (updated in place; zero before the
 * first step).  All device pointers, 4-byte aligned at least; 16-byte aligned
 * pointers and cols % 8 == 0 take the vectorised path.  W and B are written, so no
 * W or B may share memory with any W, G or B of the call (MUON_ERR_INVALID); one
 * gradient buffer may be given for several matrices. */
typedef struct {
    int rows, cols, count;
    int grad_dtype;          /* muon_dtype */
    float scale;             /* MUON_SCALE_CUSTOM only */
    float* const* W;
    const void* const* G;
    float* const* B;
} muon_group;

typedef struct muon_handle muon_handle;

/* Fills the defaults: lr 0.02, momentum 0.95, nesterov 1, ns_steps 5,
 * (a,b,c) = (3.4445, -4.7750, 2.0315), eps 1e-7, weight_decay 0, scale NONE,
 * rms_target 0.2, precision BF16. */
void muon_config_default(muon_config* cfg);

/* Host-only checks, usable without a GPU.  MUON_OK or MUON_ERR_INVALID. */
muon_status muon_validate_config(const muon_config* cfg);
muon_status muon_validate_groups(const muon_group* groups, int n_groups);

/* Creates a handle on `device` (which must be sm_100).  Allocates no large
 * memory: the workspace is allocated by the first muon_step / muon_orthogonalize
 * that needs it, and grows when a later call needs more (so the first call on a
 * new shape set must not be inside a CUDA graph capture).  *out is set only on
 * MUON_OK. */
muon_status muon_create(const muon_config* cfg, int device, muon_handle** out);

/* Replaces the hyperparameters of a handle (validated first). */
muon_status muon_set_config(muon_handle* h, const muon_config* cfg);

/* Caps the device memory the handle may hold (workspace, host-step staging and
 * phase scratch together) at `bytes`; 0 removes the cap.  Buffers already held
 * are kept.  A later call whose buffers would grow past the cap returns
 * MUON_ERR_OOM before it launches anything, leaving W, B and the caller's other
 * buffers untouched; the handle stays usable (raise the cap, or call with fewer
 * matrices).  MUON_ERR_INVALID for a NULL handle. */
muon_status muon_set_memory_limit(muon_handle* h, size_t bytes);

/* Device bytes the handle holds now (*bytes).  MUON_ERR_INVALID for NULL arguments. */
muon_status muon_memory_held(const muon_handle* h, size_t* bytes);

/* One Muon step for every matrix of every group (section 4 eqs. 1-5, eq. 3 with
 * result 2's decay and scale).  Device pointers.  Work is enqueued on `stream`
 * (a cudaStream_t; NULL = legacy default stream). */
muon_status muon_step(muon_handle* h, const muon_group* groups, int n_groups, void* stream);

/* The same step with W, G and B in HOST memory (pinned memory gives full copy
 * bandwidth): G, W and B are copied to a library-owned device staging area,
 * the step runs, and the new W and B are copied back, all on `stream`.  The host
 * buffers must stay untouched until the stream reaches the end of the call. */
muon_status muon_step_host(muon_handle* h, const muon_group* groups, int n_groups, void* stream);

/* The step without its weight update, for callers that apply the update
 * themselves (the data-parallel sharded step: each rank computes the update
 * direction of the matrices it owns, the ranks exchange O, and every rank applies
 * every O with muon_apply).  B <- mu*B + G and the Newton-Schulz direction O are
 * computed exactly as in muon_step; O (rows x cols, de-oriented, scale s not
 * applied) is written to O[k] in out_dtype -- fp32, or bf16 rounded to nearest --
 * and W is neither read nor written.  G: bf16 or fp32, read only; B: fp32,
 * updated in place; O: device buffers, written.  B and O may not overlap any
 * buffer of the call (MUON_ERR_INVALID).  Same conventions as muon_group. */
typedef struct {
    int rows, cols, count;
    int grad_dtype;          /* muon_dtype of G */
    int out_dtype;           /* muon_dtype of O */
    const void* const* G;
    float* const* B;
    void* const* O;
} muon_direction_group;

muon_status muon_step_direction(muon_handle* h, const muon_direction_group* groups, int n_groups, void* stream);

/* The weight update of eq. 3 with result 2's decay and scale, from a caller's O:
 * W <- W - lr*wd*W - lr*s*O for every matrix, with the handle's lr, weight_decay and
 * scale mode (s from the shape for MATCH_RMS, group.scale for CUSTOM, 1 for NONE).
 * W: fp32 rows x cols, device, updated in place; O: rows x cols in o_dtype (fp32 or
 * bf16), device, read only.  No W may overlap any W or O of the call
 * (MUON_ERR_INVALID).  The first call with a new set of pointers uploads a small
 * table and synchronises the stream. */
typedef struct {
    int rows, cols, count;
    int o_dtype;             /* muon_dtype of O */
    float scale;             /* MUON_SCALE_CUSTOM only */
    float* const* W;
    const void* const* O;
} muon_apply_group;

muon_status muon_apply(muon_handle* h, const muon_apply_group* groups, int n_groups, void* stream);

/* Orthogonalisation alone: O = NS_k(M / (||M||_F + eps)) per matrix, with the
 * orientation rule of section 4 and the handle's ns_steps / coefficients /
 * precision.  M: bf16 or fp32 rows x cols (device, read only); O: fp32 rows x cols
 * (device, written; it may not overlap any M or O of the call).  Same conventions
 * as muon_group. */
typedef struct {
    int rows, cols, count;
    int in_dtype;            /* muon_dtype */
    const void* const* M;
    float* const* O;
} muon_ortho_group;

muon_status muon_orthogonalize(muon_handle* h, const muon_ortho_group* groups, int n_groups, void* stream);

/* One Newton-Schulz building block on caller buffers, for per-kernel checks and
 * for callers composing their own iteration (section 4 eq. 4 grouped as
 * A = XX^T, P = bA + cA^2, X' = aX + PX).  All buffers are device memory, densely
 * packed [count][rows][cols], 16-byte aligned.  With precision BF16, m and n must
 * be multiples of 8.
 *
 *  MUON_NS_GRAM:   out(m x m)   = alpha * X X^T            X = x_op (m x n)
 *  MUON_NS_POLY:   out(m x m)   = beta * A + alpha * A A   A = a_in (m x m, symmetric)
 *  MUON_NS_UPDATE: X'(m x n)    = alpha * P X + beta * X   P = a_in (m x m)
 *
 * BF16 precision: x_op, a_in and the GRAM / POLY out are bf16.  The iterate of
 * UPDATE is a pair of bf16 arrays, X = x_op + x_master (high part, which is also
 * the GEMM operand, and low part); the result is written the same way,
 * X' = out + out_op with out = bf16(X') and out_op = bf16(X' - out).
 * FP32_DEBUG precision: every buffer is fp32; UPDATE reads X = x_op for the
 * product and x_master for the beta term, and writes X' to out. */
typedef enum { MUON_NS_GRAM = 0, MUON_NS_POLY = 1, MUON_NS_UPDATE = 2 } muon_ns_phase;

typedef struct {
    int phase;               /* muon_ns_phase  */
    int precision;           /* muon_precision */
    int m, n, count;
    float alpha, beta;
    const void* x_op;
    const void* a_in;
    const void* x_master;
    void* out;
    void* out_op;
} muon_ns_phase_args;

muon_status muon_ns_phase_run(muon_handle* h, const muon_ns_phase_args* args, void* stream);

/* QK-Clip of MuonClip ("关键实验/定理" result 3: after the Muon step, each attention
 * head's query and key projections are rescaled according to the head's maximum
 * logit; the page gives no formula).  With gamma_h = min(1, tau / max_logits[h]),
 * the rows of head h -- rows h*head_dim .. (h+1)*head_dim - 1 -- of Wq and of Wk
 * are multiplied by sqrt(gamma_h), so every logit of the head scales by gamma_h.
 * Wq, Wk: fp32 (n_heads*head_dim) x cols, row-major, device, updated in place
 * (Wk may be NULL); max_logits: n_heads floats, device, produced by the caller's
 * attention; tau > 0. */
muon_status muon_qk_clip(muon_handle* h, float* Wq, float* Wk, const float* max_logits, int n_heads, int head_dim,
                         int cols, float tau, void* stream);

/* Waits for the handle's work on `stream`, then reports a kernel that gave up a
 * bounded wait (MUON_ERR_DEVICE_TIMEOUT, flag cleared) or an asynchronous CUDA
 * error (MUON_ERR_CUDA). */
muon_status muon_sync(muon_handle* h, void* stream);

/* Copies the Frobenius norms ||U||_F of the last step's matrices (groups in
 * order, matrices in order) to `out` (host, `cap` floats).  Synchronises the
 * stream.  *n_out gets the number of matrices. */
muon_status muon_last_norms(muon_handle* h, float* out, int cap, int* n_out, void* stream);

/* Copies the update direction O of the last muon_step for matrix `index` of
 * group `group` (fp32, rows x cols, de-oriented) to the device buffer `dst`, on
 * `stream`.  Valid until the next step or orthogonalisation on the handle. */
muon_status muon_last_update(muon_handle* h, int group, int index, float* dst, void* stream);

/* RMS of the update that the last muon_step applied to each matrix,
 * lr * |s| * sqrt(sum(O^2) / (rows * cols)) with the matrix's per-shape scale s
 * (the "实践 checklist" of the Muon note asks for the update RMS to be logged; with
 * MUON_SCALE_MATCH_RMS and a full-rank O it is close to lr * rms_target).  Computed
 * on the device from the final iterate in a fixed summation order, then copied to
 * `out` (host, `cap` floats; groups in order, matrices in order); synchronises the
 * stream.  *n_out gets the number of matrices.  After muon_orthogonalize it reports
 * lr * RMS(O) of that call's outputs. */
muon_status muon_last_update_rms(muon_handle* h, float* out, int cap, int* n_out, void* stream);

/* Per-phase device timing.  While enabled, every launch of the step is
 * bracketed by CUDA events recorded on the launching stream.  muon_timing_read
 * synchronises the stream, adds the elapsed times of all launches since the last
 * read per phase, and writes ms[k] and launches[k] for k < n_kinds (6 kinds:
 * 0 momentum+norm, 1 norm finalize, 2 Gram GEMM, 3 polynomial GEMM, 4 update
 * GEMM, 5 apply). */
#define MUON_TIMING_KINDS 6
muon_status muon_timing_enable(muon_handle* h, int enable);
muon_status muon_timing_read(muon_handle* h, double* ms, int* launches, int n_kinds, void* stream);

/* Releases the workspace and the handle (synchronises the device first). */
muon_status muon_destroy(muon_handle* h);

/* Message of the last failing call on this handle ("" if none).  Valid until
 * the next call on the handle. */
const char* muon_last_error(const muon_handle* h);
const char* muon_status_string(muon_status s);

/* ---- no-allocation entry point -----------------------------------------------
 * The pages have no counterpart to this call.  It is for callers that cannot
 * allocate device memory at all -- a runtime that owns a fixed device-memory pool
 * and forbids allocations by anyone else, or code that runs while another
 * component holds the allocator -- and so can use neither muon_create (which
 * allocates an error word) nor the workspace of muon_step.
 *
 * It runs the momentum phase of ONE matrix (rows x cols, row-major, densely
 * packed, device pointers on the current device): B <- momentum*B + G in place;
 * the update direction U = G + momentum*B (nesterov = 1) or U = B (nesterov = 0)
 * written to U_out (fp32, optional: NULL skips it); and ||U||_F written to
 * norm_out (one float in device memory).  G is bf16 or fp32 (grad_dtype).
 *
 * It calls no cudaMalloc, cudaFree or other allocating routine and needs no
 * handle.  Its only scratch, one fp64 partial sum per 8192 elements, is a static
 * device array of MUON_NOALLOC_MAX_BLOCKS doubles (512 KiB) that every GPU which
 * loads the library holds until the process exits; a matrix of more than
 * MUON_NOALLOC_MAX_BLOCKS * 8192 elements is rejected with MUON_ERR_UNSUPPORTED.
 * Every call looks up the array's device address (cudaGetSymbolAddress) on the
 * current device, so the address stays right after cudaDeviceReset or a new
 * primary context.  With the CUDA runtime's lazy module loading (the default since
 * CUDA 12) the first call on a device (and the first after a reset) is when the
 * module is loaded and the 512 KiB are reserved on the device: make it a warm-up
 * call while device memory is still available and before any stream capture.
 * B, U_out and norm_out are written, so none of them may overlap another buffer
 * of the call (MUON_ERR_INVALID).
 * All calls share the one array, and each call overwrites the partial sums it
 * reads: calls whose work overlaps on the GPU (unordered streams) race and give
 * wrong norms.  err_msg (optional host buffer of err_cap bytes) receives a
 * message on failure. */
#define MUON_NOALLOC_MAX_BLOCKS 65536
muon_status muon_momentum_norm_noalloc(int rows, int cols, int grad_dtype, const void* G, float* B, float* U_out,
                                       float momentum, int nesterov, float* norm_out, void* stream,
                                       char* err_msg, int err_cap);

/* ---- planner queries (host only, no GPU needed) ------------------------------
 * The persistent tensor-core GEMMs walk a tile list built once per shape set.
 * muon_plan_tiles writes the list a launch of `phase` would walk for the given
 * groups: 4 ints per tile (group, matrix, tile_row, tile_col), tiles of
 * muon_plan_tile_m() x muon_plan_tile_n() output elements.  GRAM/POLY lists hold
 * only tiles that touch the upper triangle (col >= row); UPDATE lists cover the
 * m x n iterate.  shapes: 3 ints per group (rows, cols, count) of the weight.
 * Returns MUON_ERR_INVALID if cap is too small (*n_tiles still gets the size). */
int muon_plan_tile_m(void);
int muon_plan_tile_n(void);
muon_status muon_plan_tiles(const int* shapes, int n_groups, int phase, int* out, int cap, int* n_tiles);

/* Work units of one launch of the two-CTA GEMM kernel built for `clusters`
 * two-CTA clusters: 11 ints per unit (cluster, group, matrix, tile_row, tile_col,
 * k_begin, k_end, kind, slot, nslots, n_half), k in 64-element blocks.
 * split = 0 (the default schedule): whole tiles, the last partial round cut along
 * N into 128-column halves when they fit one per cluster (n_half 1 / 2).
 * split = 1: the K-blocks of the last partial round are divided over all clusters;
 * kind 0 = a whole tile; 1 = the first K range of a split tile, which adds the
 * partial sums of slots [slot, slot + nslots); 2 = a later K range, which stores
 * its partial sum to `slot`.  Same conventions as muon_plan_tiles. */
muon_status muon_plan_units(const int* shapes, int n_groups, int phase, int clusters, int split, int* out, int cap,
                            int* n_units);

#ifdef __cplusplus
}
#endif

#endif /* MUON_B200_H */
