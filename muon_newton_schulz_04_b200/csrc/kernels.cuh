// kernels.cuh -- device-side descriptors and kernel launchers of the Muon step.
//
// Layout in HBM (library-owned workspace, per group of same-shape matrices):
//   xb[2]  bf16 [count][m][ldn]   high part of the iterate, hi = bf16(X), which is
//                                 also the tensor-core operand (ping-pong)
//   xl     bf16 [count][m][ldn]   low part, lo = bf16(X - hi): X = hi + lo carries
//                                 about 16 significant bits (updated in place)
//   a, p   bf16 [count][m][ldm]   Gram matrix A = XX^T and P = bA + cA^2
// The fp32 debug path keeps X in two fp32 ping-pong buffers and A, P in fp32.
// with m = min(rows, cols), n = max(rows, cols), ldm / ldn rounded up to 8
// elements so that every row starts on a 16-byte boundary (a TMA requirement).
// The caller's W, G, B stay where the caller put them.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace muon {

// GEMM tile shape of the tensor-core kernels: 128 x 256 output elements per
// tile, 64-element K blocks (one 128-byte swizzle atom of bf16).
constexpr int TC_BM = 128;
constexpr int TC_BN = 256;
constexpr int TC_BK = 64;

enum GemmMode { MODE_GRAM = 0, MODE_POLY = 1, MODE_UPDATE = 2 };

// Elementwise work unit: one matrix.  Built on the host whenever the caller's
// pointers or the plan change.
struct EwSeg {
    const void* g;        // gradient (step) or input M (orthogonalize): rows x cols
    float* b;             // momentum buffer (nullptr: no momentum, U = G)
    float* w;             // weight (apply) or output O (copy-out)
    float* xf0;           // fp32 debug path: X0 written by the momentum kernel (m x ldn)
    __nv_bfloat16* xhi0;  // bf16 path: X0 = hi + lo written by the momentum kernel
    __nv_bfloat16* xlo0;
    const float* o_src;   // fp32 debug path: final iterate read by the apply kernel
    const __nv_bfloat16* o_hi;   // bf16 path: final iterate = o_hi + o_lo
    const __nv_bfloat16* o_lo;
    int rows, cols;       // of W
    int ldn;              // row stride of the oriented iterate
    int transposed;       // rows > cols: X = U^T
    int g_bf16;           // gradient dtype
    int vec;              // flat 8-wide vector path allowed
    int blk_begin;        // first block of this matrix in the momentum launch (= partial index)
    int blk_count;
    int apply_begin;      // first block in the apply launch
    int apply_count;
    int mat;              // global matrix index (norm / scale arrays)
    float update_scale;   // per-shape scale s of the update
    int out_bf16;         // copy-out only: `w` receives O as bf16 instead of fp32
};

struct alignas(64) GemmMaps {
    CUtensorMap xb_k[2];   // X operand, box {64, 128}: rows of X (K-major operand)
    CUtensorMap xb_mn[2];  // X operand, box {64, 64}: X as an N-contiguous operand
    CUtensorMap a;         // A, box {64, 128}
    CUtensorMap p;         // P, box {64, 128}
    // UPDATE epilogue of the two-CTA kernel: 128 x 32 boxes of the iterate, 64-byte
    // swizzle, loaded into and stored from shared memory (hi in / hi out follow the
    // ping-pong parity; lo in and lo out are the same array in a step)
    CUtensorMap xe_hi[2];
    CUtensorMap xe_lo_in;
    CUtensorMap xe_lo_out;
    // GRAM / POLY epilogue of the two-CTA kernel: A and P, [0] the same 128 x 32 box
    // (64-byte swizzle) for direct stores (and the polynomial's load of A), [1] a
    // 32 x 128 box (no swizzle) for the mirrored stores of tiles off the diagonal
    CUtensorMap se_a[2];
    CUtensorMap se_p[2];
};

struct GemmGroupInfo {
    int m, n, ldm, ldn;
    int count;
    int mat_base;                 // global index of this group's matrix 0
    __nv_bfloat16* xb[2];         // high parts of X (ping-pong; the GEMM operand)
    const __nv_bfloat16* xlo_in;  // UPDATE: low part of X read for the beta term
    __nv_bfloat16* xlo_out;       // UPDATE: low part of X' written (equal to xlo_in in a step)
    __nv_bfloat16* a;             // GRAM output / POLY input
    __nv_bfloat16* p;             // POLY output / UPDATE input (via map)
};

struct GemmParams {
    const int4* tiles;            // (group, matrix, tile_row, tile_col), cost-descending
    int ntiles;
    const GemmMaps* maps;
    const GemmGroupInfo* groups;
    int parity;                   // which xb holds the current iterate
    float alpha, beta;            // GRAM: alpha; POLY: alpha = c, beta = b; UPDATE: alpha = 1, beta = a
    const float* scale;           // per-matrix 1/(||U||+eps) on the first iteration, else nullptr
    int write_op;                 // unused (kept for the layout of the launch parameters)
    int* err;                     // device error word (bounded waits)
    // UPDATE of the last iteration only: 1 = also apply W <- decay*W - lr*s*O,
    // 2 = also copy O out to the caller (orthogonalisation), 0 = neither.
    int apply_mode;
    float decay, lr;
    const EwSeg* segs;            // per-matrix W / output pointer, orientation and scale
    // two-CTA kernel: per-cluster work units (see plan.h), two int4 per unit:
    // (group, matrix, tile_row, tile_col) and (k_begin, k_end, kind, slot | nslots << 16)
    const int4* units;
    const int* unit_begin;        // clusters + 1 offsets
    float* sk_partial;            // partial-sum slots, SK_SLOT_FLOATS each
    int* sk_count;                // per slot: epilogue warps that have stored their part
    int* sk_flag;                 // per slot: epoch of the last complete partial
    int epoch;                    // distinct per launch on a handle
};

// One partial-sum slot: both CTAs' 128 x 256 fp32 accumulator halves.
constexpr int SK_SLOT_FLOATS = 2 * 128 * 256;

// box of the two-CTA UPDATE epilogue: rows x columns (128 x 32 bf16)
int tc_gemm_epi_cols();
int tc_gemm_epi_rows();
int tc_gemm_threads();
// pair = 1: the two-CTA kernel (256 x 256 tiles, grid = 2 x clusters);
// pair = 0: the one-CTA kernel (128 x 256 tiles).
int tc_gemm_tile_m(int pair);
int tc_gemm_tile_n(int pair);
cudaError_t tc_gemm_prepare();    // sets the dynamic shared-memory attribute once per device
cudaError_t tc_gemm_max_clusters(int* n);
// var: shared-memory configuration of the two-CTA kernel (tc_gemm_var), ignored by the
// one-CTA kernel
cudaError_t launch_tc_gemm(int mode, int pair, const GemmParams& p, int grid, cudaStream_t s, int var = 0);
// Configuration of a two-CTA launch of `mode` whose tiles have the average K avg_k.
int tc_gemm_var(int mode, int avg_k);

// Default GEMM variant of new handles and planner queries: the two-CTA kernel unless
// the environment variable MUON_GEMM_PAIR is "0".
int tc_gemm_default_pair();

// fp32 FFMA debug GEMM: C = alpha_eff * A op(B) + beta_eff * Cin, batched over `count`.
// op(B)[k][j] = B[j][k] when b_kmajor, else B[k][j].  With `scale`, alpha_eff =
// alpha * s^scale_pow and beta_eff = beta * s^scale_pow where s = scale[mat_base + z].
struct SimtGemmArgs {
    const float* A; const float* B; float* C; const float* Cin;
    int M, N, K, lda, ldb, ldc, ldcin;
    long long sA, sB, sC, sCin;
    int count, b_kmajor;
    float alpha, beta;
    const float* scale; int scale_pow; int mat_base;
};
cudaError_t launch_simt_gemm(const SimtGemmArgs& a, cudaStream_t s);

// Elementwise kernels.
// Momentum, Nesterov direction, oriented X0 and, per matrix, ||U||_F and
// s = 1/(||U||_F + eps).  counters: one int per matrix, zero between calls.
cudaError_t launch_momentum_norm(const EwSeg* segs, int nseg, int nblocks, double* partials,
                                 float mu, int nesterov, int bf16_operand, int* counters, float eps,
                                 float* norms, float* scale, cudaStream_t s);
cudaError_t launch_apply(const EwSeg* segs, int nseg, int nblocks, float decay, float lr,
                         const float* o_scale, int copy_out, cudaStream_t s);
cudaError_t launch_copy_out_one(const EwSeg& seg, float* dst, const float* o_scale, cudaStream_t s);
// Per matrix: rms[i] = lr * |s_i| * sqrt(sum of O_i^2 / (rows * cols)) over the final
// iterate; `part` holds UPDATE_RMS_PARTIALS doubles per matrix (fixed-order partial sums).
constexpr int UPDATE_RMS_PARTIALS = 256;
cudaError_t launch_update_rms(const EwSeg* segs, int nseg, const float* o_scale, float lr, double* part, float* rms,
                              cudaStream_t s);
// QK-Clip: rows of head h of W_q and W_k (n_heads * head_dim rows, `cols` columns)
// times sqrt(min(1, tau / max_logits[h])).  wk may be nullptr.
cudaError_t launch_qk_clip(float* wq, float* wk, const float* max_logits, int n_heads, int head_dim, int cols,
                           float tau, int num_sms, cudaStream_t s);

// Launch with programmatic stream serialisation (see pdl_wait / pdl_trigger in
// ptx.cuh): the kernel may start while the previous kernel of the stream drains and
// waits on the device before it touches that kernel's data.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

constexpr int EW_THREADS = 256;
constexpr int EW_FLAT_ELEMS = 8192;      // elements per block on the flat path
// transpose tile of the momentum and apply kernels for tall matrices (rows x cols of W)
constexpr int MT_ROWS = 64, MT_COLS = 128;

}  // namespace muon
