// gemm_tc.cu -- the Newton-Schulz GEMMs on the sm_100a tensor cores.
//
// One quintic step X <- aX + b(XX^T)X + c(XX^T)^2 X ("Muon: An optimizer for
// hidden layers in neural networks", section 4, eqs. 4-5) is run as three
// grouped, persistent GEMM launches over every matrix of the step:
//
//   GRAM    A  = alpha * X X^T            (upper-triangle tiles, mirrored)
//   POLY    P  = b*A + c * A A            (A symmetric: A A = A A^T; upper tiles, mirrored)
//   UPDATE  X' = alpha * P X + beta * X   (the aX term in the epilogue; X = hi + lo, the
//                                         bf16 pair, read and written by the epilogue)
//
// On the first step alpha/beta absorb the Frobenius normalisation s = 1/(||U||+eps):
// A0 = s^2 UU^T and X1 = s P U + a s U.
//
// Two kernels:
//
//  ns_gemm_tc_kernel (one CTA per tile, 128 x 256 tiles), 320 threads:
//   warp 0      TMA producer: 4-stage ring of (128x64 A-operand, 256x64 B-operand)
//               bf16 tiles in 128-byte-swizzled shared memory, plain 3-D tiled loads.
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators) and issues
//               tcgen05.mma kind::f16 (M=128, N=256, K=16) from one thread.
//   warps 2-9   epilogue: tcgen05.ld of the accumulator (each warp owns the 32 TMEM
//               lanes its rank allows and half of the columns), scale, residual, and
//               stores through the load/store units.
//
//  ns_gemm_tc2_kernel (a cluster of two CTAs per 256 x 256 tile), 384 threads per CTA:
//   warp 0      TMA producer: each CTA stages its 128 rows of A and its 128 columns of B
//               (a ring of 4 or 5 stages of 16 + 16 KiB); the odd CTA's loads complete
//               on the even CTA's barrier; each load fills one CTA's shared memory.
//   warp 1      the even CTA's elected thread issues tcgen05.mma.cta_group::2 (M=256,
//               N=256, K=16), which reads both CTAs' shared memory; each CTA's TMEM
//               receives its 128 accumulator rows; completion is committed to the
//               barriers of both CTAs by address.
//   warps 2-9   epilogue compute: two column halves of four warps; tcgen05.ld, then
//               the mode's arithmetic on 128 x 32 boxes in shared memory.
//   warps 10-11 epilogue TMA, one per column half: load the boxes the epilogue reads
//               (X = hi + lo for UPDATE, A for POLY) ahead of time and store the
//               finished boxes with bulk tensor stores.
//   Per SM this moves half the B-operand bytes of the one-CTA tile through shared
//   memory, and the epilogue's global traffic leaves the load/store units.
//
// The double-buffered accumulator lets the epilogue of tile i overlap the main
// loop of tile i+1.  Tiles are taken from per-cluster lists built from a cost-sorted
// list that spans all matrices of the call, so many small matrices fill the 148 SMs.
#include "kernels.cuh"
#include "ptx.cuh"

namespace muon {
namespace {

constexpr int BK = TC_BK;
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr int ACC_COLS = 256;                 // one accumulator: 128 lanes x 256 fp32 columns
constexpr int TMEM_COLS = 2 * ACC_COLS;       // two accumulators

// per epilogue warp: a 32 x 32 fp32 chunk for the UPDATE epilogue's re-layout,
// rows padded to 33 words so that both access patterns are free of bank conflicts
constexpr int STAGE_LD = 33;
constexpr int STAGE_FLOATS = 32 * STAGE_LD;
constexpr int STAGE_BYTES = NUM_EPI_WARPS * STAGE_FLOATS * 4;

// one-CTA kernel
constexpr int S1_BM = 128, S1_BN = 256, S1_STAGES = 4;
constexpr int S1_A = S1_BM * BK * 2;          // 16 KiB
constexpr int S1_B = S1_BN * BK * 2;          // 32 KiB
constexpr int S1_SMEM = 1024 + S1_STAGES * (S1_A + S1_B) + 256 + STAGE_BYTES;

// two-CTA kernel (per CTA)
constexpr int S2_BM = 256, S2_BN = 256;
constexpr int S2_A = 128 * BK * 2;            // 16 KiB: this CTA's 128 rows of A
constexpr int S2_B = 128 * BK * 2;            // 16 KiB: this CTA's 128 columns of B

// UPDATE epilogue of the two-CTA kernel: each column half of the CTA's 128 x 256
// accumulator streams the iterate through a ring of EU_DEPTH shared-memory buffers,
// each one 128-row x 32-column box of hi and one of lo (64-byte swizzle).  A TMA warp
// per half (warps 10 and 11) loads the boxes up to EU_DEPTH - 1 chunks ahead, across
// tile boundaries; the half's four compute warps rewrite each chunk in place, and
// the TMA warp stores it once all four have arrived on the chunk's barrier.  The
// operand ring of this mode is S2U_STAGES deep.
#ifndef MUON_EU_DEPTH
#define MUON_EU_DEPTH 3
#endif
#ifndef MUON_S2U_STAGES
#define MUON_S2U_STAGES 4
#endif
// Long K (polynomial from K = 1024, update from K = 2048): a ring of two boxes per
// half and a fifth operand stage.
#ifndef MUON_ES_DEPTH
#define MUON_ES_DEPTH 2
#endif
#ifndef MUON_S2S_STAGES
#define MUON_S2S_STAGES 5
#endif
#ifndef MUON_EU_COLS
#define MUON_EU_COLS 32
#endif
constexpr int EU_COLS = MUON_EU_COLS;               // columns per chunk: one 64- or 128-byte bf16 box row
static_assert(EU_COLS == 32 || EU_COLS == 64, "epilogue chunks are 32 or 64 columns");
constexpr int EU_ROWS = 128;                        // rows per chunk: the CTA's accumulator rows
constexpr int EU_DEPTH = MUON_EU_DEPTH;            // update epilogue ring depth
constexpr int ES_DEPTH = MUON_ES_DEPTH;            // ring depth of the long-K configuration
// Three shared-memory configurations of the two-CTA kernel: VAR 0 (ring depth EU_DEPTH,
// S2U_STAGES operand stages) for short K, VAR 1 (ES_DEPTH, S2S_STAGES) for long K and
// VAR 2 (one epilogue buffer per half, S2L_STAGES operand stages) for the longest K,
// where a tile's main loop leaves the epilogue enough time to run one chunk at a time.
// Each launch takes the one tc_gemm_var picks from the plan's K.
#ifndef MUON_S2L_STAGES
#define MUON_S2L_STAGES 6
#endif
constexpr int S2L_STAGES = MUON_S2L_STAGES;
__host__ __device__ constexpr int eu_depth(int var) { return var == 2 ? 1 : var ? ES_DEPTH : EU_DEPTH; }
constexpr int EU_ROW_BYTES = EU_COLS * 2;
constexpr int EU_BOX = EU_ROWS * EU_ROW_BYTES;      // 8 KiB
constexpr int EU_BUF = 2 * EU_BOX;                  // hi + lo
constexpr int S2U_STAGES = MUON_S2U_STAGES;
constexpr int S2S_STAGES = MUON_S2S_STAGES;
constexpr int NUM_THREADS_U = NUM_THREADS + 64;     // + the two epilogue TMA warps
static_assert(EU_DEPTH >= 2 && EU_DEPTH <= 6 && ES_DEPTH >= 2 && ES_DEPTH <= 6, "epilogue ring depth out of range");

// Every mode of the two-CTA kernel uses the TMA epilogue (the Gram and polynomial
// products store their symmetric output through the same ring of boxes).
constexpr int s2_stages(int var) { return var == 2 ? S2L_STAGES : var ? S2S_STAGES : S2U_STAGES; }
constexpr int s2_epi_bytes(int var) { return 2 * eu_depth(var) * EU_BUF; }
constexpr int s2_threads(int) { return NUM_THREADS_U; }
// barriers: full / empty per stage, two tfull / tempty, drain, the epilogue ring's
// (UPDATE), then the TMEM address and the abort flag
constexpr int s2_bar_bytes(int var) {
    // (+ the epilogue TMA warps' chunk coordinates, 2 x ring depth int4)
    return (8 * (2 * s2_stages(var) + 5 + 4 * eu_depth(var)) + 8 + 16 + 2 * eu_depth(var) * 16 + 127) / 128 * 128;
}
// [operand ring][epilogue buffers][barriers]; the ring and the buffers are 1024-byte aligned
constexpr int s2_smem(int var) {
    return 1024 + s2_stages(var) * (S2_A + S2_B) + s2_epi_bytes(var) + s2_bar_bytes(var);
}
constexpr int S2_SMEM = s2_smem(1);
constexpr int S2U_SMEM = s2_smem(0);
constexpr int S2L_SMEM = s2_smem(2);
static_assert(S1_SMEM <= 232448 && S2_SMEM <= 232448 && S2U_SMEM <= 232448 && S2L_SMEM <= 232448,
              "dynamic shared memory above the 227 KiB limit");
static_assert((s2_stages(0) * (S2_A + S2_B)) % 1024 == 0 && (s2_stages(1) * (S2_A + S2_B)) % 1024 == 0 &&
              EU_BUF % 1024 == 0, "buffer alignment");

// error codes written to the device error word when a bounded wait gives up
constexpr int ERR_PRODUCER = 0x101, ERR_MMA_SLOT = 0x102, ERR_MMA_ACC = 0x103, ERR_EPILOGUE = 0x104,
              ERR_TAIL = 0x105, ERR_SPLIT = 0x106;

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

// Bounded wait until *flag == value (a partial sum published by another cluster).
__device__ __forceinline__ bool flag_wait(const int* flag, int value, volatile int* abort_flag, int* err, int code) {
    if (ld_acquire_gpu(flag) == value) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        __nanosleep(64);
        if (ld_acquire_gpu(flag) == value) return true;
        if (*abort_flag) return false;
        if (globaltimer_ns() - t0 > MUON_WAIT_NS) {
            atomicCAS(err, 0, code);
            *abort_flag = 1;
            return false;
        }
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_bits_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_bits_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Update of the weight (apply_mode 1: W <- decay*W - lr*s*O, eq. 3 with decoupled
// decay and the per-shape scale) or copy-out of O (apply_mode 2) for the 32
// finished values O[row][col0..col0+31] of the oriented result.  A matrix that was
// transposed for the smaller Gram gets W[c][row]: lanes hold consecutive rows, so
// each store instruction of the warp covers 32 consecutive elements of W's row c.
__device__ __forceinline__ void apply_chunk(const GemmParams& p, const GemmGroupInfo& gi, int mat, int row,
                                            int col0, const float (&val)[32]) {
    const EwSeg& sg = p.segs[gi.mat_base + mat];
    float* w = sg.w;
    const float step = p.lr * sg.update_scale;
    const bool copy = p.apply_mode == 2;
    if (copy && sg.out_bf16) {
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(sg.w);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int c = col0 + j;
            if (c < gi.n) o[sg.transposed ? (size_t)c * sg.cols + row : (size_t)row * sg.cols + c] = __float2bfloat16_rn(val[j]);
        }
        return;
    }
    if (!sg.transposed) {
        float* wr = w + (size_t)row * sg.cols;
        if (sg.vec && col0 + 31 < gi.n) {
            float4* w4 = reinterpret_cast<float4*>(wr + col0);
#pragma unroll
            for (int qq = 0; qq < 8; ++qq) {
                float4 o = make_float4(val[4 * qq], val[4 * qq + 1], val[4 * qq + 2], val[4 * qq + 3]);
                if (!copy) {
                    const float4 x = w4[qq];
                    o.x = fmaf(-step, o.x, p.decay * x.x);
                    o.y = fmaf(-step, o.y, p.decay * x.y);
                    o.z = fmaf(-step, o.z, p.decay * x.z);
                    o.w = fmaf(-step, o.w, p.decay * x.w);
                }
                w4[qq] = o;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int c = col0 + j;
                if (c < gi.n) wr[c] = copy ? val[j] : fmaf(-step, val[j], p.decay * wr[c]);
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int c = col0 + j;
            if (c < gi.n) {
                float* wp = w + (size_t)c * sg.cols + row;
                *wp = copy ? val[j] : fmaf(-step, val[j], p.decay * *wp);
            }
        }
    }
}

// UPDATE epilogue operands of one thread, pulled into L2 while the tile's MMAs run:
// the thread's `ncols` columns from `col_start` of its row of X = hi + lo and, when
// the weight update is fused (apply_mode 1), the matching elements of W.  Every
// range stays inside its buffer: X rows end at ldn (a multiple of 8 elements),
// W is touched only inside its rows x cols.
__device__ __forceinline__ void prefetch_update_operands(const GemmParams& p, const GemmGroupInfo& gi, int mat,
                                                         int row, int col_start, int ncols) {
    if (row >= gi.m || col_start >= gi.n) return;
    const int nc = min(ncols, gi.ldn - col_start);
    const size_t off = (size_t)mat * gi.m * gi.ldn + (size_t)row * gi.ldn + col_start;
    prefetch_l2_bulk(gi.xb[p.parity] + off, (uint32_t)nc * 2u);
    prefetch_l2_bulk(gi.xlo_in + off, (uint32_t)nc * 2u);
    if (p.apply_mode != 1) return;
    const EwSeg& sg = p.segs[gi.mat_base + mat];
    const int ncw = min(ncols, gi.n - col_start);
    if (!sg.transposed) {
        const float* wr = sg.w + (size_t)row * sg.cols + col_start;
        if (sg.vec) {
            prefetch_l2_bulk(wr, (uint32_t)ncw * 4u);
        } else {
            for (int c = 0; c < ncw; c += 32) prefetch_l2_line(wr + c);
        }
    } else {
        // W[c][row]: the warp's 32 consecutive rows are one 128-byte run of W's row c;
        // lane l takes W rows col_start + l, col_start + l + 32, ...
        const int lane = (int)(threadIdx.x & 31u);
        const int row0 = row - lane;
        for (int c = lane; c < ncw; c += 32) prefetch_l2_line(sg.w + (size_t)(col_start + c) * sg.cols + row0);
    }
}

// Weight update (apply_mode 1) or copy-out (apply_mode 2) of 8 finished values
// O[r][c..c+7] of a matrix that was not transposed (W has the layout of O).
__device__ __forceinline__ void apply_run8(const GemmParams& p, const EwSeg& sg, int n, int r, int c,
                                           const float (&val)[8]) {
    float* wr = sg.w + (size_t)r * sg.cols + c;
    const float step = p.lr * sg.update_scale;
    const bool copy = p.apply_mode == 2;
    if (copy && sg.out_bf16) {
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(sg.w) + (size_t)r * sg.cols + c;
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (c + k < n) o[k] = __float2bfloat16_rn(val[k]);
        return;
    }
    if (sg.vec && c + 7 < n) {
        float4* w4 = reinterpret_cast<float4*>(wr);
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
            float4 o = make_float4(val[4 * qq], val[4 * qq + 1], val[4 * qq + 2], val[4 * qq + 3]);
            if (!copy) {
                const float4 x = w4[qq];
                o.x = fmaf(-step, o.x, p.decay * x.x);
                o.y = fmaf(-step, o.y, p.decay * x.y);
                o.z = fmaf(-step, o.z, p.decay * x.z);
                o.w = fmaf(-step, o.w, p.decay * x.w);
            }
            w4[qq] = o;
        }
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (c + k < n) wr[k] = copy ? val[k] : fmaf(-step, val[k], p.decay * wr[k]);
    }
}

// Writes the warp's accumulator chunk (one row per lane, as tcgen05.ld 32x32b
// delivers it) into its shared buffer.
__device__ __forceinline__ void stage_chunk(const uint32_t (&v)[32], float* stage) {
    const int lane = (int)(threadIdx.x & 31u);
    __syncwarp();                                   // the previous chunk's reads are done
#pragma unroll
    for (int j = 0; j < 32; ++j) stage[lane * STAGE_LD + j] = __uint_as_float(v[j]);
    __syncwarp();
}

// UPDATE epilogue of one 32 x 32 chunk: X' = alpha * acc + beta * (hi + lo), stored
// as the pair hi' = bf16(X'), lo' = bf16(X' - hi').  The accumulator arrives one row
// per lane (tcgen05.ld 32x32b); it goes through the warp's shared buffer so that lane
// l works on rows l/4 + 8i (i = 0..3), columns 8(l%4) .. 8(l%4)+7 of the chunk.  Each
// 16-byte access of the warp then covers 8 rows x 64 contiguous bytes, a quarter of
// the cache lines that the row-per-lane layout touches.  hw / lw: this lane's hi and
// lo words in that layout, loaded by the caller (valid where the 8 columns are inside
// the matrix).
__device__ __forceinline__ void update_chunk(const GemmParams& p, const GemmGroupInfo& gi, int mat, int row,
                                             int col0, float alpha, float beta, const uint32_t (&v)[32],
                                             const uint4 (&hw)[4], const uint4 (&lw)[4], float* stage) {
    const int lane = (int)(threadIdx.x & 31u);
    const int row_w = row - lane;
    const int lr = lane >> 2, lc = (lane & 3) * 8;
    stage_chunk(v, stage);
    const EwSeg* sg = p.apply_mode != 0 ? &p.segs[gi.mat_base + mat] : nullptr;
    const bool apply_t = sg != nullptr && sg->transposed;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = row_w + lr + 8 * i, c = col0 + lc;
        float* slot = stage + (lr + 8 * i) * STAGE_LD + lc;     // this lane's 8 words of row lr + 8i
        float acc8[8], res[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            acc8[k] = slot[k];
            res[k] = 0.f;
        }
        if (r < gi.m) {
            const size_t o = (size_t)mat * gi.m * gi.ldn + (size_t)r * gi.ldn + c;
            __nv_bfloat16* hout = gi.xb[p.parity ^ 1] + o;
            __nv_bfloat16* lout = gi.xlo_out + o;
            if (c + 7 < gi.n) {
                const uint32_t h4[4] = {hw[i].x, hw[i].y, hw[i].z, hw[i].w};
                const uint32_t l4[4] = {lw[i].x, lw[i].y, lw[i].z, lw[i].w};
                uint32_t ho[4], lo[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float x0 = bf16_bits_lo(h4[e]) + bf16_bits_lo(l4[e]);
                    const float x1 = bf16_bits_hi(h4[e]) + bf16_bits_hi(l4[e]);
                    const float y0 = alpha * acc8[2 * e] + beta * x0;
                    const float y1 = alpha * acc8[2 * e + 1] + beta * x1;
                    const __nv_bfloat162 hh = __floats2bfloat162_rn(y0, y1);
                    const float2 hf = __bfloat1622float2(hh);
                    const __nv_bfloat162 ll = __floats2bfloat162_rn(y0 - hf.x, y1 - hf.y);
                    ho[e] = *reinterpret_cast<const uint32_t*>(&hh);
                    lo[e] = *reinterpret_cast<const uint32_t*>(&ll);
                }
                *reinterpret_cast<uint4*>(hout) = make_uint4(ho[0], ho[1], ho[2], ho[3]);
                *reinterpret_cast<uint4*>(lout) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                if (sg != nullptr) {
                    // the stored pair is the result: the weight update uses exactly it
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        res[2 * e] = bf16_bits_lo(ho[e]) + bf16_bits_lo(lo[e]);
                        res[2 * e + 1] = bf16_bits_hi(ho[e]) + bf16_bits_hi(lo[e]);
                    }
                }
            } else {
                const __nv_bfloat16* hin = gi.xb[p.parity] + o;
                const __nv_bfloat16* lin = gi.xlo_in + o;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (c + k >= gi.n) continue;
                    const float y = alpha * acc8[k] + beta * (__bfloat162float(hin[k]) + __bfloat162float(lin[k]));
                    const __nv_bfloat16 hh = __float2bfloat16_rn(y);
                    const __nv_bfloat16 ll = __float2bfloat16_rn(y - __bfloat162float(hh));
                    hout[k] = hh;
                    lout[k] = ll;
                    res[k] = __bfloat162float(hh) + __bfloat162float(ll);
                }
            }
            if (sg != nullptr && !apply_t) apply_run8(p, *sg, gi.n, r, c, res);
        }
        // a transposed matrix's W update goes back through this lane's own words of
        // the buffer (no other lane reads or writes them in between)
        if (apply_t) {
#pragma unroll
            for (int k = 0; k < 8; ++k) slot[k] = res[k];
        }
    }
    if (apply_t) {
        // W[c][r]: back to one row per lane, where the warp's lanes are 32
        // consecutive elements of one row of W
        __syncwarp();
        float val[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) val[j] = stage[lane * STAGE_LD + j];
        if (row < gi.m) apply_chunk(p, gi, mat, row, col0, val);
    }
}

// GRAM / POLY epilogue of one 32 x 32 chunk of a symmetric m x m output (only
// tiles with tile column >= tile row run): y = alpha * acc, plus beta * A for the
// polynomial.  Element (r, c) is stored at (r, c) when c >= r and mirrored to
// (c, r) when c > r, so every element of the output is written exactly once.  The
// chunk goes through the warp's shared buffer: the direct stores use the layout of
// update_chunk (lane l: rows l/4 + 8i, 8 columns from 8(l%4)), the mirrored ones its
// transpose (lane l: output row col0 + l/4 + 8i, 8 columns from row_w + 8(l%4)), so
// each 16-byte store instruction of the warp covers 8 rows x 64 contiguous bytes.
// aw: this lane's words of A in the first layout (polynomial only; valid where the 8
// columns are inside the matrix).
template <int MODE>
__device__ __forceinline__ void sym_chunk(__nv_bfloat16* __restrict__ out, const __nv_bfloat16* A, int m, int ldm,
                                          int row, int col0, float alpha, float beta, const uint32_t (&v)[32],
                                          const uint4 (&aw)[4], float* stage) {
    const int lane = (int)(threadIdx.x & 31u);
    const int row_w = row - lane, lr = lane >> 2, lc = (lane & 3) * 8;
    if (col0 + 31 < row_w) return;              // every element below the diagonal: nothing to store
    stage_chunk(v, stage);
    const bool above = col0 >= row_w + 32;      // every element has c > r
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = row_w + lr + 8 * i, c = col0 + lc;
        float* slot = stage + (lr + 8 * i) * STAGE_LD + lc;
        float y[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) y[k] = alpha * slot[k];
        if (MODE == MODE_POLY) {
            if (r < m && c + 7 < m) {
                const uint32_t w4[4] = {aw[i].x, aw[i].y, aw[i].z, aw[i].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    y[2 * e] += beta * bf16_bits_lo(w4[e]);
                    y[2 * e + 1] += beta * bf16_bits_hi(w4[e]);
                }
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (r < m && c + k < m) y[k] += beta * __bfloat162float(A[(size_t)r * ldm + c + k]);
            }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) slot[k] = y[k];
        if (r >= m) continue;
        if (above && c + 7 < m) {
            *reinterpret_cast<uint4*>(out + (size_t)r * ldm + c) =
                make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                           pack_bf16x2(y[6], y[7]));
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (c + k >= r && c + k < m) out[(size_t)r * ldm + c + k] = __float2bfloat16_rn(y[k]);
        }
    }
    __syncwarp();                               // every lane's values are in the buffer
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int cc = col0 + lr + 8 * i, rr = row_w + lc;   // output row cc holds column cc's mirror
        if (cc >= m) continue;
        float y[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) y[k] = stage[(lc + k) * STAGE_LD + lr + 8 * i];
        if (above && rr + 7 < m) {
            *reinterpret_cast<uint4*>(out + (size_t)cc * ldm + rr) =
                make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]), pack_bf16x2(y[4], y[5]),
                           pack_bf16x2(y[6], y[7]));
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k)
                if (cc > rr + k && rr + k < m) out[(size_t)cc * ldm + rr + k] = __float2bfloat16_rn(y[k]);
        }
    }
}

// Epilogue of one accumulator row segment: 4 chunks of 32 columns starting at
// column `c_begin` of the accumulator whose TMEM address (lane quarter included)
// is `tacc`.  `row` is the global output row of this thread, `col_base` the
// global column of accumulator column 0.
//
// Split tiles (two-CTA kernel): kind 2 stores the raw fp32 accumulator row to its
// partial-sum slot at `sk_row` and does nothing else; kind 1 adds the `nslots`
// partial rows at sk_row, sk_row + SK_SLOT_FLOATS, ... (in K order) before the
// usual epilogue; kind 0 is a whole tile.
template <int MODE>
__device__ __forceinline__ void epilogue_segment(const GemmParams& p, const GemmGroupInfo& gi, int mat, int row,
                                                 int col_base, uint32_t tacc, int c_begin, float* stage,
                                                 int kind = 0, float* sk_row = nullptr, int nslots = 0,
                                                 int nchunks = 4) {
    float alpha = p.alpha, beta = p.beta;
    if (p.scale != nullptr) {
        const float s = p.scale[gi.mat_base + mat];
        if (MODE == MODE_GRAM) alpha = p.alpha * s * s;
        if (MODE == MODE_UPDATE) { alpha = p.alpha * s; beta = p.beta * s; }
    }
#pragma unroll 1
    for (int chunk = 0; chunk < nchunks; ++chunk) {
        const int c_local = c_begin + chunk * 32;
        const int col0 = col_base + c_local;
        // UPDATE works in the coalesced layout (see update_chunk); the iterate's loads
        // go out before the accumulator read so that their latency overlaps it.
        const int lane = (int)(threadIdx.x & 31u);
        const int row_w = row - lane;                  // first row of this warp's slice
        const int lr = lane >> 2, lc = (lane & 3) * 8;
        uint4 hw[4], lw[4];
        if (MODE == MODE_POLY && kind != 2) {
            // the polynomial's b A term, in the same layout
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = row_w + lr + 8 * i, c = col0 + lc;
                if (r < gi.m && c + 7 < gi.m)
                    hw[i] = *reinterpret_cast<const uint4*>(gi.a + (size_t)mat * gi.m * gi.ldm + (size_t)r * gi.ldm + c);
            }
        }
        if (MODE == MODE_UPDATE && kind != 2) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = row_w + lr + 8 * i, c = col0 + lc;
                if (r < gi.m && c + 7 < gi.n) {
                    const size_t o = (size_t)mat * gi.m * gi.ldn + (size_t)r * gi.ldn + c;
                    hw[i] = *reinterpret_cast<const uint4*>(gi.xb[p.parity] + o);
                    lw[i] = *reinterpret_cast<const uint4*>(gi.xlo_in + o);
                }
            }
        }
        uint32_t v[32];
        tmem_ld_32x32b_x32(tacc + (uint32_t)c_local, v);
        tmem_ld_wait();
        if (kind == 2) {
            float4* dst = reinterpret_cast<float4*>(sk_row + c_local);
#pragma unroll
            for (int qq = 0; qq < 8; ++qq)
                dst[qq] = make_float4(__uint_as_float(v[4 * qq]), __uint_as_float(v[4 * qq + 1]),
                                      __uint_as_float(v[4 * qq + 2]), __uint_as_float(v[4 * qq + 3]));
            continue;
        }
        if (kind == 1) {
            for (int sl = 0; sl < nslots; ++sl) {
                const float4* src = reinterpret_cast<const float4*>(sk_row + (size_t)sl * SK_SLOT_FLOATS + c_local);
#pragma unroll
                for (int qq = 0; qq < 8; ++qq) {
                    const float4 x = __ldcg(src + qq);
                    v[4 * qq + 0] = __float_as_uint(__uint_as_float(v[4 * qq + 0]) + x.x);
                    v[4 * qq + 1] = __float_as_uint(__uint_as_float(v[4 * qq + 1]) + x.y);
                    v[4 * qq + 2] = __float_as_uint(__uint_as_float(v[4 * qq + 2]) + x.z);
                    v[4 * qq + 3] = __float_as_uint(__uint_as_float(v[4 * qq + 3]) + x.w);
                }
            }
        }
        if (MODE == MODE_GRAM) {
            sym_chunk<MODE_GRAM>(gi.a + (size_t)mat * gi.m * gi.ldm, nullptr, gi.m, gi.ldm, row, col0, alpha, beta,
                                 v, hw, stage);
        } else if (MODE == MODE_POLY) {
            sym_chunk<MODE_POLY>(gi.p + (size_t)mat * gi.m * gi.ldm, gi.a + (size_t)mat * gi.m * gi.ldm, gi.m, gi.ldm,
                                 row, col0, alpha, beta, v, hw, stage);
        } else {
            update_chunk(p, gi, mat, row, col0, alpha, beta, v, hw, lw, stage);
        }
    }
}

template <int MODE>
__device__ __forceinline__ void operand_maps(const GemmParams& p, int g, const void*& mapA, const void*& mapB) {
    const GemmMaps* mp = p.maps + g;
    mapA = (MODE == MODE_GRAM) ? (const void*)&mp->xb_k[p.parity]
         : (MODE == MODE_POLY) ? (const void*)&mp->a : (const void*)&mp->p;
    mapB = (MODE == MODE_GRAM) ? (const void*)&mp->xb_k[p.parity]
         : (MODE == MODE_POLY) ? (const void*)&mp->a : (const void*)&mp->xb_mn[p.parity];
}

__device__ __forceinline__ void spin_ns(uint64_t ns) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < ns) { }
}

// Weight update (apply_mode 1) or copy-out (apply_mode 2) of NC finished values
// O[row][col0 .. col0 + NC) of the oriented result, one row per lane.  A matrix that
// was transposed for the smaller Gram gets W[c][row]: lanes hold consecutive rows,
// so each store instruction of the warp covers 32 consecutive elements of W's row c.
template <int NC>
__device__ __forceinline__ void apply_row(const GemmParams& p, const GemmGroupInfo& gi, const EwSeg& sg, int row,
                                          int col0, const uint32_t (&bits)[NC]) {
    float val[NC];
#pragma unroll
    for (int j = 0; j < NC; ++j) val[j] = __uint_as_float(bits[j]);
    float* w = sg.w;
    const float step = p.lr * sg.update_scale;
    const bool copy = p.apply_mode == 2;
    if (copy && sg.out_bf16) {
        __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(sg.w);
        if (!sg.transposed) {
            __nv_bfloat16* orow = o + (size_t)row * sg.cols;
            if (sg.vec && col0 + NC - 1 < gi.n) {
#pragma unroll
                for (int qq = 0; qq < NC / 8; ++qq)
                    *reinterpret_cast<uint4*>(orow + col0 + 8 * qq) =
                        make_uint4(pack_bf16x2(val[8 * qq], val[8 * qq + 1]), pack_bf16x2(val[8 * qq + 2], val[8 * qq + 3]),
                                   pack_bf16x2(val[8 * qq + 4], val[8 * qq + 5]), pack_bf16x2(val[8 * qq + 6], val[8 * qq + 7]));
            } else {
#pragma unroll
                for (int j = 0; j < NC; ++j)
                    if (col0 + j < gi.n) orow[col0 + j] = __float2bfloat16_rn(val[j]);
            }
        } else {
#pragma unroll
            for (int j = 0; j < NC; ++j)
                if (col0 + j < gi.n) o[(size_t)(col0 + j) * sg.cols + row] = __float2bfloat16_rn(val[j]);
        }
        return;
    }
    // every load of W is issued before the first store: with the stores in between,
    // the compiler cannot tell that the addresses differ and waits out each load
    if (!sg.transposed) {
        float* wr = w + (size_t)row * sg.cols;
        if (sg.vec && col0 + NC - 1 < gi.n) {
            float4* w4 = reinterpret_cast<float4*>(wr + col0);
            float4 x[NC / 4];
            if (!copy) {
#pragma unroll
                for (int qq = 0; qq < NC / 4; ++qq) x[qq] = __ldcg(w4 + qq);
            }
#pragma unroll
            for (int qq = 0; qq < NC / 4; ++qq) {
                float4 o = make_float4(val[4 * qq], val[4 * qq + 1], val[4 * qq + 2], val[4 * qq + 3]);
                if (!copy) {
                    o.x = fmaf(-step, o.x, p.decay * x[qq].x);
                    o.y = fmaf(-step, o.y, p.decay * x[qq].y);
                    o.z = fmaf(-step, o.z, p.decay * x[qq].z);
                    o.w = fmaf(-step, o.w, p.decay * x[qq].w);
                }
                w4[qq] = o;
            }
        } else {
            float x[NC];
#pragma unroll
            for (int j = 0; j < NC; ++j) x[j] = (!copy && col0 + j < gi.n) ? __ldcg(wr + col0 + j) : 0.f;
#pragma unroll
            for (int j = 0; j < NC; ++j)
                if (col0 + j < gi.n) wr[col0 + j] = copy ? val[j] : fmaf(-step, val[j], p.decay * x[j]);
        }
    } else {
        // W[c][row]: lanes hold consecutive rows, so each access of the warp is coalesced
        float x[NC];
#pragma unroll
        for (int j = 0; j < NC; ++j)
            x[j] = (!copy && col0 + j < gi.n) ? __ldcg(w + (size_t)(col0 + j) * sg.cols + row) : 0.f;
#pragma unroll
        for (int j = 0; j < NC; ++j)
            if (col0 + j < gi.n)
                w[(size_t)(col0 + j) * sg.cols + row] = copy ? val[j] : fmaf(-step, val[j], p.decay * x[j]);
    }
}

// Where chunk c of a unit lies for one column half of the two-CTA UPDATE epilogue:
// the CTA's 128 accumulator rows and EU_COLS columns of the half.  A chunk is a
// "load chunk" when it needs the iterate (its unit is not a split part that only
// stores a partial sum) and touches the matrix (gm x gn, the group's oriented shape).
struct EuChunk {
    int g, mat, row0, col0, tcol;   // group, matrix, first row / column, TMEM column
    bool load;
};

__device__ __forceinline__ int eu_nchunks(int4 sk) {
    return (sk.z & 0xFF) == 2 ? 0 : ((sk.z >> 8) ? 64 : 128) / EU_COLS;
}

__device__ __forceinline__ EuChunk eu_chunk(int4 tile, int4 sk, int gm, int gn, int c, int rank, int half) {
    const int nh = sk.z >> 8;
    EuChunk ch;
    ch.g = tile.x;
    ch.mat = tile.y;
    ch.row0 = tile.z * S2_BM + rank * 128;
    ch.tcol = half * (nh ? 64 : 128) + c * EU_COLS;
    ch.col0 = tile.w * S2_BN + (nh ? (nh - 1) * 128 : 0) + ch.tcol;
    ch.load = (sk.z & 0xFF) != 2 && ch.row0 < gm && ch.col0 < gn;
    return ch;
}

// Byte offset of 16-byte slot k of row r inside a box with EU_ROW_BYTES-byte rows and
// the swizzle of that span (64B: slot ^= (r >> 1) & 3; 128B: slot ^= r & 7): the 8
// lanes of a quarter-warp access read 8 distinct 16-byte bank groups, so the
// row-per-lane accesses are conflict free.
__device__ __forceinline__ uint32_t eu_off(int r, int k) {
    if (EU_ROW_BYTES == 64) return (uint32_t)(r * EU_ROW_BYTES + ((k ^ ((r >> 1) & 3)) << 4));
    return (uint32_t)(r * EU_ROW_BYTES + ((k ^ (r & 7)) << 4));
}

// X' = alpha * acc + beta * (hi + lo) for this lane's row of one chunk, in place in
// the swizzled hi / lo boxes at hi_s / lo_s; with APPLY, v[] is overwritten with the
// values of the stored pair, hi' + lo' (fp32 bits), for the weight update.
template <bool APPLY>
__device__ __forceinline__ void eu_compute(uint32_t hi_s, uint32_t lo_s, int lane, float alpha, float beta,
                                           uint32_t (&v)[32], int kbase = 0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t off = eu_off(lane, kbase + k);
        const uint4 hv = lds128(hi_s + off), lv = lds128(lo_s + off);
        const uint32_t h4[4] = {hv.x, hv.y, hv.z, hv.w};
        const uint32_t l4[4] = {lv.x, lv.y, lv.z, lv.w};
        uint32_t ho[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float x0 = bf16_bits_lo(h4[e]) + bf16_bits_lo(l4[e]);
            const float x1 = bf16_bits_hi(h4[e]) + bf16_bits_hi(l4[e]);
            const float y0 = alpha * __uint_as_float(v[8 * k + 2 * e]) + beta * x0;
            const float y1 = alpha * __uint_as_float(v[8 * k + 2 * e + 1]) + beta * x1;
            const __nv_bfloat162 hh = __floats2bfloat162_rn(y0, y1);
            const float2 hf = __bfloat1622float2(hh);
            const __nv_bfloat162 ll = __floats2bfloat162_rn(y0 - hf.x, y1 - hf.y);
            ho[e] = *reinterpret_cast<const uint32_t*>(&hh);
            lo[e] = *reinterpret_cast<const uint32_t*>(&ll);
            if (APPLY) {
                // the stored pair is the result: the weight update uses exactly it
                v[8 * k + 2 * e] = __float_as_uint(bf16_bits_lo(ho[e]) + bf16_bits_lo(lo[e]));
                v[8 * k + 2 * e + 1] = __float_as_uint(bf16_bits_hi(ho[e]) + bf16_bits_hi(lo[e]));
            }
        }
        sts128(hi_s + off, make_uint4(ho[0], ho[1], ho[2], ho[3]));
        sts128(lo_s + off, make_uint4(lo[0], lo[1], lo[2], lo[3]));
    }
}


// ============================================================================ one-CTA kernel

template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1) ns_gemm_tc_kernel(const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + S1_STAGES * S1_A;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S1_STAGES * (S1_A + S1_B));
    uint64_t* empty = full + S1_STAGES;
    uint64_t* tfull = empty + S1_STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const uint32_t warp = warp_id();
    const uint32_t lane = threadIdx.x & 31u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S1_STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], NUM_EPI_WARPS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_trigger();
    pdl_wait();             // operands and outputs belong to the previous kernels

    if (warp == 0) {
        if (elect_one()) {
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x) {
                const int4 tile = p.tiles[t];
                const GemmGroupInfo& gi = p.groups[tile.x];
                const int K = (MODE == MODE_GRAM) ? gi.n : gi.m;
                const int kblocks = (K + BK - 1) / BK;
                const void *mapA, *mapB;
                operand_maps<MODE>(p, tile.x, mapA, mapB);
                const int row0 = tile.z * S1_BM, col0 = tile.w * S1_BN, mat = tile.y;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, ERR_PRODUCER)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[stage], S1_A + S1_B);
                    const int k0 = kb * BK;
                    uint8_t* a_dst = sA + stage * S1_A;
                    uint8_t* b_dst = sB + stage * S1_B;
                    tma_load_3d(a_dst, mapA, &full[stage], k0, row0, mat);
                    if (MODE == MODE_UPDATE) {
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            tma_load_3d(b_dst + c * (BK * 128), mapB, &full[stage], col0 + 64 * c, k0, mat);
                    } else {
                        tma_load_3d(b_dst, mapB, &full[stage], k0, col0, mat);
                        tma_load_3d(b_dst + 128 * 128, mapB, &full[stage], k0, col0 + 128, mat);
                    }
                    if (++stage == S1_STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            // tail: every slot released once more, so no MMA completion is still
            // on its way to this CTA's barriers when it retires
            for (int i = 0; i < S1_STAGES && ok; ++i) {
                if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, ERR_TAIL)) ok = false;
                if (++stage == S1_STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok || *abort_flag) spin_ns(2000000ull);   // let loads in flight land
        }
    } else if (warp == 1) {
        if (elect_one()) {
            constexpr uint32_t idesc = idesc_bf16_f32(S1_BM, S1_BN, MODE == MODE_UPDATE ? 1u : 0u);
            uint32_t stage = 0, phase = 0;
            int local = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x, ++local) {
                const int4 tile = p.tiles[t];
                const GemmGroupInfo& gi = p.groups[tile.x];
                const int K = (MODE == MODE_GRAM) ? gi.n : gi.m;
                const int kblocks = (K + BK - 1) / BK;
                const uint32_t acc = local & 1;
                const uint32_t acc_phase = (local >> 1) & 1;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, p.err, ERR_MMA_ACC)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag, p.err, ERR_MMA_SLOT)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA + stage * S1_A);
                    const uint32_t b_base = smem_u32(sB + stage * S1_B);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // K-major 128B-swizzled: rows 128 B apart, 8-row groups 1024 B apart;
                        // a 16-element K step is a 32-byte move inside the swizzle atom.
                        const uint64_t adesc = smem_desc_sw128(a_base + kk * 32, 16, 1024);
                        uint64_t bdesc;
                        if (MODE == MODE_UPDATE) {
                            // N-contiguous 128B-swizzled: 64-column chunks 8 KiB apart (LBO),
                            // 8-row K groups 1024 B apart (SBO); 16 K rows = 2048 B.
                            bdesc = smem_desc_sw128(b_base + kk * 2048, BK * 128, 1024);
                        } else {
                            bdesc = smem_desc_sw128(b_base + kk * 32, 16, 1024);
                        }
                        tc_mma_f16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    tc_commit(&empty[stage]);
                    if (++stage == S1_STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&tfull[acc]);
            }
            if (!ok || *abort_flag) {
                tc_commit(drain);
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < 100000000ull) { }
            }
        }
    } else {
        const uint32_t q = warp & 3u;
        const uint32_t half = (warp - 2) >> 2;
        float* stage = reinterpret_cast<float*>(smem + S1_STAGES * (S1_A + S1_B) + 256) + (warp - 2) * STAGE_FLOATS;
        int local = 0;
        for (int t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++local) {
            const int4 tile = p.tiles[t];
            const GemmGroupInfo& gi = p.groups[tile.x];
            const uint32_t acc = local & 1;
            const uint32_t acc_phase = (local >> 1) & 1;
            const int row = tile.z * S1_BM + (int)(q * 32 + lane);
            if (MODE == MODE_UPDATE)
                prefetch_update_operands(p, gi, tile.y, row, tile.w * S1_BN + (int)half * 128, 128);
            bool ok = mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err, ERR_EPILOGUE);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
            epilogue_segment<MODE>(p, gi, tile.y, row, tile.w * S1_BN,
                                   tmem_base + acc * ACC_COLS + ((q * 32u) << 16), (int)half * 128, stage);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ============================================================================ two-CTA UPDATE epilogue

// L2 prefetch of the weight elements that the fused apply of this thread's row will
// read and write (apply_mode 1 only); the iterate itself arrives by TMA.
__device__ __forceinline__ void prefetch_w_row(const GemmParams& p, const GemmGroupInfo& gi, int mat, int row,
                                               int col_start, int ncols) {
    if (p.apply_mode != 1 || row >= gi.m || col_start >= gi.n) return;
    const EwSeg& sg = p.segs[gi.mat_base + mat];
    const int ncw = min(ncols, gi.n - col_start);
    if (!sg.transposed) {
        const float* wr = sg.w + (size_t)row * sg.cols + col_start;
        if (sg.vec) prefetch_l2_bulk(wr, (uint32_t)ncw * 4u);
        else for (int c = 0; c < ncw; c += 32) prefetch_l2_line(wr + c);
    } else {
        const int lane = (int)(threadIdx.x & 31u);
        const int row0 = row - lane;
        for (int c = lane; c < ncw; c += 32) prefetch_l2_line(sg.w + (size_t)(col_start + c) * sg.cols + row0);
    }
}

// GRAM / POLY epilogue of this lane's row (brow, 0..127 in the chunk's boxes) of one
// chunk: y = alpha * acc (+ beta * A for the polynomial, read from the D box) written
// as bf16 to the D box in place (64-byte swizzle) and, for a tile off the diagonal,
// to the transposed box T[c][brow] (32 rows of 128 columns, no swizzle), whose store
// writes the mirrored elements.  d_s: the D box row of the warp's first row.
template <int MODE>
__device__ __forceinline__ void sym_compute(uint32_t d_s, uint32_t t_s, int lane, int brow, float alpha, float beta,
                                            const uint32_t (&v)[32], bool offdiag, int kbase = 0) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t off = eu_off(lane, kbase + k);
        float y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] = alpha * __uint_as_float(v[8 * k + e]);
        if (MODE == MODE_POLY) {
            const uint4 av = lds128(d_s + off);
            const uint32_t a4[4] = {av.x, av.y, av.z, av.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                y[2 * e] += beta * bf16_bits_lo(a4[e]);
                y[2 * e + 1] += beta * bf16_bits_hi(a4[e]);
            }
        }
        const uint32_t w0 = pack_bf16x2(y[0], y[1]), w1 = pack_bf16x2(y[2], y[3]);
        const uint32_t w2 = pack_bf16x2(y[4], y[5]), w3 = pack_bf16x2(y[6], y[7]);
        sts128(d_s + off, make_uint4(w0, w1, w2, w3));
        if (offdiag) {
            const uint32_t w[4] = {w0, w1, w2, w3};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const uint32_t c = (uint32_t)(8 * (kbase + k) + 2 * e);
                asm volatile("st.shared.b16 [%0], %1;" :: "r"(t_s + c * 256u + (uint32_t)brow * 2u),
                             "h"((unsigned short)(w[e] & 0xFFFFu)) : "memory");
                asm volatile("st.shared.b16 [%0], %1;" :: "r"(t_s + (c + 1u) * 256u + (uint32_t)brow * 2u),
                             "h"((unsigned short)(w[e] >> 16)) : "memory");
            }
        }
    }
}

// The TMA warp of one column half of the two-CTA epilogue (one elected
// thread): walks the half's load chunks of every unit of its cluster in order,
// loading chunk j + D - 1 into the ring once chunk j - 1's stores have read
// their buffer (with a ring of one buffer: chunk j + 1 once chunk j's stores have),
// and storing chunk j once the half's four compute warps have arrived on its done
// barrier.  Returns false when a bounded wait gave up.
template <int MODE, int D>
__device__ __forceinline__ bool pair_epilogue_tma(const GemmParams& p, uint32_t rank, int half, uint8_t* ebuf,
                                                  uint64_t* efull, uint64_t* edone, int4* coord,
                                                  volatile int* abort_flag, int cid) {
    const int u_begin = p.unit_begin[cid], u_end = p.unit_begin[cid + 1];
    // next (unit, chunk) to look at, with that unit's descriptor and group shape
    int iu = u_begin - 1, ic = 0, inch = 0, igm = 0, ign = 0;
    int4 itile = make_int4(0, 0, 0, 0), isk = make_int4(0, 0, 0, 0);
    // coord[b]: (group, matrix, row0, col0) of the chunk in buffer b (shared memory)
    uint32_t issued = 0, stored = 0;
    bool more = true, ok = true;
    // store groups that may still be reading their buffer after the wait below
    constexpr uint32_t WR = D > 1 ? 1u : 0u;
    while (true) {
        // load chunk i once the stores of chunk i - D have read its buffer: after
        // the wait below, every store but the last WR ones has
        while (more && issued + WR < stored + D) {
            if (ic >= inch) {
                if (++iu >= u_end) { more = false; break; }
                itile = p.units[2 * iu];
                isk = p.units[2 * iu + 1];
                inch = eu_nchunks(isk);
                igm = p.groups[itile.x].m;
                ign = MODE == MODE_UPDATE ? p.groups[itile.x].n : igm;     // GRAM / POLY: m x m output
                ic = 0;
                continue;
            }
            const EuChunk ch = eu_chunk(itile, isk, igm, ign, ic, (int)rank, half);
            ++ic;
            if (!ch.load) continue;
            const uint32_t b = issued % D;
            uint8_t* dst = ebuf + b * EU_BUF;
            const GemmMaps& mp = p.maps[ch.g];
            coord[b] = make_int4(ch.g, ch.mat, ch.row0, ch.col0);
            if (MODE == MODE_UPDATE) {
                mbar_arrive_expect_tx(&efull[b], EU_BUF);
                tma_load_3d(dst, &mp.xe_hi[p.parity], &efull[b], ch.col0, ch.row0, ch.mat);
                tma_load_3d(dst + EU_BOX, &mp.xe_lo_in, &efull[b], ch.col0, ch.row0, ch.mat);
            } else if (MODE == MODE_POLY) {
                mbar_arrive_expect_tx(&efull[b], EU_BOX);     // A, for the b*A term
                tma_load_3d(dst, &mp.se_a[0], &efull[b], ch.col0, ch.row0, ch.mat);
            } else {
                mbar_arrive(&efull[b]);                        // GRAM: the buffer is free
            }
            ++issued;
        }
        if (stored == issued) break;
        const uint32_t b = stored % D;
        if (!mbar_wait(&edone[b], (stored / D) & 1u, abort_flag, p.err, ERR_EPILOGUE)) { ok = false; break; }
        const int4 cd = coord[b];
        const GemmMaps& mp = p.maps[cd.x];
        if (MODE == MODE_UPDATE) {
            tma_store_3d(&mp.xe_hi[p.parity ^ 1], ebuf + b * EU_BUF, cd.w, cd.z, cd.y);
            tma_store_3d(&mp.xe_lo_out, ebuf + b * EU_BUF + EU_BOX, cd.w, cd.z, cd.y);
        } else {
            const CUtensorMap* out = MODE == MODE_GRAM ? mp.se_a : mp.se_p;
            tma_store_3d(&out[0], ebuf + b * EU_BUF, cd.w, cd.z, cd.y);
            // a tile off the diagonal also writes its mirror: rows col0.., columns row0..
            if ((cd.z / S2_BM) != (cd.w / S2_BN)) tma_store_3d(&out[1], ebuf + b * EU_BUF + EU_BOX, cd.z, cd.w, cd.y);
        }
        bulk_commit();
        ++stored;
        bulk_wait_read<WR>();             // every store but the last WR ones has read its buffer
    }
    bulk_wait_all();
    // loads still in flight (after an abort) must land before the CTA retires
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = stored; i < issued; ++i)
        while (!mbar_try_wait(&efull[i % D], (i / D) & 1u) && globaltimer_ns() - t0 < 100000000ull) { }
    return ok;
}

// One compute warp of the two-CTA UPDATE epilogue: X' = alpha * acc + beta * (hi + lo),
// stored as the pair hi' = bf16(X'), lo' = bf16(X' - hi'), for the warp's 32 rows of
// every chunk of its column half.  Each lane owns one row (the tcgen05.ld 32x32b
// layout) and rewrites its row of both boxes in place; the warp then arrives on the
// chunk's done barrier for the TMA warp.  The fused weight update (last iteration)
// follows from registers.  Returns false when a bounded wait gave up.
template <int MODE, int D>
__device__ __forceinline__ bool pair_epilogue_compute(const GemmParams& p, uint32_t rank, uint32_t warp,
                                                      uint32_t tmem_base, uint8_t* ebuf, uint64_t* efull,
                                                      uint64_t* edone, uint64_t* tfull, uint64_t* tempty,
                                                      volatile int* abort_flag, int cid) {
    const uint32_t lane = threadIdx.x & 31u;
    const int q = (int)(warp & 3u), half = (int)((warp - 2) >> 2);
    const int u_begin = p.unit_begin[cid], u_end = p.unit_begin[cid + 1];
    const int brow = q * 32 + (int)lane;             // this lane's row in the chunk boxes
    uint32_t consumed = 0;
    bool ok = true;
    int local = 0;
    for (int u = u_begin; u < u_end && ok; ++u, ++local) {
        const int4 tile = p.units[2 * u];
        const int4 sk = p.units[2 * u + 1];
        const int kind = sk.z & 0xFF, nh = sk.z >> 8, slot = sk.w & 0xFFFF, nsl = sk.w >> 16;
        const GemmGroupInfo& gi = p.groups[tile.x];
        const int gm = gi.m, gn = MODE == MODE_UPDATE ? gi.n : gi.m;
        const uint32_t acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        const int row = tile.z * S2_BM + (int)rank * 128 + brow;
        const bool offdiag = tile.z != tile.w;
        if (MODE == MODE_UPDATE && kind != 2)
            prefetch_w_row(p, gi, tile.y, row, tile.w * S2_BN + (nh ? (nh - 1) * 128 + half * 64 : half * 128),
                           nh ? 64 : 128);
        ok = mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err, ERR_EPILOGUE);
        if (kind == 1 && lane == 0) {
            for (int sl = 0; sl < nsl && ok; ++sl)
                ok = flag_wait(&p.sk_flag[slot + sl], p.epoch, abort_flag, p.err, ERR_SPLIT);
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0 && ok;
        if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
        tc_fence_after();
        float alpha = p.alpha, beta = p.beta;
        if (p.scale != nullptr) {
            // first iteration: A0 = s^2 U U^T, X1 = s P U + a s U
            const float sc = p.scale[gi.mat_base + tile.y];
            alpha *= MODE == MODE_GRAM ? sc * sc : sc;
            if (MODE == MODE_UPDATE) beta *= sc;
        }
        float* sk_row = kind == 0 ? nullptr
                      : p.sk_partial + (size_t)slot * SK_SLOT_FLOATS + ((size_t)rank * 128 + brow) * 256;
        const uint32_t tacc = tmem_base + acc * ACC_COLS + (((uint32_t)q * 32u) << 16);
        const EwSeg* sg = (MODE == MODE_UPDATE && p.apply_mode != 0) ? &p.segs[gi.mat_base + tile.y] : nullptr;
        const int nch = (nh ? 64 : 128) / EU_COLS;
        for (int c = 0; c < nch; ++c) {
            const EuChunk ch = eu_chunk(tile, sk, gm, gn, c, (int)rank, half);
            if (kind == 2) {
                // a later K range of a split tile: its raw partial sum goes to the slot
                for (int sub = 0; sub < EU_COLS / 32; ++sub) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tacc + (uint32_t)(ch.tcol + 32 * sub), v);
                    tmem_ld_wait();
                    float4* dst = reinterpret_cast<float4*>(sk_row + ch.tcol + 32 * sub);
#pragma unroll
                    for (int qq = 0; qq < 8; ++qq)
                        dst[qq] = make_float4(__uint_as_float(v[4 * qq]), __uint_as_float(v[4 * qq + 1]),
                                              __uint_as_float(v[4 * qq + 2]), __uint_as_float(v[4 * qq + 3]));
                }
                continue;
            }
            if (!ch.load) continue;               // the CTA's rows or the columns lie outside the matrix
            const uint32_t b = consumed % D;
            ok = mbar_wait(&efull[b], (consumed / D) & 1u, abort_flag, p.err, ERR_EPILOGUE);
            if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
            const uint32_t hi_s = smem_u32(ebuf + b * EU_BUF) + (uint32_t)(q * 32 * EU_ROW_BYTES), lo_s = hi_s + EU_BOX;
            // 32 accumulator columns at a time (one tcgen05.ld)
#pragma unroll 1
            for (int sub = 0; sub < EU_COLS / 32; ++sub) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tacc + (uint32_t)(ch.tcol + 32 * sub), v);
                tmem_ld_wait();
                if (kind == 1) {
                    for (int sl = 0; sl < nsl; ++sl) {
                        const float4* src =
                            reinterpret_cast<const float4*>(sk_row + (size_t)sl * SK_SLOT_FLOATS + ch.tcol + 32 * sub);
#pragma unroll
                        for (int qq = 0; qq < 8; ++qq) {
                            const float4 x = __ldcg(src + qq);
                            v[4 * qq + 0] = __float_as_uint(__uint_as_float(v[4 * qq + 0]) + x.x);
                            v[4 * qq + 1] = __float_as_uint(__uint_as_float(v[4 * qq + 1]) + x.y);
                            v[4 * qq + 2] = __float_as_uint(__uint_as_float(v[4 * qq + 2]) + x.z);
                            v[4 * qq + 3] = __float_as_uint(__uint_as_float(v[4 * qq + 3]) + x.w);
                        }
                    }
                }
                if (MODE != MODE_UPDATE) {
                    // hi_s: the D box rows of this warp; the T box follows the D box
                    sym_compute<MODE>(hi_s, smem_u32(ebuf + b * EU_BUF) + EU_BOX, (int)lane, brow, alpha, beta, v,
                                      offdiag, 4 * sub);
                } else if (sg != nullptr) {
                    eu_compute<true>(hi_s, lo_s, (int)lane, alpha, beta, v, 4 * sub);
                    if (row < gm) apply_row<32>(p, gi, *sg, row, ch.col0 + 32 * sub, v);
                } else {
                    eu_compute<false>(hi_s, lo_s, (int)lane, alpha, beta, v, 4 * sub);
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&edone[b]);
            ++consumed;
        }
        if (!ok) break;
        tc_fence_before();
        if (kind == 2) __threadfence();
        __syncwarp();
        if (lane == 0) {
            if (kind == 2 && atomicAdd(&p.sk_count[slot], 1) == 2 * NUM_EPI_WARPS - 1) {
                // last of the 16 epilogue warps of the pair: the slot is complete
                p.sk_count[slot] = 0;
                __threadfence();
                st_release_gpu(&p.sk_flag[slot], p.epoch);
            }
            mbar_arrive_remote(mapa_shared(smem_u32(&tempty[acc]), 0));
        }
    }
    return ok;
}

// ============================================================================ two-CTA kernel

template <int MODE, int VAR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(s2_threads(MODE), 1)
ns_gemm_tc2_kernel(const __grid_constant__ GemmParams p) {
    constexpr int STAGES = s2_stages(VAR);
    constexpr int ED = eu_depth(VAR);                  // epilogue ring depth
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * S2_A;
    uint8_t* sE = smem + STAGES * (S2_A + S2_B);          // epilogue buffers
    uint64_t* full = reinterpret_cast<uint64_t*>(sE + s2_epi_bytes(VAR));
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint64_t* ebar = drain + 1;                            // UPDATE: ED per epilogue warp
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ebar + 4 * ED);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    // 2 x ED chunk coordinates after the TMEM address and the abort flag, rounded
    // up to a 16-byte boundary
    int4* ecoord = reinterpret_cast<int4*>((reinterpret_cast<uintptr_t>(tmem_slot + 2) + 15) & ~uintptr_t(15));

    const uint32_t warp = warp_id();
    const uint32_t rank = cluster_ctarank();          // 0: issues the MMA
    const int cid = (int)cluster_id_x();               // index of this pair's unit list

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);                   // used in CTA 0: its producer's arrive + both CTAs' bytes
            mbar_init(&empty[s], 1);                  // one commit from the MMA thread
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 2 * NUM_EPI_WARPS); // used in CTA 0: epilogue warps of both CTAs
        }
        mbar_init(drain, 1);
        for (int h = 0; h < 2; ++h)
                for (int i = 0; i < ED; ++i) {
                    mbar_init(&ebar[h * 2 * ED + i], 1);                  // full: the TMA warp's expect_tx
                    mbar_init(&ebar[h * 2 * ED + ED + i], 4);       // done: the half's compute warps
                }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_trigger();
    pdl_wait();             // operands and outputs belong to the previous kernels

    if (warp == 0) {
        if (elect_one()) {
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            const int u_begin = p.unit_begin[cid], u_end = p.unit_begin[cid + 1];
            // the next unit's descriptor is loaded one unit ahead: its latency hides
            // behind the current unit's loads instead of stalling the ring
            int4 tile_next = make_int4(0, 0, 0, 0), sk_next = make_int4(0, 0, 0, 0);
            if (u_begin < u_end) { tile_next = p.units[2 * u_begin]; sk_next = p.units[2 * u_begin + 1]; }
            for (int u = u_begin; u < u_end && ok; ++u) {
                const int4 tile = tile_next;
                const int4 sk = sk_next;
                if (u + 1 < u_end) { tile_next = p.units[2 * u + 2]; sk_next = p.units[2 * u + 3]; }
                const void *mapA, *mapB;
                operand_maps<MODE>(p, tile.x, mapA, mapB);
                const int nh = sk.z >> 8;                              // 0: full tile, 1/2: column half
                const int row0 = tile.z * S2_BM + (int)rank * 128;     // this CTA's rows of A
                const int colh = tile.w * S2_BN + (nh ? (nh - 1) * 128 + (int)rank * 64 : (int)rank * 128);
                const int mat = tile.y;
                for (int kb = sk.x; kb < sk.y; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, ERR_PRODUCER)) { ok = false; break; }
                    const uint32_t full0 = mapa_shared(smem_u32(&full[stage]), 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * (S2_A + S2_B));
                    const int k0 = kb * BK;
                    uint8_t* a_dst = sA + stage * S2_A;
                    uint8_t* b_dst = sB + stage * S2_B;
                    tma_load_3d_pair(a_dst, mapA, full0, k0, row0, mat);
                    if (MODE == MODE_UPDATE) {
                        tma_load_3d_pair(b_dst, mapB, full0, colh, k0, mat);
                        tma_load_3d_pair(b_dst + BK * 128, mapB, full0, colh + 64, k0, mat);
                    } else {
                        tma_load_3d_pair(b_dst, mapB, full0, k0, colh, mat);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            for (int i = 0; i < STAGES && ok; ++i) {
                if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, ERR_TAIL)) ok = false;
                if (++stage == STAGES) { stage = 0; phase ^= 1u; }
            }
            if (!ok || *abort_flag) spin_ns(2000000ull);
        }
    } else if (warp == 1) {
        if (rank == 0 && elect_one()) {
            constexpr uint32_t idesc_full = idesc_bf16_f32(S2_BM, S2_BN, MODE == MODE_UPDATE ? 1u : 0u);
            constexpr uint32_t idesc_half = idesc_bf16_f32(S2_BM, S2_BN / 2, MODE == MODE_UPDATE ? 1u : 0u);
            uint32_t stage = 0, phase = 0;
            int local = 0;
            bool ok = true;
            const int u_begin = p.unit_begin[cid], u_end = p.unit_begin[cid + 1];
            // loaded one unit ahead, so that the tensor pipe does not drain while the
            // next unit's K range is fetched
            int4 sk_next = u_begin < u_end ? p.units[2 * u_begin + 1] : make_int4(0, 0, 0, 0);
            for (int u = u_begin; u < u_end && ok; ++u, ++local) {
                const int4 sk = sk_next;
                if (u + 1 < u_end) sk_next = p.units[2 * u + 3];
                const uint32_t idesc = (sk.z >> 8) ? idesc_half : idesc_full;
                const uint32_t acc = local & 1;
                const uint32_t acc_phase = (local >> 1) & 1;
                if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, p.err, ERR_MMA_ACC)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + acc * ACC_COLS;
                for (int kb = sk.x; kb < sk.y; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag, p.err, ERR_MMA_SLOT)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA + stage * S2_A);
                    const uint32_t b_base = smem_u32(sB + stage * S2_B);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t adesc = smem_desc_sw128(a_base + kk * 32, 16, 1024);
                        uint64_t bdesc;
                        if (MODE == MODE_UPDATE) bdesc = smem_desc_sw128(b_base + kk * 2048, BK * 128, 1024);
                        else bdesc = smem_desc_sw128(b_base + kk * 32, 16, 1024);
                        tc_mma_f16_pair(d_tmem, adesc, bdesc, idesc, (kb != sk.x || kk != 0) ? 1u : 0u);
                    }
                    const uint32_t e_own = mapa_shared(smem_u32(&empty[stage]), 0);
                    const uint32_t e_peer = mapa_shared(smem_u32(&empty[stage]), 1);
                    tc_commit_pair(e_own);
                    tc_commit_pair(e_peer);
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit_pair(mapa_shared(smem_u32(&tfull[acc]), 0));
                tc_commit_pair(mapa_shared(smem_u32(&tfull[acc]), 1));
            }
            if (!ok || *abort_flag) {
                tc_commit_pair(mapa_shared(smem_u32(drain), 0));
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < 100000000ull) { }
            }
        }
    } else {
        // ring of column half h: buffers sE + h * ED * EU_BUF, barriers
        // ebar[2h * ED ...]: ED full (TMA loads), then ED done (compute warps)
        if (warp < 2 + NUM_EPI_WARPS) {
            const int h = (int)((warp - 2) >> 2);
            pair_epilogue_compute<MODE, ED>(p, rank, warp, tmem_base, sE + h * (ED * EU_BUF), ebar + h * 2 * ED,
                                        ebar + h * 2 * ED + ED, tfull, tempty, abort_flag, cid);
        } else if (elect_one()) {
            const int h = (int)(warp - 2 - NUM_EPI_WARPS);
            pair_epilogue_tma<MODE, ED>(p, rank, h, sE + h * (ED * EU_BUF), ebar + h * 2 * ED,
                                    ebar + h * 2 * ED + ED, ecoord + h * ED, abort_flag, cid);
        }
    }

    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

}  // namespace

int tc_gemm_epi_cols() { return EU_COLS; }
int tc_gemm_epi_rows() { return EU_ROWS; }
int tc_gemm_threads() { return NUM_THREADS; }
int tc_gemm_tile_m(int pair) { return pair ? S2_BM : S1_BM; }
int tc_gemm_tile_n(int pair) { return pair ? S2_BN : S1_BN; }

cudaError_t tc_gemm_prepare() {
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(ns_gemm_tc_kernel<MODE_GRAM>, cudaFuncAttributeMaxDynamicSharedMemorySize, S1_SMEM)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ns_gemm_tc_kernel<MODE_POLY>, cudaFuncAttributeMaxDynamicSharedMemorySize, S1_SMEM)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ns_gemm_tc_kernel<MODE_UPDATE>, cudaFuncAttributeMaxDynamicSharedMemorySize, S1_SMEM)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ns_gemm_tc2_kernel<MODE_GRAM, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, S2_SMEM)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ns_gemm_tc2_kernel<MODE_POLY, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, S2U_SMEM)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ns_gemm_tc2_kernel<MODE_POLY, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, S2_SMEM)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ns_gemm_tc2_kernel<MODE_UPDATE, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize, S2U_SMEM)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ns_gemm_tc2_kernel<MODE_UPDATE, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, S2_SMEM)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ns_gemm_tc2_kernel<MODE_GRAM, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, S2L_SMEM)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ns_gemm_tc2_kernel<MODE_POLY, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, S2L_SMEM)) != cudaSuccess) return e;
    return cudaFuncSetAttribute(ns_gemm_tc2_kernel<MODE_UPDATE, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, S2L_SMEM);
}

cudaError_t tc_gemm_max_clusters(int* n) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS_U, 1, 1);
    cfg.dynamicSmemBytes = S2U_SMEM;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nu = 0, ng = 0;
    cudaError_t e = cudaOccupancyMaxActiveClusters(&nu, ns_gemm_tc2_kernel<MODE_UPDATE, 0>, &cfg);
    if (e != cudaSuccess) return e;
    cfg.dynamicSmemBytes = S2L_SMEM;
    e = cudaOccupancyMaxActiveClusters(&ng, ns_gemm_tc2_kernel<MODE_GRAM, 2>, &cfg);
    *n = nu < ng ? nu : ng;
    return e;
}

// average K from which a phase takes VAR 2 (the deepest operand ring).  The Gram's
// epilogue loads nothing, so it takes VAR 2 at every K (measured 1-2 % faster than
// VAR 1 on the GPT-2 and MoE workloads, equal at 4096^2); for the polynomial and
// the update a one-buffer ring is only good when a tile's main loop is long.
#ifndef MUON_GRAM_VAR2_K
#define MUON_GRAM_VAR2_K 0
#endif
#ifndef MUON_POLY_VAR2_K
#define MUON_POLY_VAR2_K (1 << 30)
#endif
#ifndef MUON_UPD_VAR2_K
#define MUON_UPD_VAR2_K 3072
#endif

int tc_gemm_var(int mode, int avg_k) {
    if (mode == MODE_GRAM) return avg_k >= MUON_GRAM_VAR2_K ? 2 : 1;
    if (mode == MODE_POLY) return avg_k >= MUON_POLY_VAR2_K ? 2 : avg_k >= 1024 ? 1 : 0;
    return avg_k >= MUON_UPD_VAR2_K ? 2 : avg_k >= 2048 ? 1 : 0;
}

cudaError_t launch_tc_gemm(int mode, int pair, const GemmParams& p, int grid, cudaStream_t s, int var) {
    if (p.ntiles <= 0) return cudaSuccess;
    const dim3 g(grid), b(NUM_THREADS), bu(NUM_THREADS_U);
    if (pair) {
        switch (mode) {
            case MODE_GRAM:
                return var == 2 ? launch_pdl(ns_gemm_tc2_kernel<MODE_GRAM, 2>, g, bu, S2L_SMEM, s, p)
                                : launch_pdl(ns_gemm_tc2_kernel<MODE_GRAM, 1>, g, bu, S2_SMEM, s, p);
            case MODE_POLY:
                return var == 2 ? launch_pdl(ns_gemm_tc2_kernel<MODE_POLY, 2>, g, bu, S2L_SMEM, s, p)
                     : var      ? launch_pdl(ns_gemm_tc2_kernel<MODE_POLY, 1>, g, bu, S2_SMEM, s, p)
                                : launch_pdl(ns_gemm_tc2_kernel<MODE_POLY, 0>, g, bu, S2U_SMEM, s, p);
            default:
                return var == 2 ? launch_pdl(ns_gemm_tc2_kernel<MODE_UPDATE, 2>, g, bu, S2L_SMEM, s, p)
                     : var      ? launch_pdl(ns_gemm_tc2_kernel<MODE_UPDATE, 1>, g, bu, S2_SMEM, s, p)
                                : launch_pdl(ns_gemm_tc2_kernel<MODE_UPDATE, 0>, g, bu, S2U_SMEM, s, p);
        }
    }
    switch (mode) {
        case MODE_GRAM: return launch_pdl(ns_gemm_tc_kernel<MODE_GRAM>, g, b, S1_SMEM, s, p);
        case MODE_POLY: return launch_pdl(ns_gemm_tc_kernel<MODE_POLY>, g, b, S1_SMEM, s, p);
        default: return launch_pdl(ns_gemm_tc_kernel<MODE_UPDATE>, g, b, S1_SMEM, s, p);
    }
}

}  // namespace muon
