// elementwise.cu -- the memory-bound phases of the Muon step.
//
//  momentum_norm   B <- mu*B + G                    ("Muon: An optimizer for hidden layers
//                  U <- G + mu*B (Nesterov) or B     in neural networks", section 4, eq. 1
//                                                    and its Nesterov remark)
//                  X0 <- U, or U^T when rows > cols  (section 4: smaller-Gram orientation)
//                  per-block sum of U^2 in fp64      (section 4: Frobenius normalisation)
//                  the last block of each matrix to finish sums that matrix's
//                  partials in a fixed order: ||U||_F and s = 1/(||U||_F + eps)
//  apply           W <- (1 - lr*wd) W - lr*s_shape*O (eq. 3 with decoupled decay and the
//                  per-shape scale of the Moonlight result), O read back transposed
//                  when the matrix was oriented; or O copied out (orthogonalisation only)
//
// One launch covers every matrix of the call: the block index is mapped to its
// matrix by a binary search over the per-matrix block ranges.  Square or wide
// matrices take a flat path (8 elements per thread per access, 16/32-byte
// vectors); tall matrices go through a 64x64 shared-memory transpose so that
// both the row-major reads and the transposed writes stay coalesced.
#include <algorithm>

#include "kernels.cuh"
#include "ptx.cuh"

#ifndef EW_GROUPS_IN_FLIGHT
#define EW_GROUPS_IN_FLIGHT 2
#endif
#ifndef EW_MIN_BLOCKS
#define EW_MIN_BLOCKS 4
#endif

namespace muon {
namespace {

__device__ __forceinline__ int find_seg(const EwSeg* segs, int nseg, int blk, bool apply) {
    int lo = 0, hi = nseg - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        const int b = apply ? segs[mid].apply_begin : segs[mid].blk_begin;
        if (b <= blk) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) red[w] = v;
    __syncthreads();
    double r = 0.0;
    if (threadIdx.x == 0) {
        for (int i = 0; i < EW_THREADS / 32; ++i) r += red[i];
    }
    return r;
}

__device__ __forceinline__ float load_g(const void* g, size_t i, int bf16) {
    return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(g)[i])
                : reinterpret_cast<const float*>(g)[i];
}

__device__ __forceinline__ float direction(float g, float* bptr, float mu, int nesterov) {
    if (bptr == nullptr) return g;                     // orthogonalisation only: U = M
    const float bn = fmaf(mu, *bptr, g);               // eq. 1
    *bptr = bn;
    return nesterov ? fmaf(mu, bn, g) : bn;
}

// hi = bf16(x), lo = bf16(x - hi), for two values, packed as bf16x2 words
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

__device__ __forceinline__ uint32_t pack2_bf16(float a, float b) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void store_x0(const EwSeg& sg, size_t xo, float u, int bf16_operand) {
    if (bf16_operand) {
        const __nv_bfloat16 h = __float2bfloat16_rn(u);
        sg.xhi0[xo] = h;
        sg.xlo0[xo] = __float2bfloat16_rn(u - __bfloat162float(h));
    } else {
        sg.xf0[xo] = u;
    }
}

// Element i (index into the oriented m x ldn iterate) of the final X: the bf16 pair
// o_hi + o_lo, o_hi alone (a bf16 O given to muon_apply), or fp32 o_src.
__device__ __forceinline__ float load_o(const EwSeg& sg, size_t i) {
    if (sg.o_hi) return __bfloat162float(sg.o_hi[i]) + (sg.o_lo ? __bfloat162float(sg.o_lo[i]) : 0.f);
    return sg.o_src[i];
}

// Eight consecutive values of O from element i (16-byte aligned for bf16, 32-byte for fp32).
__device__ __forceinline__ void load_o8(const EwSeg& sg, size_t i, float (&o)[8]) {
    if (sg.o_hi) {
        const uint4 h = *reinterpret_cast<const uint4*>(sg.o_hi + i);
        const uint4 l = sg.o_lo ? *reinterpret_cast<const uint4*>(sg.o_lo + i) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t hw[4] = {h.x, h.y, h.z, h.w}, lw[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            o[2 * q] = __uint_as_float(hw[q] << 16) + __uint_as_float(lw[q] << 16);
            o[2 * q + 1] = __uint_as_float(hw[q] & 0xFFFF0000u) + __uint_as_float(lw[q] & 0xFFFF0000u);
        }
    } else {
        const float4 a = *reinterpret_cast<const float4*>(sg.o_src + i);
        const float4 b = *reinterpret_cast<const float4*>(sg.o_src + i + 4);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w; o[4] = b.x; o[5] = b.y; o[6] = b.z; o[7] = b.w;
    }
}

// Copy-out of one value of O to element i of the destination (fp32, or bf16 when
// the segment asks for it).
__device__ __forceinline__ void store_out(const EwSeg& sg, float* dst, size_t i, float v) {
    if (sg.out_bf16) reinterpret_cast<__nv_bfloat16*>(dst)[i] = __float2bfloat16_rn(v);
    else dst[i] = v;
}

__global__ void __launch_bounds__(EW_THREADS, EW_MIN_BLOCKS) momentum_norm_kernel(const EwSeg* __restrict__ segs, int nseg,
                                                                  double* __restrict__ partials, float mu,
                                                                  int nesterov, int bf16_operand,
                                                                  int* __restrict__ counters, float eps,
                                                                  float* __restrict__ norms, float* __restrict__ scale) {
    __shared__ float tile_t[MT_COLS][MT_ROWS + 1];     // transposed tile of a tall matrix
    __shared__ double red[EW_THREADS / 32];
    pdl_trigger();
    pdl_wait();
    const int si = find_seg(segs, nseg, blockIdx.x, false);
    const EwSeg sg = segs[si];
    const int lb = blockIdx.x - sg.blk_begin;
    double acc = 0.0;
    // bf16 path: X0 = hi + lo (hi = bf16(u), lo = bf16(u - hi)); fp32 debug path: X0 in fp32

    if (!sg.transposed) {
        const size_t total = (size_t)sg.rows * sg.cols;
        const size_t e0 = (size_t)lb * EW_FLAT_ELEMS;
        const size_t e1 = min(total, e0 + EW_FLAT_ELEMS);
        if (sg.vec && sg.b != nullptr) {
            // rows are dense and 8-aligned: the oriented X has the same flat index.
            // All loads of the thread's (up to) 4 groups of 8 elements are issued
            // before any arithmetic: 12 (bf16 G) or 16 (fp32 G) 16-byte loads per
            // thread in flight.  bf16 G stays packed until it is used.
            constexpr int GROUPS = EW_FLAT_ELEMS / (EW_THREADS * 8);
            constexpr int GB = EW_GROUPS_IN_FLIGHT;
#pragma unroll 1
            for (int k0 = 0; k0 < GROUPS; k0 += GB) {
            uint4 graw[GB][2];
            float4 braw[GB][2];
#pragma unroll
            for (int kk = 0; kk < GB; ++kk) {
                const int k = k0 + kk;
                const size_t e = e0 + ((size_t)k * EW_THREADS + threadIdx.x) * 8;
                if (e >= e1) continue;
                if (sg.g_bf16) {
                    graw[kk][0] = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(sg.g) + e);
                } else {
                    graw[kk][0] = *reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(sg.g) + e);
                    graw[kk][1] = *reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(sg.g) + e + 4);
                }
                const float4* bp = reinterpret_cast<const float4*>(sg.b + e);
                braw[kk][0] = bp[0];
                braw[kk][1] = bp[1];
            }
#pragma unroll
            for (int kk = 0; kk < GB; ++kk) {
                const int k = k0 + kk;
                const size_t e = e0 + ((size_t)k * EW_THREADS + threadIdx.x) * 8;
                if (e >= e1) continue;
                float g[8], b[8], u[8];
                if (sg.g_bf16) {
                    const uint32_t w[4] = {graw[kk][0].x, graw[kk][0].y, graw[kk][0].z, graw[kk][0].w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        g[2 * i] = __uint_as_float(w[i] << 16);
                        g[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
                    }
                } else {
                    const uint32_t w[8] = {graw[kk][0].x, graw[kk][0].y, graw[kk][0].z, graw[kk][0].w,
                                           graw[kk][1].x, graw[kk][1].y, graw[kk][1].z, graw[kk][1].w};
#pragma unroll
                    for (int i = 0; i < 8; ++i) g[i] = __uint_as_float(w[i]);
                }
                b[0] = braw[kk][0].x; b[1] = braw[kk][0].y; b[2] = braw[kk][0].z; b[3] = braw[kk][0].w;
                b[4] = braw[kk][1].x; b[5] = braw[kk][1].y; b[6] = braw[kk][1].z; b[7] = braw[kk][1].w;
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    b[i] = fmaf(mu, b[i], g[i]);
                    u[i] = nesterov ? fmaf(mu, b[i], g[i]) : b[i];
                    acc += (double)u[i] * (double)u[i];
                }
                float4* bp = reinterpret_cast<float4*>(sg.b + e);
                bp[0] = make_float4(b[0], b[1], b[2], b[3]);
                bp[1] = make_float4(b[4], b[5], b[6], b[7]);
                if (bf16_operand) {
                    uint32_t hw[4], lw[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) split_bf16x2(u[2 * i], u[2 * i + 1], hw[i], lw[i]);
                    *reinterpret_cast<uint4*>(sg.xhi0 + e) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4*>(sg.xlo0 + e) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                } else {
                    float4* xp = reinterpret_cast<float4*>(sg.xf0 + e);
                    xp[0] = make_float4(u[0], u[1], u[2], u[3]);
                    xp[1] = make_float4(u[4], u[5], u[6], u[7]);
                }
            }
            }
        } else {
            for (size_t e = e0 + threadIdx.x; e < e1; e += EW_THREADS) {
                const size_t r = e / (size_t)sg.cols, c = e - r * (size_t)sg.cols;
                const float u = direction(load_g(sg.g, e, sg.g_bf16), sg.b ? sg.b + e : nullptr, mu, nesterov);
                acc += (double)u * (double)u;
                store_x0(sg, r * (size_t)sg.ldn + c, u, bf16_operand);
            }
        }
    } else {
        // tall matrix: X = U^T.  Tile of U rows [i0, i0 + MT_ROWS) x cols [j0, j0 + MT_COLS):
        // 8192 elements, the flat path's block size.  U is read and B written along W's
        // rows; X0 is written along X's rows from the shared tile tr[j][i] (row stride
        // MT_ROWS + 1), so both sides of the transpose stay coalesced.
        const int tiles_c = (sg.cols + MT_COLS - 1) / MT_COLS;
        const int i0 = (lb / tiles_c) * MT_ROWS, j0 = (lb % tiles_c) * MT_COLS;
        if (sg.vec && sg.b != nullptr) {
            // thread (cg, r): columns j0 + 8cg .. +7 of rows i0 + r + 16p, p = 0..3, two
            // rows' loads in flight before any arithmetic (cols % 8 == 0: a group of 8
            // columns lies wholly inside the matrix or wholly outside)
            const int cg = threadIdx.x & 15, r = threadIdx.x >> 4;
            const int j = j0 + 8 * cg;
#pragma unroll
            for (int p0 = 0; p0 < MT_ROWS / 16; p0 += 2) {
                uint4 graw[2][2];
                float4 braw[2][2];
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {
                    const int i = i0 + r + 16 * (p0 + pp);
                    if (i >= sg.rows || j >= sg.cols) continue;
                    const size_t e = (size_t)i * sg.cols + j;
                    if (sg.g_bf16) {
                        graw[pp][0] = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(sg.g) + e);
                    } else {
                        graw[pp][0] = *reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(sg.g) + e);
                        graw[pp][1] = *reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(sg.g) + e + 4);
                    }
                    const float4* bp = reinterpret_cast<const float4*>(sg.b + e);
                    braw[pp][0] = bp[0];
                    braw[pp][1] = bp[1];
                }
#pragma unroll
                for (int pp = 0; pp < 2; ++pp) {
                    const int ir = r + 16 * (p0 + pp), i = i0 + ir;
                    float u[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    if (i < sg.rows && j < sg.cols) {
                        float g[8];
                        if (sg.g_bf16) {
                            const uint32_t w[4] = {graw[pp][0].x, graw[pp][0].y, graw[pp][0].z, graw[pp][0].w};
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                g[2 * q] = __uint_as_float(w[q] << 16);
                                g[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
                            }
                        } else {
                            const uint32_t w[8] = {graw[pp][0].x, graw[pp][0].y, graw[pp][0].z, graw[pp][0].w,
                                                   graw[pp][1].x, graw[pp][1].y, graw[pp][1].z, graw[pp][1].w};
#pragma unroll
                            for (int q = 0; q < 8; ++q) g[q] = __uint_as_float(w[q]);
                        }
                        float bb[8] = {braw[pp][0].x, braw[pp][0].y, braw[pp][0].z, braw[pp][0].w,
                                       braw[pp][1].x, braw[pp][1].y, braw[pp][1].z, braw[pp][1].w};
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            bb[q] = fmaf(mu, bb[q], g[q]);
                            u[q] = nesterov ? fmaf(mu, bb[q], g[q]) : bb[q];
                            acc += (double)u[q] * (double)u[q];
                        }
                        float4* bp = reinterpret_cast<float4*>(sg.b + (size_t)i * sg.cols + j);
                        bp[0] = make_float4(bb[0], bb[1], bb[2], bb[3]);
                        bp[1] = make_float4(bb[4], bb[5], bb[6], bb[7]);
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q) tile_t[8 * cg + q][ir] = u[q];
                }
            }
        } else {
            // consecutive threads take consecutive columns of a row of U
            for (int e = threadIdx.x; e < MT_ROWS * MT_COLS; e += EW_THREADS) {
                const int ii = e / MT_COLS, jj = e % MT_COLS;
                const int i = i0 + ii, j = j0 + jj;
                float u = 0.f;
                if (i < sg.rows && j < sg.cols) {
                    const size_t ge = (size_t)i * sg.cols + j;
                    u = direction(load_g(sg.g, ge, sg.g_bf16), sg.b ? sg.b + ge : nullptr, mu, nesterov);
                    acc += (double)u * (double)u;
                }
                tile_t[jj][ii] = u;
            }
        }
        __syncthreads();
        // X0[j0 + jj][i0 + 8ig .. +7] = U[i0 + 8ig ..][j0 + jj]: thread (ig, jr) takes rows
        // jj = jr + 32s of X, s = 0..3; 8 lanes cover 64 contiguous elements of one row
        const int ig = threadIdx.x & 7, jr = threadIdx.x >> 3;
        const int ix = i0 + 8 * ig;
#pragma unroll
        for (int sidx = 0; sidx < MT_COLS / 32; ++sidx) {
            const int jj = jr + 32 * sidx, jx = j0 + jj;
            if (jx >= sg.cols || ix >= sg.rows) continue;
            float u[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) u[q] = tile_t[jj][8 * ig + q];
            const size_t xo = (size_t)jx * sg.ldn + ix;
            if (ix + 7 < sg.rows) {
                if (bf16_operand) {
                    uint32_t hw[4], lw[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) split_bf16x2(u[2 * q], u[2 * q + 1], hw[q], lw[q]);
                    *reinterpret_cast<uint4*>(sg.xhi0 + xo) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    *reinterpret_cast<uint4*>(sg.xlo0 + xo) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                } else {
                    float4* xp = reinterpret_cast<float4*>(sg.xf0 + xo);
                    xp[0] = make_float4(u[0], u[1], u[2], u[3]);
                    xp[1] = make_float4(u[4], u[5], u[6], u[7]);
                }
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    if (ix + q < sg.rows) store_x0(sg, xo + q, u[q], bf16_operand);
            }
        }
    }
    const double tot = block_sum(acc, red);
    __shared__ int is_last;
    if (threadIdx.x == 0) {
        partials[blockIdx.x] = tot;
        __threadfence();
        is_last = atomicAdd(&counters[sg.mat], 1) == sg.blk_count - 1;
    }
    __syncthreads();
    if (!is_last) return;
    // Last block of this matrix: every partial is visible.  Thread t sums partials
    // t, t + 256, ...; the block reduction then adds them in a fixed order, so the
    // result does not depend on which block finished last.
    __threadfence();
    double s2 = 0.0;
    for (int i = threadIdx.x; i < sg.blk_count; i += EW_THREADS)
        s2 += reinterpret_cast<volatile double*>(partials)[sg.blk_begin + i];
    __syncthreads();
    const double total = block_sum(s2, red);
    if (threadIdx.x == 0) {
        const double nrm = sqrt(total);
        norms[sg.mat] = (float)nrm;
        scale[sg.mat] = (float)(1.0 / (nrm + (double)eps));
        counters[sg.mat] = 0;           // ready for the next call
    }
}

// Apply (copy_out == 0) or copy-out (copy_out == 1) for one block of one matrix.
__device__ __forceinline__ void apply_block(const EwSeg& sg, int lb, float decay, float lr, const float* o_scale,
                                            int copy_out, float* dst) {
    const float os = o_scale ? o_scale[sg.mat] : 1.0f;
    const float step = lr * sg.update_scale;
    if (!sg.transposed) {
        const size_t total = (size_t)sg.rows * sg.cols;
        const size_t e0 = (size_t)lb * EW_FLAT_ELEMS;
        const size_t e1 = min(total, e0 + EW_FLAT_ELEMS);
        if (sg.vec) {
            for (size_t e = e0 + (size_t)threadIdx.x * 8; e < e1; e += (size_t)EW_THREADS * 8) {
                float4 o0, o1;
                if (sg.o_hi) {
                    const uint4 h = *reinterpret_cast<const uint4*>(sg.o_hi + e);
                    const uint4 l = sg.o_lo ? *reinterpret_cast<const uint4*>(sg.o_lo + e) : make_uint4(0u, 0u, 0u, 0u);
                    auto f = [](uint32_t a, uint32_t b, bool hi_half) {
                        return hi_half ? __uint_as_float(a & 0xFFFF0000u) + __uint_as_float(b & 0xFFFF0000u)
                                       : __uint_as_float(a << 16) + __uint_as_float(b << 16);
                    };
                    o0 = make_float4(f(h.x, l.x, false), f(h.x, l.x, true), f(h.y, l.y, false), f(h.y, l.y, true));
                    o1 = make_float4(f(h.z, l.z, false), f(h.z, l.z, true), f(h.w, l.w, false), f(h.w, l.w, true));
                } else {
                    const float4* op = reinterpret_cast<const float4*>(sg.o_src + e);
                    o0 = op[0];
                    o1 = op[1];
                }
                float4* wp = reinterpret_cast<float4*>(dst + e);
                if (copy_out) {
                    o0.x *= os; o0.y *= os; o0.z *= os; o0.w *= os; o1.x *= os; o1.y *= os; o1.z *= os; o1.w *= os;
                    if (sg.out_bf16) {
                        *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(dst) + e) =
                            make_uint4(pack2_bf16(o0.x, o0.y), pack2_bf16(o0.z, o0.w), pack2_bf16(o1.x, o1.y),
                                       pack2_bf16(o1.z, o1.w));
                    } else {
                        wp[0] = o0; wp[1] = o1;
                    }
                } else {
                    float4 w0 = wp[0], w1 = wp[1];
                    w0.x = fmaf(-step, o0.x * os, decay * w0.x); w0.y = fmaf(-step, o0.y * os, decay * w0.y);
                    w0.z = fmaf(-step, o0.z * os, decay * w0.z); w0.w = fmaf(-step, o0.w * os, decay * w0.w);
                    w1.x = fmaf(-step, o1.x * os, decay * w1.x); w1.y = fmaf(-step, o1.y * os, decay * w1.y);
                    w1.z = fmaf(-step, o1.z * os, decay * w1.z); w1.w = fmaf(-step, o1.w * os, decay * w1.w);
                    wp[0] = w0; wp[1] = w1;
                }
            }
        } else {
            for (size_t e = e0 + threadIdx.x; e < e1; e += EW_THREADS) {
                const size_t r = e / (size_t)sg.cols, c = e - r * (size_t)sg.cols;
                const float o = load_o(sg, r * (size_t)sg.ldn + c) * os;
                if (copy_out) store_out(sg, dst, e, o);
                else dst[e] = fmaf(-step, o, decay * dst[e]);
            }
        }
    } else {
        // O = X^T.  Tile of W rows [i0, i0 + MT_ROWS) x cols [j0, j0 + MT_COLS), the
        // momentum kernel's tile in reverse: O is read along X's rows into
        // tile_t[j][i], then W is read and written along its own rows, so both sides of
        // the transpose stay coalesced.
        __shared__ float tile_t[MT_COLS][MT_ROWS + 1];
        const int tiles_c = (sg.cols + MT_COLS - 1) / MT_COLS;
        const int i0 = (lb / tiles_c) * MT_ROWS, j0 = (lb % tiles_c) * MT_COLS;
        {
            // thread (ig, jr): X rows jj = jr + 32s, s = 0..3, elements i0 + 8ig .. +7;
            // 8 lanes cover 64 contiguous elements of a row, all four rows' loads in flight
            const int ig = threadIdx.x & 7, jr = threadIdx.x >> 3;
            const int ix = i0 + 8 * ig;
            float o[MT_COLS / 32][8];
#pragma unroll
            for (int sidx = 0; sidx < MT_COLS / 32; ++sidx) {
                const int jx = j0 + jr + 32 * sidx;
#pragma unroll
                for (int q = 0; q < 8; ++q) o[sidx][q] = 0.f;
                if (jx >= sg.cols || ix >= sg.rows) continue;
                const size_t xo = (size_t)jx * sg.ldn + ix;
                if (ix + 7 < sg.rows) load_o8(sg, xo, o[sidx]);
                else
                    for (int q = 0; q < 8; ++q)
                        if (ix + q < sg.rows) o[sidx][q] = load_o(sg, xo + q);
            }
#pragma unroll
            for (int sidx = 0; sidx < MT_COLS / 32; ++sidx)
#pragma unroll
                for (int q = 0; q < 8; ++q) tile_t[jr + 32 * sidx][8 * ig + q] = o[sidx][q] * os;
        }
        __syncthreads();
        if (sg.vec) {
            // thread (cg, r): columns j0 + 8cg .. +7 of rows i0 + r + 16p, p = 0..3 (cols % 8
            // == 0: a group of 8 columns lies wholly inside the matrix or wholly outside)
            const int cg = threadIdx.x & 15, r = threadIdx.x >> 4;
            const int j = j0 + 8 * cg;
            if (j < sg.cols) {
                float4 wv[MT_ROWS / 16][2];
                if (!copy_out) {
#pragma unroll
                    for (int pp = 0; pp < MT_ROWS / 16; ++pp) {
                        const int i = i0 + r + 16 * pp;
                        if (i >= sg.rows) continue;
                        const float4* wp = reinterpret_cast<const float4*>(dst + (size_t)i * sg.cols + j);
                        wv[pp][0] = wp[0];
                        wv[pp][1] = wp[1];
                    }
                }
#pragma unroll
                for (int pp = 0; pp < MT_ROWS / 16; ++pp) {
                    const int ir = r + 16 * pp, i = i0 + ir;
                    if (i >= sg.rows) continue;
                    float v[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) v[q] = tile_t[8 * cg + q][ir];
                    const size_t e = (size_t)i * sg.cols + j;
                    if (copy_out && sg.out_bf16) {
                        *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(dst) + e) =
                            make_uint4(pack2_bf16(v[0], v[1]), pack2_bf16(v[2], v[3]), pack2_bf16(v[4], v[5]),
                                       pack2_bf16(v[6], v[7]));
                        continue;
                    }
                    if (!copy_out) {
                        const float w8[8] = {wv[pp][0].x, wv[pp][0].y, wv[pp][0].z, wv[pp][0].w,
                                             wv[pp][1].x, wv[pp][1].y, wv[pp][1].z, wv[pp][1].w};
#pragma unroll
                        for (int q = 0; q < 8; ++q) v[q] = fmaf(-step, v[q], decay * w8[q]);
                    }
                    float4* wp = reinterpret_cast<float4*>(dst + e);
                    wp[0] = make_float4(v[0], v[1], v[2], v[3]);
                    wp[1] = make_float4(v[4], v[5], v[6], v[7]);
                }
            }
        } else {
            // consecutive threads take consecutive columns of a row of W
            for (int e = threadIdx.x; e < MT_ROWS * MT_COLS; e += EW_THREADS) {
                const int ii = e / MT_COLS, jj = e % MT_COLS;
                const int i = i0 + ii, j = j0 + jj;
                if (i >= sg.rows || j >= sg.cols) continue;
                const size_t we = (size_t)i * sg.cols + j;
                const float o = tile_t[jj][ii];
                if (copy_out) store_out(sg, dst, we, o);
                else dst[we] = fmaf(-step, o, decay * dst[we]);
            }
        }
    }
}

__global__ void __launch_bounds__(EW_THREADS) apply_kernel(const EwSeg* __restrict__ segs, int nseg, float decay,
                                                          float lr, const float* __restrict__ o_scale, int copy_out) {
    pdl_trigger();
    pdl_wait();
    const int si = find_seg(segs, nseg, blockIdx.x, true);
    const EwSeg sg = segs[si];
    apply_block(sg, blockIdx.x - sg.apply_begin, decay, lr, o_scale, copy_out, sg.w);
}

__global__ void __launch_bounds__(EW_THREADS) copy_out_one_kernel(const EwSeg sg, float* dst, const float* o_scale) {
    pdl_trigger();
    pdl_wait();
    apply_block(sg, blockIdx.x, 1.0f, 0.0f, o_scale, 1, dst);
}

// RMS of the applied update lr * s * O of every matrix, over the final iterate
// (RMS does not depend on the orientation).  Block (c, mat) sums the squares of
// rows c, c + RMS_CHUNKS, ... of the matrix's oriented m x n iterate in fp64;
// update_rms_finish_kernel adds the RMS_CHUNKS partials of each matrix in a fixed
// order, so the result is bitwise reproducible.
constexpr int RMS_CHUNKS = UPDATE_RMS_PARTIALS;

__global__ void __launch_bounds__(EW_THREADS) update_sq_kernel(const EwSeg* __restrict__ segs,
                                                               const float* __restrict__ o_scale,
                                                               double* __restrict__ part) {
    __shared__ double red[EW_THREADS / 32];
    pdl_trigger();
    pdl_wait();
    const EwSeg sg = segs[blockIdx.y];
    const int m = sg.transposed ? sg.cols : sg.rows, n = sg.transposed ? sg.rows : sg.cols;
    const float os = o_scale ? o_scale[sg.mat] : 1.0f;
    double acc = 0.0;
    // bf16 pair with 16-byte rows (ldn is a multiple of 8): 8 elements per load
    const bool vec = sg.o_hi != nullptr && sg.o_lo != nullptr && sg.ldn % 8 == 0;
    const int n8 = vec ? n / 8 : 0;
    for (int r = blockIdx.x; r < m; r += RMS_CHUNKS) {
        const size_t row = (size_t)r * sg.ldn;
        for (int c8 = threadIdx.x; c8 < n8; c8 += EW_THREADS) {
            const uint4 hv = __ldcs(reinterpret_cast<const uint4*>(sg.o_hi + row) + c8);
            const uint4 lv = __ldcs(reinterpret_cast<const uint4*>(sg.o_lo + row) + c8);
            const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w}, lw[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
            for (int t = 0; t < 4; ++t) {
                const float2 h2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&hw[t]));
                const float2 l2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&lw[t]));
                const double v0 = (double)((h2.x + l2.x) * os), v1 = (double)((h2.y + l2.y) * os);
                acc += v0 * v0;
                acc += v1 * v1;
            }
        }
        for (int c = 8 * n8 + threadIdx.x; c < n; c += EW_THREADS) {
            const double v = (double)(load_o(sg, row + c) * os);
            acc += v * v;
        }
    }
    const double tot = block_sum(acc, red);
    if (threadIdx.x == 0) part[(size_t)blockIdx.y * RMS_CHUNKS + blockIdx.x] = tot;
}

__global__ void __launch_bounds__(EW_THREADS) update_rms_finish_kernel(const EwSeg* __restrict__ segs,
                                                                       const double* __restrict__ part, float lr,
                                                                       float* __restrict__ rms) {
    __shared__ double red[EW_THREADS / 32];
    pdl_trigger();
    pdl_wait();
    const EwSeg sg = segs[blockIdx.x];
    const double v = block_sum(part[(size_t)blockIdx.x * RMS_CHUNKS + threadIdx.x], red);
    if (threadIdx.x == 0)
        rms[blockIdx.x] = (float)((double)lr * fabs((double)sg.update_scale) *
                                  sqrt(v / ((double)sg.rows * (double)sg.cols)));
}
static_assert(RMS_CHUNKS == EW_THREADS, "the finish kernel reduces one partial per thread");

}  // namespace

cudaError_t launch_update_rms(const EwSeg* segs, int nseg, const float* o_scale, float lr, double* part, float* rms,
                              cudaStream_t s) {
    if (nseg <= 0) return cudaSuccess;
    cudaError_t e = launch_pdl(update_sq_kernel, dim3(RMS_CHUNKS, nseg), dim3(EW_THREADS), 0, s, segs, o_scale, part);
    if (e != cudaSuccess) return e;
    return launch_pdl(update_rms_finish_kernel, dim3(nseg), dim3(EW_THREADS), 0, s, segs, (const double*)part, lr, rms);
}

cudaError_t launch_momentum_norm(const EwSeg* segs, int nseg, int nblocks, double* partials, float mu,
                                 int nesterov, int bf16_operand, int* counters, float eps, float* norms,
                                 float* scale, cudaStream_t s) {
    if (nblocks <= 0) return cudaSuccess;
    return launch_pdl(momentum_norm_kernel, dim3(nblocks), dim3(EW_THREADS), 0, s, segs, nseg, partials, mu, nesterov,
                      bf16_operand, counters, eps, norms, scale);
}

cudaError_t launch_apply(const EwSeg* segs, int nseg, int nblocks, float decay, float lr, const float* o_scale,
                         int copy_out, cudaStream_t s) {
    if (nblocks <= 0) return cudaSuccess;
    return launch_pdl(apply_kernel, dim3(nblocks), dim3(EW_THREADS), 0, s, segs, nseg, decay, lr, o_scale, copy_out);
}

cudaError_t launch_copy_out_one(const EwSeg& seg, float* dst, const float* o_scale, cudaStream_t s) {
    if (seg.apply_count <= 0) return cudaSuccess;
    EwSeg sg = seg;
    sg.out_bf16 = 0;                  // the destination of this copy is fp32
    if (reinterpret_cast<uintptr_t>(dst) % 16 != 0) sg.vec = 0;
    return launch_pdl(copy_out_one_kernel, dim3(sg.apply_count), dim3(EW_THREADS), 0, s, sg, dst, o_scale);
}

}  // namespace muon

// ---------------------------------------------------------------- QK-Clip
// After the Muon step, MuonClip rescales each attention head's rows of the query
// and key projections by sqrt(gamma_h), gamma_h = min(1, tau / S_h) for the head's
// maximum logit S_h (the Kimi K2 result of the Muon synthesis note), so every logit
// of the head scales by gamma_h.  One launch covers W_q and W_k; blockIdx.y picks
// the matrix.  Rows are grouped by head: head = row / head_dim.
namespace muon {
namespace {

__global__ void __launch_bounds__(EW_THREADS) qk_clip_kernel(float* __restrict__ wq, float* __restrict__ wk,
                                                            const float* __restrict__ max_logits, int head_dim,
                                                            int cols, size_t total, float tau, int vec) {
    pdl_trigger();
    pdl_wait();
    float* w = blockIdx.y == 0 ? wq : wk;
    if (w == nullptr) return;
    const size_t stride = (size_t)gridDim.x * EW_THREADS * (vec ? 4 : 1);
    for (size_t e = ((size_t)blockIdx.x * EW_THREADS + threadIdx.x) * (vec ? 4 : 1); e < total; e += stride) {
        const int head = (int)((e / (size_t)cols) / (size_t)head_dim);
        const float s = max_logits[head];
        const float f = s > tau ? sqrtf(tau / s) : 1.0f;
        if (f == 1.0f) continue;
        if (vec) {
            float4 x = *reinterpret_cast<float4*>(w + e);
            x.x *= f; x.y *= f; x.z *= f; x.w *= f;
            *reinterpret_cast<float4*>(w + e) = x;
        } else {
            w[e] *= f;
        }
    }
}

}  // namespace

cudaError_t launch_qk_clip(float* wq, float* wk, const float* max_logits, int n_heads, int head_dim, int cols,
                           float tau, int num_sms, cudaStream_t s) {
    const size_t total = (size_t)n_heads * head_dim * cols;
    if (total == 0) return cudaSuccess;
    const int vec = (cols % 4 == 0) && (reinterpret_cast<uintptr_t>(wq) % 16 == 0) &&
                    (wk == nullptr || reinterpret_cast<uintptr_t>(wk) % 16 == 0);
    const size_t work = vec ? total / 4 : total;
    const int blocks = (int)std::min<size_t>((work + EW_THREADS - 1) / EW_THREADS, (size_t)num_sms * 8);
    return launch_pdl(qk_clip_kernel, dim3(blocks, 2), dim3(EW_THREADS), 0, s, wq, wk, max_logits, head_dim, cols,
                      total, tau, vec);
}

}  // namespace muon
