// gemm_tc.cu -- the Newton-Schulz GEMMs on the sm_100a tensor cores.
//
// One quintic step X <- aX + b(XX^T)X + c(XX^T)^2 X ("Muon: An optimizer for
// hidden layers in neural networks", section 4, eqs. 4-5) is run as three
// grouped, persistent GEMM launches over every matrix of the step:
//
//   GRAM    A  = alpha * X X^T            (upper-triangle tiles, mirrored)
//   POLY    P  = b*A + c * A A            (A symmetric: A A = A A^T; upper tiles, mirrored)
//   UPDATE  X' = alpha * P X + beta * X   (the aX term in the epilogue, X read in fp32)
//
// On the first step alpha/beta absorb the Frobenius normalisation s = 1/(||U||+eps):
// A0 = s^2 UU^T and X1 = s P U + a s U.
//
// Kernel structure (one CTA per SM, 320 threads):
//   warp 0      TMA producer: 4-stage ring of (128x64 A-operand, 256x64 B-operand)
//               bf16 tiles in 128-byte-swizzled shared memory, plain (non-multicast)
//               3-D tiled loads, zero fill outside the matrix.
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators) and
//               issues tcgen05.mma kind::f16 (M=128, N=256, K=16) from one thread;
//               tcgen05.commit frees ring slots and publishes finished accumulators.
//   warps 2-9   epilogue: tcgen05.ld of the accumulator (each warp owns the 32 TMEM
//               lanes its rank allows and half of the columns), scale, add the
//               residual term, round, store; mirrored stores for the symmetric outputs.
// The double-buffered accumulator lets the epilogue of tile i overlap the
// main loop of tile i+1.  Tiles are taken round-robin from a cost-sorted list
// that spans all matrices of the call, so many small matrices fill the 148 SMs.
#include "kernels.cuh"
#include "ptx.cuh"

namespace muon {
namespace {

constexpr int BM = TC_BM, BN = TC_BN, BK = TC_BK;
constexpr int STAGES = 4;
constexpr int A_STAGE = BM * BK * 2;      // 16 KiB
constexpr int B_STAGE = BN * BK * 2;      // 32 KiB
constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr int TMEM_COLS = 2 * BN;          // two accumulators
constexpr int SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + 256 /*barriers*/;

// error codes written to the device error word when a bounded wait gives up
constexpr int ERR_PRODUCER = 0x101, ERR_MMA_SLOT = 0x102, ERR_MMA_ACC = 0x103, ERR_EPILOGUE = 0x104;

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_bits_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_bits_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Epilogue of one 32-column chunk of one output row for the symmetric outputs
// (GRAM and POLY).  val[] holds the finished fp32 values of columns col0..col0+31.
// Element (row, c) is stored directly when c >= row and mirrored to (c, row) when
// c > row, so every element of the m x m output is written exactly once.
__device__ __forceinline__ void store_symmetric(__nv_bfloat16* __restrict__ out, int m, int ldm,
                                                int row, int col0, const float (&val)[32]) {
    if (row >= m) return;
    if (col0 >= row && col0 + 31 < m) {
        uint4* dst = reinterpret_cast<uint4*>(out + (size_t)row * ldm + col0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint4 w;
            w.x = pack_bf16x2(val[8 * q + 0], val[8 * q + 1]);
            w.y = pack_bf16x2(val[8 * q + 2], val[8 * q + 3]);
            w.z = pack_bf16x2(val[8 * q + 4], val[8 * q + 5]);
            w.w = pack_bf16x2(val[8 * q + 6], val[8 * q + 7]);
            dst[q] = w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            const int c = col0 + j;
            if (c >= row && c < m) out[(size_t)row * ldm + c] = __float2bfloat16_rn(val[j]);
        }
    }
    // mirror: lanes hold consecutive rows, so each store instruction of the warp
    // writes 32 consecutive elements of row c.
#pragma unroll
    for (int j = 0; j < 32; ++j) {
        const int c = col0 + j;
        if (c > row && c < m) out[(size_t)c * ldm + row] = __float2bfloat16_rn(val[j]);
    }
}

template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1) ns_gemm_tc_kernel(const __grid_constant__ GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_STAGE;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + 2;
    uint64_t* drain = tempty + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const uint32_t warp = warp_id();
    const uint32_t lane = threadIdx.x & 31u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
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

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (elect_one()) {
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < p.ntiles && ok; t += gridDim.x) {
                const int4 tile = p.tiles[t];
                const GemmGroupInfo& gi = p.groups[tile.x];
                const GemmMaps* mp = p.maps + tile.x;
                const int K = (MODE == MODE_GRAM) ? gi.n : gi.m;
                const int kblocks = (K + BK - 1) / BK;
                const void* mapA = (MODE == MODE_GRAM) ? (const void*)&mp->xb_k[p.parity]
                                 : (MODE == MODE_POLY) ? (const void*)&mp->a : (const void*)&mp->p;
                const void* mapB = (MODE == MODE_GRAM) ? (const void*)&mp->xb_k[p.parity]
                                 : (MODE == MODE_POLY) ? (const void*)&mp->a : (const void*)&mp->xb_mn[p.parity];
                const int row0 = tile.z * BM, col0 = tile.w * BN, mat = tile.y;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err, ERR_PRODUCER)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
                    const int k0 = kb * BK;
                    uint8_t* a_dst = sA + stage * A_STAGE;
                    uint8_t* b_dst = sB + stage * B_STAGE;
                    tma_load_3d(a_dst, mapA, &full[stage], k0, row0, mat);
                    if (MODE == MODE_UPDATE) {
                        // B = X rows k0..k0+63, columns col0..col0+255, as four 64-column boxes
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            tma_load_3d(b_dst + c * (BK * 128), mapB, &full[stage], col0 + 64 * c, k0, mat);
                    } else {
                        tma_load_3d(b_dst, mapB, &full[stage], k0, col0, mat);
                        tma_load_3d(b_dst + 128 * 128, mapB, &full[stage], k0, col0 + 128, mat);
                    }
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
            }
            if (!ok || *abort_flag) {
                // let any load still in flight land before the CTA retires
                const uint64_t t0 = globaltimer_ns();
                while (globaltimer_ns() - t0 < 2000000ull) { }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (elect_one()) {
            constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, MODE == MODE_UPDATE ? 1u : 0u);
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
                const uint32_t d_tmem = tmem_base + acc * BN;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&full[stage], phase, abort_flag, p.err, ERR_MMA_SLOT)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA + stage * A_STAGE);
                    const uint32_t b_base = smem_u32(sB + stage * B_STAGE);
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
                    if (++stage == STAGES) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&tfull[acc]);
            }
            if (!ok || *abort_flag) {
                // wait (bounded) until every MMA issued so far has finished
                tc_commit(drain);
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < 100000000ull) { }
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const uint32_t q = warp & 3u;                 // TMEM lane quarter this warp may access
        const uint32_t half = (warp - 2) >> 2;        // column half of the tile
        int local = 0;
        for (int t = blockIdx.x; t < p.ntiles; t += gridDim.x, ++local) {
            const int4 tile = p.tiles[t];
            const GemmGroupInfo& gi = p.groups[tile.x];
            const uint32_t acc = local & 1;
            const uint32_t acc_phase = (local >> 1) & 1;
            bool ok = mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err, ERR_EPILOGUE);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();

            const int mat = tile.y;
            const int row = tile.z * BM + (int)(q * 32 + lane);
            float alpha = p.alpha, beta = p.beta;
            if (p.scale != nullptr) {
                const float s = p.scale[gi.mat_base + mat];
                if (MODE == MODE_GRAM) alpha = p.alpha * s * s;
                if (MODE == MODE_UPDATE) { alpha = p.alpha * s; beta = p.beta * s; }
            }
#pragma unroll 1
            for (int chunk = 0; chunk < 4; ++chunk) {
                const int c_local = (int)half * 128 + chunk * 32;
                uint32_t v[32];
                tmem_ld_32x32b_x32(tmem_base + acc * BN + ((q * 32u) << 16) + (uint32_t)c_local, v);
                tmem_ld_wait();
                const int col0 = tile.w * BN + c_local;
                float val[32];
                if (MODE == MODE_GRAM) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) val[j] = alpha * __uint_as_float(v[j]);
                    store_symmetric(gi.a + (size_t)mat * gi.m * gi.ldm, gi.m, gi.ldm, row, col0, val);
                } else if (MODE == MODE_POLY) {
                    const __nv_bfloat16* A = gi.a + (size_t)mat * gi.m * gi.ldm;
                    if (row < gi.m && col0 + 31 < gi.m) {
                        const uint4* src = reinterpret_cast<const uint4*>(A + (size_t)row * gi.ldm + col0);
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq) {
                            const uint4 w = src[qq];
                            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                val[8 * qq + 2 * e] = alpha * __uint_as_float(v[8 * qq + 2 * e]) + beta * bf16_bits_lo(ws[e]);
                                val[8 * qq + 2 * e + 1] = alpha * __uint_as_float(v[8 * qq + 2 * e + 1]) + beta * bf16_bits_hi(ws[e]);
                            }
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const int c = col0 + j;
                            const float av = (row < gi.m && c < gi.m) ? __bfloat162float(A[(size_t)row * gi.ldm + c]) : 0.f;
                            val[j] = alpha * __uint_as_float(v[j]) + beta * av;
                        }
                    }
                    store_symmetric(gi.p + (size_t)mat * gi.m * gi.ldm, gi.m, gi.ldm, row, col0, val);
                } else {
                    if (row < gi.m) {
                        const size_t off = (size_t)mat * gi.m * gi.ldn + (size_t)row * gi.ldn;
                        const float* xin = gi.xf_in + off;
                        float* xout = gi.xf_out + off;
                        __nv_bfloat16* xb = gi.xb[p.parity ^ 1] + off;
                        if (col0 + 31 < gi.n) {
                            const float4* src = reinterpret_cast<const float4*>(xin + col0);
#pragma unroll
                            for (int qq = 0; qq < 8; ++qq) {
                                const float4 x = src[qq];
                                val[4 * qq + 0] = alpha * __uint_as_float(v[4 * qq + 0]) + beta * x.x;
                                val[4 * qq + 1] = alpha * __uint_as_float(v[4 * qq + 1]) + beta * x.y;
                                val[4 * qq + 2] = alpha * __uint_as_float(v[4 * qq + 2]) + beta * x.z;
                                val[4 * qq + 3] = alpha * __uint_as_float(v[4 * qq + 3]) + beta * x.w;
                            }
                            float4* dst = reinterpret_cast<float4*>(xout + col0);
#pragma unroll
                            for (int qq = 0; qq < 8; ++qq)
                                dst[qq] = make_float4(val[4 * qq], val[4 * qq + 1], val[4 * qq + 2], val[4 * qq + 3]);
                            if (p.write_op) {
                                uint4* db = reinterpret_cast<uint4*>(xb + col0);
#pragma unroll
                                for (int qq = 0; qq < 4; ++qq) {
                                    uint4 w;
                                    w.x = pack_bf16x2(val[8 * qq + 0], val[8 * qq + 1]);
                                    w.y = pack_bf16x2(val[8 * qq + 2], val[8 * qq + 3]);
                                    w.z = pack_bf16x2(val[8 * qq + 4], val[8 * qq + 5]);
                                    w.w = pack_bf16x2(val[8 * qq + 6], val[8 * qq + 7]);
                                    db[qq] = w;
                                }
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j) {
                                const int c = col0 + j;
                                if (c < gi.n) {
                                    const float r = alpha * __uint_as_float(v[j]) + beta * xin[c];
                                    xout[c] = r;
                                    if (p.write_op) xb[c] = __float2bfloat16_rn(r);
                                }
                            }
                        }
                    }
                }
            }
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

}  // namespace

size_t tc_gemm_smem_bytes() { return SMEM_BYTES; }
int tc_gemm_threads() { return NUM_THREADS; }

cudaError_t tc_gemm_prepare() {
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(ns_gemm_tc_kernel<MODE_GRAM>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(ns_gemm_tc_kernel<MODE_POLY>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) != cudaSuccess) return e;
    return cudaFuncSetAttribute(ns_gemm_tc_kernel<MODE_UPDATE>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
}

cudaError_t launch_tc_gemm(int mode, const GemmParams& p, int grid, cudaStream_t s) {
    if (p.ntiles <= 0) return cudaSuccess;
    switch (mode) {
        case MODE_GRAM: ns_gemm_tc_kernel<MODE_GRAM><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(p); break;
        case MODE_POLY: ns_gemm_tc_kernel<MODE_POLY><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(p); break;
        default: ns_gemm_tc_kernel<MODE_UPDATE><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(p); break;
    }
    return cudaGetLastError();
}

}  // namespace muon
