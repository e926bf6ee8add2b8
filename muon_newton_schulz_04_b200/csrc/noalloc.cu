// noalloc.cu -- momentum + Nesterov direction + Frobenius norm of one matrix,
// for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: a runtime that owns a fixed device
// memory pool and forbids outside allocations, code that runs while another
// component holds the allocator, or a process whose device memory is already
// spoken for.  For them this file offers one entry point that allocates nothing.
// The only scratch it needs -- one fp64 partial sum of squares per block of 8192
// elements -- lives in the file-scope array below, which the CUDA runtime places
// in device memory when the library's module is loaded on a device; every GPU
// that loads the library holds it until the process exits.
//
// The array's name in host code is a host-side stand-in, not a device address,
// so every call looks the address up with cudaGetSymbolAddress (with the device
// current) and passes it to the kernels.  The lookup is not cached: after a
// cudaDeviceReset or a new primary context the module is loaded again, possibly at
// another address.
#include <cuda_runtime.h>

#include <cstdio>

#include "../../include/muon.h"
#include "kernels.cuh"

namespace muon {
namespace {

constexpr int NA_THREADS = 256;
constexpr int NA_ELEMS_PER_BLOCK = 8192;   // 256 threads x 8 elements x 4 rounds

static __device__ __align__(256) double g_noalloc_partials[MUON_NOALLOC_MAX_BLOCKS];


__device__ __forceinline__ double na_block_sum(double v, double* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    double r = 0.0;
    if (threadIdx.x == 0)
        for (int i = 0; i < NA_THREADS / 32; ++i) r += red[i];
    return r;
}

__device__ __forceinline__ float na_load(const void* g, size_t i, int bf16) {
    return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(g)[i]) : reinterpret_cast<const float*>(g)[i];
}

// B <- mu B + G;  U = G + mu B (Nesterov) or B;  partials[block] = sum of U^2 over the block.
__global__ void __launch_bounds__(NA_THREADS) momentum_norm_noalloc_kernel(const void* __restrict__ g, int g_bf16,
                                                                          float* __restrict__ b, float* __restrict__ u_out,
                                                                          size_t total, float mu, int nesterov,
                                                                          double* __restrict__ partials) {
    __shared__ double red[NA_THREADS / 32];
    const size_t e0 = (size_t)blockIdx.x * NA_ELEMS_PER_BLOCK;
    const size_t e1 = min(total, e0 + NA_ELEMS_PER_BLOCK);
    double acc = 0.0;
    for (size_t e = e0 + threadIdx.x; e < e1; e += NA_THREADS) {
        const float gv = na_load(g, e, g_bf16);
        const float bn = fmaf(mu, b[e], gv);
        b[e] = bn;
        const float u = nesterov ? fmaf(mu, bn, gv) : bn;
        if (u_out) u_out[e] = u;
        acc += (double)u * (double)u;
    }
    const double t = na_block_sum(acc, red);
    if (threadIdx.x == 0) partials[blockIdx.x] = t;
}

// norm = sqrt(sum of the partials), summed in a fixed order.
__global__ void __launch_bounds__(NA_THREADS) norm_noalloc_kernel(const double* __restrict__ partials, int nblocks,
                                                                 float* __restrict__ norm_out) {
    __shared__ double red[NA_THREADS / 32];
    double s = 0.0;
    for (int i = threadIdx.x; i < nblocks; i += NA_THREADS) s += partials[i];
    const double t = na_block_sum(s, red);
    if (threadIdx.x == 0) *norm_out = (float)sqrt(t);
}

void put_msg(char* buf, int cap, const char* msg) {
    if (buf && cap > 0) snprintf(buf, (size_t)cap, "%s", msg);
}

// [a, a + na) and [b, b + nb) share at least one byte.
bool spans_overlap(const void* a, size_t na, const void* b, size_t nb) {
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" muon_status muon_momentum_norm_noalloc(int rows, int cols, int grad_dtype, const void* G, float* B,
                                                  float* U_out, float momentum, int nesterov, float* norm_out,
                                                  void* stream, char* err_msg, int err_cap) {
    put_msg(err_msg, err_cap, "");
    if (rows <= 0 || cols <= 0) { put_msg(err_msg, err_cap, "rows and cols must be > 0"); return MUON_ERR_INVALID; }
    if (grad_dtype != MUON_BF16 && grad_dtype != MUON_FP32) { put_msg(err_msg, err_cap, "bad grad_dtype"); return MUON_ERR_INVALID; }
    if (!G || !B || !norm_out) { put_msg(err_msg, err_cap, "G, B and norm_out are required"); return MUON_ERR_INVALID; }
    if (!(momentum >= 0.f && momentum < 1.f)) { put_msg(err_msg, err_cap, "momentum must be in [0, 1)"); return MUON_ERR_INVALID; }
    if (nesterov != 0 && nesterov != 1) { put_msg(err_msg, err_cap, "nesterov must be 0 or 1"); return MUON_ERR_INVALID; }
    const size_t total = (size_t)rows * (size_t)cols;
    const size_t nblocks = (total + NA_ELEMS_PER_BLOCK - 1) / NA_ELEMS_PER_BLOCK;
    if (nblocks > (size_t)MUON_NOALLOC_MAX_BLOCKS) {
        char msg[160];
        snprintf(msg, sizeof msg, "matrix of %zu elements exceeds the no-allocation limit of %llu elements", total,
                 (unsigned long long)MUON_NOALLOC_MAX_BLOCKS * NA_ELEMS_PER_BLOCK);
        put_msg(err_msg, err_cap, msg);
        return MUON_ERR_UNSUPPORTED;
    }
    // B and U_out are written (and declared __restrict__ in the kernel): neither may
    // share memory with another buffer of the call; the one-float norm neither
    const size_t gbytes = total * (grad_dtype == MUON_BF16 ? 2 : 4), fbytes = total * 4;
    if (spans_overlap(B, fbytes, G, gbytes) || (U_out && (spans_overlap(U_out, fbytes, G, gbytes) ||
                                                          spans_overlap(U_out, fbytes, B, fbytes))) ||
        spans_overlap(norm_out, 4, G, gbytes) || spans_overlap(norm_out, 4, B, fbytes) ||
        (U_out && spans_overlap(norm_out, 4, U_out, fbytes))) {
        put_msg(err_msg, err_cap, "B, U_out and norm_out are written: they may not overlap each other or G");
        return MUON_ERR_INVALID;
    }
    void* p = nullptr;
    {
        const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_partials);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            put_msg(err_msg, err_cap, "cudaGetSymbolAddress of the static scratch failed");
            return MUON_ERR_CUDA;
        }
    }
    double* scratch = static_cast<double*>(p);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    momentum_norm_noalloc_kernel<<<(unsigned)nblocks, NA_THREADS, 0, s>>>(G, grad_dtype == MUON_BF16 ? 1 : 0, B, U_out,
                                                                         total, momentum, nesterov, scratch);
    norm_noalloc_kernel<<<1, NA_THREADS, 0, s>>>(scratch, (int)nblocks, norm_out);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        put_msg(err_msg, err_cap, cudaGetErrorString(e));
        return MUON_ERR_CUDA;
    }
    return MUON_OK;
}
