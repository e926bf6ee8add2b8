// gemm_simt.cu -- fp32 FFMA GEMM for the fp32 debug precision of the
// Newton-Schulz iteration (section 4, eq. 4 of "Muon: An optimizer for hidden
// layers in neural networks").  No TF32: every product is an fp32 FMA, so the
// debug path sits within ~1e-5 of the fp64 oracle and isolates the bf16
// rounding of the tensor-core path.  Not a performance path.
//
// C[z] = alpha_eff * A[z] op(B[z]) + beta_eff * Cin[z], 64x64 output tile per
// block, 256 threads with a 4x4 register tile each, K staged 16 at a time.
#include "kernels.cuh"
#include "ptx.cuh"

namespace muon {
namespace {

constexpr int SB = 64, SK = 16;

__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtGemmArgs a) {
    __shared__ float As[SK][SB + 4];
    __shared__ float Bs[SK][SB + 4];
    pdl_trigger();
    pdl_wait();
    const int z = blockIdx.z;
    const int i0 = blockIdx.y * SB, j0 = blockIdx.x * SB;
    const float* A = a.A + (size_t)z * a.sA;
    const float* B = a.B + (size_t)z * a.sB;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < a.K; k0 += SK) {
        // A tile: 64 rows x 16 k (row-major A[i][k])
        for (int e = threadIdx.x; e < SB * SK; e += 256) {
            const int r = e / SK, k = e % SK;
            const int gi = i0 + r, gk = k0 + k;
            As[k][r] = (gi < a.M && gk < a.K) ? A[(size_t)gi * a.lda + gk] : 0.f;
        }
        for (int e = threadIdx.x; e < SB * SK; e += 256) {
            int c, k;
            if (a.b_kmajor) { c = e / SK; k = e % SK; } else { k = e / SB; c = e % SB; }
            const int gj = j0 + c, gk = k0 + k;
            float v = 0.f;
            if (gj < a.N && gk < a.K) v = a.b_kmajor ? B[(size_t)gj * a.ldb + gk] : B[(size_t)gk * a.ldb + gj];
            Bs[k][c] = v;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < SK; ++k) {
            float av[4], bv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) { av[u] = As[k][ty * 4 + u]; bv[u] = Bs[k][tx * 4 + u]; }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
        }
        __syncthreads();
    }
    float alpha = a.alpha, beta = a.beta;
    if (a.scale) {
        const float s = a.scale[a.mat_base + z];
        float sp = 1.f;
        for (int t = 0; t < a.scale_pow; ++t) sp *= s;
        alpha *= sp;
        beta *= sp;
    }
    float* C = a.C + (size_t)z * a.sC;
    const float* Cin = a.Cin ? a.Cin + (size_t)z * a.sCin : nullptr;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int gi = i0 + ty * 4 + u;
        if (gi >= a.M) continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int gj = j0 + tx * 4 + v;
            if (gj >= a.N) continue;
            float r = alpha * acc[u][v];
            if (Cin) r = fmaf(beta, Cin[(size_t)gi * a.ldcin + gj], r);
            C[(size_t)gi * a.ldc + gj] = r;
        }
    }
}

}  // namespace

cudaError_t launch_simt_gemm(const SimtGemmArgs& a, cudaStream_t s) {
    if (a.M <= 0 || a.N <= 0 || a.count <= 0) return cudaSuccess;
    dim3 grid((a.N + SB - 1) / SB, (a.M + SB - 1) / SB, a.count);
    return launch_pdl(simt_gemm_kernel, grid, dim3(256), 0, s, a);
}

}  // namespace muon
