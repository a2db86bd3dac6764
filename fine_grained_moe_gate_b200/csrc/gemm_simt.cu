// SIMT grouped GEMM for the fp32 layer (tensor-core TF32 cannot meet the
// fp32 layer's 1e-5 bound).  C = A . B^T per group, fp32 FFMA accumulation.
//   up   (SwiGLU epilogue):  h = silu(A . W1^T) * (A . W3^T)
//   down (plain epilogue):   y = A . W2^T
// Group g owns rows [off(g), off(g+1)) of A and C, and B block g.  Groups
// and tiles are resolved on the device from the offsets array, so no host
// read-back of the routing is needed.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kSm = 64, kSn = 64, kSk = 16;

template <typename T, bool SWIGLU>
__global__ void __launch_bounds__(256) simt_grouped_gemm_kernel(GemmArgs p) {
    __shared__ float As[kSk][kSm + 4];
    __shared__ float Bs[kSk][kSn + 4];
    __shared__ float B3s[SWIGLU ? kSk : 1][kSn + 4];
    __shared__ int tile_prefix[kMaxGroups + 1];
    __shared__ int mtiles[kMaxGroups];

    const int G = p.G;
    const int n_tiles = (p.N + kSn - 1) / kSn;
    // per-group m-tile counts and prefix of tile counts
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        int rows = p.M;
        if (p.offsets) {
            const int rs = p.offsets[g], re = p.offsets[g + 1];
            rows = re - rs;
            if (rs < 0 || rows < 0 || re > p.M) rows = 0;  // corrupt offsets: skip (the permute pass reports)
        }
        mtiles[g] = (rows + kSm - 1) / kSm;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int g = 0; g < G; ++g) {
            tile_prefix[g] = acc;
            acc += mtiles[g] * n_tiles;
        }
        tile_prefix[G] = acc;
    }
    __syncthreads();
    const int total = tile_prefix[G];
    const T* A = static_cast<const T*>(p.A);
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;

    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        int lo = 0, hi = G - 1;
        while (lo < hi) {  // last g with tile_prefix[g] <= tile
            const int mid = (lo + hi + 1) >> 1;
            if (tile_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
        }
        const int g = lo;
        const int q = tile - tile_prefix[g];
        const int mt = mtiles[g];
        const int n0 = (q / mt) * kSn;
        const int m0 = (q % mt) * kSm;
        const int row0 = p.offsets ? p.offsets[g] : 0;
        const int Mg = mtiles[g] == 0 ? 0 : (p.offsets ? (p.offsets[g + 1] - row0) : p.M);
        const T* B0 = static_cast<const T*>(p.B0) + (size_t)g * p.b_gstride;
        const T* B1 = SWIGLU ? static_cast<const T*>(p.B1) + (size_t)g * p.b_gstride : nullptr;

        float acc[4][4], acc3[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = acc3[i][j] = 0.f;

        for (int k0 = 0; k0 < p.K; k0 += kSk) {
            __syncthreads();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int qq = threadIdx.x * 4 + i;
                const int r = qq / kSk, kk = qq % kSk;
                const int kg = k0 + kk;
                float va = 0.f, vb = 0.f, v3 = 0.f;
                if (kg < p.K) {
                    if (m0 + r < Mg) {
                        const int ar = p.gather ? p.gather[row0 + m0 + r] / p.gather_div : row0 + m0 + r;
                        va = to_f32(A[(size_t)ar * p.lda + kg]);
                    }
                    if (n0 + r < p.N) {
                        const size_t boff = (size_t)(kg / p.kseg) * p.seg_stride + (size_t)(n0 + r) * p.ldb +
                                            (size_t)(kg % p.kseg);
                        vb = to_f32(B0[boff]);
                        if (SWIGLU) v3 = to_f32(B1[boff]);
                    }
                }
                As[kk][r] = va;
                Bs[kk][r] = vb;
                if (SWIGLU) B3s[kk][r] = v3;
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < kSk; ++kk) {
                float a[4], b[4], b3[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    a[i] = As[kk][ty * 4 + i];
                    b[i] = Bs[kk][tx * 4 + i];
                    if (SWIGLU) b3[i] = B3s[kk][tx * 4 + i];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
                        if (SWIGLU) acc3[i][j] = fmaf(a[i], b3[j], acc3[i][j]);
                    }
            }
        }
        T* C = static_cast<T*>(p.C);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = m0 + ty * 4 + i;
            if (r >= Mg) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int n = n0 + tx * 4 + j;
                if (n >= p.N) continue;
                const float v = SWIGLU ? silu_f32(acc[i][j]) * acc3[i][j] : acc[i][j];
                store_f32(&C[(size_t)(row0 + r) * p.ldc + n], v);
            }
        }
    }
}

cudaError_t launch_simt_gemm(const GemmArgs& p, bool bf16, bool swiglu, int num_sms, cudaStream_t st) {
    if (p.G <= 0 || p.G > kMaxGroups) return cudaErrorInvalidValue;
    const int grid = num_sms * 4;
    if (bf16) {
        if (swiglu) simt_grouped_gemm_kernel<__nv_bfloat16, true><<<grid, 256, 0, st>>>(p);
        else simt_grouped_gemm_kernel<__nv_bfloat16, false><<<grid, 256, 0, st>>>(p);
    } else {
        if (swiglu) simt_grouped_gemm_kernel<float, true><<<grid, 256, 0, st>>>(p);
        else simt_grouped_gemm_kernel<float, false><<<grid, 256, 0, st>>>(p);
    }
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
