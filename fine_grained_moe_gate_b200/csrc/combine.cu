// Weighted combine back into token order ("Scaling Efficiency: A Deep Dive
// into the DeepSeek-V3 Architecture", DeepSeekMoE sketch: each routed
// expert's output scaled by its gate weight and added to the token, plus the
// shared experts' output):
//   y[t] = shared[t] + sum_j w[t][j] * y_perm[inv_row[t*k + j]]
// fp32 accumulation in that fixed order (deterministic), one rounding to the
// output type.  One CTA per token, 16-byte vector loads.  HBM bound:
// (k + 1) rows read and one written per token.
#include "common.cuh"
#include "kernels.h"

namespace moe {

template <typename T>
struct Vec;
template <>
struct Vec<float> {
    static constexpr int n = 4;
    __device__ static void unpack(const uint4& u, float* f) {
        f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
        f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
    }
    __device__ static uint4 pack(const float* f) {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
    }
};
template <>
struct Vec<__nv_bfloat16> {
    static constexpr int n = 8;
    __device__ static void unpack(const uint4& u, float* f) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ static uint4 pack(const float* f) {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<const uint32_t*>(&b);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

// The k rows' vectors are all loaded before the sum (KMAX-wide, predicated),
// so each thread keeps k loads in flight instead of one.
template <typename T, int KMAX>
__global__ void combine_kernel(const uint4* __restrict__ y_perm, const float* __restrict__ w,
                               const int32_t* __restrict__ inv_row, const uint4* __restrict__ shared, int k,
                               int vec_per_row, int total_rows, uint4* __restrict__ y, int* status) {
    constexpr int n = Vec<T>::n;
    const int t = blockIdx.x;
    __shared__ int rows[KMAX];
    __shared__ float ws[KMAX];
    if (threadIdx.x < k) {
        int r = inv_row[(size_t)t * k + threadIdx.x];
        if ((unsigned)r >= (unsigned)total_rows) {
            report(status, kStDeviceCheck);
            r = -1;
        }
        rows[threadIdx.x] = r;
        ws[threadIdx.x] = w[(size_t)t * k + threadIdx.x];
    }
    __syncthreads();
    for (int v = threadIdx.x; v < vec_per_row; v += blockDim.x) {
        uint4 in[KMAX];
#pragma unroll
        for (int j = 0; j < KMAX; ++j)
            if (j < k && rows[j] >= 0) in[j] = y_perm[(size_t)rows[j] * vec_per_row + v];
        float acc[n], tmp[n];
        if (shared) {
            Vec<T>::unpack(shared[(size_t)t * vec_per_row + v], acc);
        } else {
#pragma unroll
            for (int i = 0; i < n; ++i) acc[i] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            if (j < k && rows[j] >= 0) {
                Vec<T>::unpack(in[j], tmp);
                const float wj = ws[j];
#pragma unroll
                for (int i = 0; i < n; ++i) acc[i] = fmaf(wj, tmp[i], acc[i]);
            }
        }
        y[(size_t)t * vec_per_row + v] = Vec<T>::pack(acc);
    }
}

template <typename T>
void launch_t(const void* y_perm, const float* w, const int32_t* inv_row, const void* shared, int T_, int k, int vec,
              void* y, int* status, cudaStream_t st) {
    // threads: a multiple of 32 that divides the row's vectors when one does (no idle tail pass)
    int threads = 256;
    for (int c = 256; c >= 96; c -= 32)
        if (vec % c == 0) {
            threads = c;
            break;
        }
    if (vec < 256) threads = ((vec + 31) / 32) * 32;
    const uint4* yp = static_cast<const uint4*>(y_perm);
    const uint4* sh = static_cast<const uint4*>(shared);
    uint4* out = static_cast<uint4*>(y);
    if (k <= 8)
        combine_kernel<T, 8><<<T_, threads, 0, st>>>(yp, w, inv_row, sh, k, vec, T_ * k, out, status);
    else
        combine_kernel<T, 16><<<T_, threads, 0, st>>>(yp, w, inv_row, sh, k, vec, T_ * k, out, status);
}

// Finish of the combine fused into the down projection's epilogue: the fp32
// accumulator holds shared[t] + sum_j w[t][j] * o_j (added tile by tile), so
// y = dtype(acc), one rounding; acc is then cleared for the next
// accumulation.  Eight elements per thread and step (two 16-byte loads, one
// or two 16-byte stores, two zero stores).  HBM bound: 4 + 4 + 2 (or 4)
// bytes per element.
template <typename T>
__global__ void __launch_bounds__(256) combine_finish_kernel(float4* __restrict__ acc, long long n8,
                                                             uint4* __restrict__ y) {
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (long long)gridDim.x * blockDim.x) {
        const float4 a = acc[2 * i], b = acc[2 * i + 1];
        acc[2 * i] = zero;
        acc[2 * i + 1] = zero;
        const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        if constexpr (Vec<T>::n == 8) {
            y[i] = Vec<T>::pack(f);
        } else {
            y[2 * i] = Vec<T>::pack(f);
            y[2 * i + 1] = Vec<T>::pack(f + 4);
        }
    }
}

cudaError_t launch_combine_finish(float* acc, long long n, bool bf16, void* y, cudaStream_t st) {
    if (n <= 0) return cudaSuccess;
    const long long n8 = n / 8;
    const long long blocks = (n8 + 255) / 256 < 148 * 16 ? (n8 + 255) / 256 : 148 * 16;
    if (bf16)
        combine_finish_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<float4*>(acc), n8,
                                                                              static_cast<uint4*>(y));
    else
        combine_finish_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<float4*>(acc), n8,
                                                                      static_cast<uint4*>(y));
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_combine(const void* y_perm, const float* w, const int32_t* inv_row, const void* shared, int T,
                           int d, int k, bool bf16, void* y, int* status, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const size_t eb = bf16 ? 2 : 4;
    const int vec = (int)((size_t)d * eb / 16);
    if (bf16)
        launch_t<__nv_bfloat16>(y_perm, w, inv_row, shared, T, k, vec, y, status, st);
    else
        launch_t<float>(y_perm, w, inv_row, shared, T, k, vec, y, status, st);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
