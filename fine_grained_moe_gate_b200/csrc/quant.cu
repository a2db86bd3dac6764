// Per-row E4M3 quantization ("DeepSeek V3 Architecture Deep Dive ...",
// "FP8 Formats": E4M3 for weights and activations; "Per-Tensor/Per-Axis
// Quantization": one scale per row/channel).
//
//   scale_r = amax_r / 448, inv_r = 448 / amax_r (fp32, IEEE division, once
//   per row; an all-zero row gets scale 1 and codes 0)
//   q[r][c] = E4M3(src[r][c] * inv_r), round to nearest even, saturating
//
// A matrix with `rows` rows may be stored as nseg column blocks of kseg
// columns ([nseg][rows][kseg], stacked experts joined along the contraction);
// its rows span all blocks.  One warp per row, two passes over the row (the
// second one from L1/L2): 16-byte loads of 8 bf16, 8-byte stores of 8 codes.
// HBM bound: 3 bytes per element (2 read, 1 written) + 4 per row.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ size_t seg_offset(long long r, int c, long long rows, int kseg) {
    const int s = c / kseg;
    return (size_t)s * (size_t)rows * kseg + (size_t)r * kseg + (size_t)(c - s * kseg);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Two codes, a in the low byte (the lower address once stored).
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
}

__global__ void __launch_bounds__(kWarps * 32) quantize_e4m3_kernel(const uint16_t* __restrict__ src, long long rows,
                                                                   int kseg, int nseg, uint8_t* __restrict__ q,
                                                                   float* __restrict__ scale) {
    const int lane = threadIdx.x & 31;
    const long long r = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int K = kseg * nseg;
    float amax = 0.0f;
    for (int c = lane * 8; c < K; c += 256) {
        const uint4 v = *reinterpret_cast<const uint4*>(src + seg_offset(r, c, rows, kseg));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
    const float inv = amax > 0.0f ? __fdiv_rn(448.0f, amax) : 0.0f;
    if (lane == 0) scale[r] = sc;
    for (int c = lane * 8; c < K; c += 256) {
        const size_t off = seg_offset(r, c, rows, kseg);
        const uint4 v = *reinterpret_cast<const uint4*>(src + off);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            p[i] = e4m3x2(__fmul_rn(bf16_lo(w[i]), inv), __fmul_rn(bf16_hi(w[i]), inv));
        // element order in memory: low byte first
        *reinterpret_cast<uint2*>(q + off) = make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
    }
}

}  // namespace

cudaError_t launch_quantize_e4m3(const void* src, long long rows, int kseg, int nseg, uint8_t* q, float* scale,
                                 cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    const long long blocks = (rows + kWarps - 1) / kWarps;
    if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
    quantize_e4m3_kernel<<<(unsigned)blocks, kWarps * 32, 0, st>>>(static_cast<const uint16_t*>(src), rows, kseg,
                                                                   nseg, q, scale);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
