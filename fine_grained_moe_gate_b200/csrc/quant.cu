// Per-tile E4M3 quantization ("DeepSeek V3 From Scratch", "The idea": FP8
// with fine-grained quantization tiles; crackai.dev "DeepSeek-V3", "How It
// Works": per-tile scaling; "DeepSeek V3 Architecture Deep Dive ...", "FP8
// Formats": E4M3 for weights and activations).
//
// A tile is 32 consecutive elements of a row along the contraction
// dimension.  Its scale is 2^e with e the smallest integer such that the
// tile's largest magnitude fits E4M3 (amax <= 448 * 2^e, so nothing
// saturates), kept as the byte e + 127 -- the unsigned power-of-two scale
// format the tensor cores' block-scaled MMA reads.  Codes are
// E4M3(v * 2^-e), round to nearest even; v * 2^-e is exact in fp32.
//
// e comes from the bits of amax (mx_tile_exponent, common.cuh); an all-zero
// tile gets e = 0 and codes 0.
//
// Scale layouts (the GEMMs' shared-memory scale atoms hold, for 128 operand
// rows and one 128-column stage, the byte of row m, tile j at
// (m % 32) * 16 + (m / 32) * 4 + j):
//   tokens:  uint32 [K/128][rows]: word (s, r) holds the 4 tile bytes of row
//            r's stage s (byte j = tile 4s + j).  A stage's words of
//            consecutive rows are contiguous, so a warp fetches 32 rows' with
//            one coalesced load, or gathers them by token index.
//   weights: 64-row half atoms of 256 bytes, [rows/64][K/128][32][8]: byte
//            (m % 32) * 8 + (m / 32) * 4 + j of half atom (r / 64, s), m =
//            r % 64.  A lane of the GEMM's scale warp copies 8 bytes per half
//            atom into the 16-byte row of the atom it builds.
// A matrix with `rows` rows may be stored as nseg column blocks of kseg
// columns ([nseg][rows][kseg], stacked experts joined along the
// contraction); its rows and tiles span all blocks.  One warp per row, one
// pass: each lane converts 8 elements, four lanes share a tile.
// HBM bound: 3 bytes per element (2 read, 1 written) + 1/32 per element.
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


template <bool kWeightLayout>
__global__ void __launch_bounds__(kWarps * 32) quantize_mx_kernel(const uint16_t* __restrict__ src, long long rows,
                                                                 int kseg, int nseg, uint8_t* __restrict__ q,
                                                                 uint8_t* __restrict__ sf) {
    const int lane = threadIdx.x & 31;
    const long long r = (long long)blockIdx.x * kWarps + (threadIdx.x >> 5);
    if (r >= rows) return;  // warp-uniform
    const int K = kseg * nseg;
    const int nst = K >> 7;  // 128-column stages
    for (int base = 0; base < K; base += 256) {
        const int c = base + lane * 8;
        const bool act = c < K;  // K % 128 == 0: whole 16-lane halves are active or not
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        size_t off = 0;
        if (act) {
            off = seg_offset(r, c, rows, kseg);
            const uint4 v = *reinterpret_cast<const uint4*>(src + off);
            w[0] = v.x;
            w[1] = v.y;
            w[2] = v.z;
            w[3] = v.w;
        }
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
        // the four lanes of a tile
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const int e = mx_tile_exponent(amax);
        const float mul = mx_inv_scale(e);  // 2^-e
        if (act) {
            uint32_t p[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                p[i] = e4m3x2(__fmul_rn(bf16_lo(w[i]), mul), __fmul_rn(bf16_hi(w[i]), mul));
            *reinterpret_cast<uint2*>(q + off) = make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
        }
        // gather the four tile bytes of this lane's 128-column stage into lane 16h (h = lane / 16)
        const uint32_t byte = (uint32_t)(e + 127);
        const uint32_t b1 = __shfl_down_sync(0xffffffffu, byte, 4);
        const uint32_t b2 = __shfl_down_sync(0xffffffffu, byte, 8);
        const uint32_t b3 = __shfl_down_sync(0xffffffffu, byte, 12);
        if (act && (lane & 15) == 0) {
            const uint32_t word = byte | (b1 << 8) | (b2 << 16) | (b3 << 24);
            const int s = c >> 7;
            if (kWeightLayout) {
                const size_t atom = ((size_t)(r >> 6) * nst + s) * 256;
                const int m = (int)(r & 63);
                *reinterpret_cast<uint32_t*>(sf + atom + (m & 31) * 8 + (m >> 5) * 4) = word;
            } else {
                reinterpret_cast<uint32_t*>(sf)[(size_t)s * rows + r] = word;
            }
        }
    }
}

// Token-layout scale words of the rows of a permutation: out[s][r] =
// xs[s][perm[r] / k] (row r of xq_perm holds token perm[r] / k), so that the
// GEMM reads a stage's words of consecutive rows with coalesced loads.
__global__ void permute_mx_scales_kernel(const uint32_t* __restrict__ xs, const int32_t* __restrict__ perm, int k,
                                         long long T, long long rows, int nst, uint32_t* __restrict__ out,
                                         int* status) {
    const long long n = rows * nst;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const int s = (int)(i / rows);
        const long long r = i - (long long)s * rows;
        const long long t = perm[r] / k;
        if (t < 0 || t >= T) {
            report(status, kStDeviceCheck);
            continue;
        }
        out[i] = xs[(size_t)s * T + t];
    }
}

}  // namespace

cudaError_t launch_permute_mx_scales(const void* xs, const int32_t* perm, int k, long long T, int K, void* out,
                                     int* status, cudaStream_t st) {
    const long long rows = T * k;
    const int nst = K / 128;
    if (rows <= 0 || nst <= 0) return cudaSuccess;
    const long long n = rows * nst;
    long long blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    permute_mx_scales_kernel<<<(unsigned)blocks, 256, 0, st>>>(static_cast<const uint32_t*>(xs), perm, k, T, rows, nst,
                                                               static_cast<uint32_t*>(out), status);
    note_launches(1);
    return cudaGetLastError();
}

size_t mx_scale_bytes(long long rows, int K, bool weight_layout) {
    const size_t nst = (size_t)(K / 128);
    if (weight_layout) return (size_t)((rows + 63) / 64) * nst * 256;
    return (size_t)rows * nst * 4;
}

cudaError_t launch_quantize_mx(const void* src, long long rows, int kseg, int nseg, bool weight_layout, uint8_t* q,
                               void* scales, cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    const long long blocks = (rows + kWarps - 1) / kWarps;
    if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
    const auto* s = static_cast<const uint16_t*>(src);
    auto* sf = static_cast<uint8_t*>(scales);
    if (weight_layout)
        quantize_mx_kernel<true><<<(unsigned)blocks, kWarps * 32, 0, st>>>(s, rows, kseg, nseg, q, sf);
    else
        quantize_mx_kernel<false><<<(unsigned)blocks, kWarps * 32, 0, st>>>(s, rows, kseg, nseg, q, sf);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
