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
// Scale layouts (the GEMMs' scale atoms hold, for 128 operand rows and one
// 128-column stage, the byte of row m, tile j at (m % 32) * 16 + (m / 32) * 4
// + j: the order the tensor-memory scale copy reads them):
//   tokens:  uint32 [K/128][rows]: word (s, r) holds the 4 tile bytes of row
//            r's stage s (byte j = tile 4s + j).
//   weights: 512-byte atoms [rows/128][K/128], row r at m = r % 128 of atom
//            (r / 128, s): the down projection's A rows, one atom per stage.
//   gate/up: W1 and W3 in one buffer of 512-byte units [rows/64][K/128];
//            row r of W1 at m = r % 64 of unit (r / 64, s), row r of W3 at
//            m = 64 + r % 64: the gate/up A rows of a CTA (64 W1 rows, then
//            the same 64 W3 rows), one unit per stage.
//   token images (per tile of the grouped GEMMs, launch_tile_scales): 256
//            words per tile and stage, word tile_image_word(j) for the tile's
//            row j, zero past its rows.
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


template <int kLayout>
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
            if (kLayout == kMxTokens) {
                reinterpret_cast<uint32_t*>(sf)[(size_t)s * rows + r] = word;
            } else {
                const int sh = kLayout == kMxWeights ? 7 : 6;  // rows per atom: 128, or 64 of each matrix
                const int m = (int)(r & ((1 << sh) - 1)) + (kLayout == kMxUp ? 64 : 0);
                const size_t atom = ((size_t)(r >> sh) * nst + s) * 512;
                *reinterpret_cast<uint32_t*>(sf + atom + (m & 31) * 16 + (m >> 5) * 4) = word;
            }
        }
    }
}

// Token images of the tiles of a grouped GEMM (one block per image): the
// block finds its group and token tile from the group sizes (the GEMMs'
// split, token_tile_split), then writes the tile's 256-word image of every
// stage.  Blocks past the last tile clear their slot, so the whole buffer is
// written.
__global__ void __launch_bounds__(256) tile_scales_kernel(const uint32_t* __restrict__ src, long long src_rows,
                                                          int nst, const int32_t* __restrict__ row_of, int row_div,
                                                          const int32_t* __restrict__ offsets, int G, long long rows,
                                                          uint32_t* __restrict__ out, int* status) {
    __shared__ int s_first[kMaxGroups + 1];  // first image of each group
    __shared__ int s_g;
    const int tid = threadIdx.x;
    // tile counts, then an exclusive scan over the groups (one warp)
    for (int g = tid; g < G; g += blockDim.x) {
        const long long n = offsets ? (long long)offsets[g + 1] - offsets[g] : rows;
        s_first[g] = n > 0 ? token_tiles((int)n) : 0;
    }
    __syncthreads();
    if (tid < 32) {
        int carry = 0;
        for (int b = 0; b < G; b += 32) {
            const int g = b + tid;
            const int v = g < G ? s_first[g] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid >= o) incl += n;
            }
            if (g < G) s_first[g] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (tid == 0) s_first[G] = carry;
    }
    __syncthreads();
    const int img = blockIdx.x;
    if (img >= s_first[G]) {  // block-uniform: an image slot past the last tile is cleared
        for (int s = 0; s < nst; ++s) out[((size_t)img * nst + s) * 256 + tid] = 0u;
        return;
    }
    for (int g = tid; g < G; g += blockDim.x)
        if (s_first[g] <= img && img < s_first[g + 1]) s_g = g;
    __syncthreads();
    const int g = s_g;
    const long long r0 = offsets ? offsets[g] : 0;
    const int n = (int)(offsets ? (long long)offsets[g + 1] - r0 : rows);
    int start, len;
    token_tile_split(n, s_first[g + 1] - s_first[g], img - s_first[g], start, len);
    const int j = tid;
    long long sr = -1;
    if (j < len) {
        const long long r = r0 + start + j;
        if (r >= 0 && r < rows) sr = row_of ? (long long)row_of[r] / row_div : r;
        if (sr < 0 || sr >= src_rows) {  // rows outside the operand, or a row index outside src
            report(status, kStDeviceCheck);
            sr = -1;
        }
    }
    uint32_t* dst = out + (size_t)img * nst * 256 + tile_image_word(j);
    for (int s = 0; s < nst; ++s) dst[(size_t)s * 256] = sr >= 0 ? src[(size_t)s * src_rows + sr] : 0u;
}

}  // namespace

long long mx_tile_images(long long rows, int groups) { return rows / kTokTile + groups; }

cudaError_t launch_tile_scales(const void* src, long long src_rows, int K, const int32_t* row_of, int row_div,
                               const int32_t* offsets, int groups, long long rows, void* out, int* status,
                               cudaStream_t st) {
    const int nst = K / 128;
    if (rows <= 0 || nst <= 0 || groups <= 0) return cudaSuccess;
    if (groups > kMaxGroups) return cudaErrorInvalidValue;
    const long long blocks = mx_tile_images(rows, groups);
    if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
    tile_scales_kernel<<<(unsigned)blocks, 256, 0, st>>>(static_cast<const uint32_t*>(src), src_rows, nst, row_of,
                                                        row_div > 0 ? row_div : 1, offsets, groups, rows,
                                                        static_cast<uint32_t*>(out), status);
    note_launches(1);
    return cudaGetLastError();
}

size_t mx_scale_bytes(long long rows, int K, int layout) {
    const size_t nst = (size_t)(K / 128);
    if (layout == kMxWeights) return (size_t)((rows + 127) / 128) * nst * 512;
    if (layout == kMxGate || layout == kMxUp) return (size_t)((rows + 63) / 64) * nst * 512;
    return (size_t)rows * nst * 4;
}

cudaError_t launch_quantize_mx(const void* src, long long rows, int kseg, int nseg, int layout, uint8_t* q,
                               void* scales, cudaStream_t st) {
    if (rows <= 0) return cudaSuccess;
    const long long blocks = (rows + kWarps - 1) / kWarps;
    if (blocks > 0x7fffffffll) return cudaErrorInvalidValue;
    const auto* s = static_cast<const uint16_t*>(src);
    auto* sf = static_cast<uint8_t*>(scales);
    const unsigned nb = (unsigned)blocks;
    constexpr int nt = kWarps * 32;
    switch (layout) {
        case kMxTokens: quantize_mx_kernel<kMxTokens><<<nb, nt, 0, st>>>(s, rows, kseg, nseg, q, sf); break;
        case kMxWeights: quantize_mx_kernel<kMxWeights><<<nb, nt, 0, st>>>(s, rows, kseg, nseg, q, sf); break;
        case kMxGate: quantize_mx_kernel<kMxGate><<<nb, nt, 0, st>>>(s, rows, kseg, nseg, q, sf); break;
        case kMxUp: quantize_mx_kernel<kMxUp><<<nb, nt, 0, st>>>(s, rows, kseg, nseg, q, sf); break;
        default: return cudaErrorInvalidValue;
    }
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
