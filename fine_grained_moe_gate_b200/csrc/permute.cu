// Expert-contiguous permutation of token rows ("DeepSeek V3 Architecture Deep
// Dive ...", "Throughput on NVIDIA H100/H800": tokens routed to the same
// expert are batched together).
//
// Rows are ordered by (expert, token), both ascending, so the order is a
// pure function of the routing table.  Deterministic, no global atomics on
// the row cursor:
//   1. hist:    per 128-token chunk c, count[c][e]                 (grid C)
//   2. scan:    per expert, exclusive scan over chunks; offsets = exclusive
//               scan over experts; base[c][e] = offsets[e] + prefix   (1 CTA)
//   3. rank:    per chunk, a bitmask of the chunk's tokens per expert; the
//               rank of token t inside expert e is popcount of the bits
//               below t; row = base[c][e] + rank                     (grid C)
//   4. scatter: token t's row is read once and written to its k rows with
//               16-byte vector stores                                 (grid T)
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kChunk = 128;       // tokens per chunk
constexpr int kChunkWords = kChunk / 32;

__global__ void permute_hist_kernel(const int32_t* __restrict__ idx, int T, int k, int E, int32_t* __restrict__ hist,
                                    int* status) {
    extern __shared__ int cnt[];
    const int c = blockIdx.x;
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const int t0 = c * kChunk;
    const int nt = min(kChunk, T - t0);
    const int na = nt * k;
    const int32_t* ib = idx + (size_t)t0 * k;
    for (int a = threadIdx.x; a < na; a += blockDim.x) {
        const int e = ib[a];
        if (e < 0 || e >= E) {
            report(status, kStDeviceCheck);
            continue;
        }
        atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)c * E + e] = cnt[e];
}

// One CTA of >= E threads (E <= 256 is validated on the host).
__global__ void permute_scan_kernel(int32_t* __restrict__ hist, int C, int E, const int32_t* __restrict__ counts,
                                    int32_t* __restrict__ offsets, int* status) {
    __shared__ int tot[256];
    __shared__ int warp_sum[8];
    const int e = threadIdx.x;
    constexpr int U = 8;  // chunk counts loaded per batch: independent loads in flight
    int running = 0;
    if (e < E) {
        for (int c0 = 0; c0 < C; c0 += U) {
            int h[U];
#pragma unroll
            for (int i = 0; i < U; ++i) h[i] = c0 + i < C ? hist[(size_t)(c0 + i) * E + e] : 0;
#pragma unroll
            for (int i = 0; i < U; ++i) running += h[i];
        }
        if (counts && counts[e] != running) report(status, kStDeviceCheck);
    }
    // exclusive scan of the per-expert totals (deterministic, warp shuffles)
    const int lane = e & 31, wid = e >> 5;
    int v = (e < E) ? running : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sum[wid] = incl;
    __syncthreads();
    int before = 0;
    for (int q = 0; q < wid; ++q) before += warp_sum[q];
    const int excl = before + incl - v;
    if (e < E) {
        tot[e] = excl;
        offsets[e] = excl;
    }
    if (e == blockDim.x - 1) {
        int all = 0;
        for (int q = 0; q < (int)(blockDim.x >> 5); ++q) all += warp_sum[q];
        offsets[E] = all;
    }
    __syncthreads();
    if (e < E) {  // base[c][e] = offsets[e] + counts of expert e in chunks before c
        int acc = tot[e];
        for (int c0 = 0; c0 < C; c0 += U) {
            int h[U];
#pragma unroll
            for (int i = 0; i < U; ++i) h[i] = c0 + i < C ? hist[(size_t)(c0 + i) * E + e] : 0;
#pragma unroll
            for (int i = 0; i < U; ++i)
                if (c0 + i < C) {
                    hist[(size_t)(c0 + i) * E + e] = acc;
                    acc += h[i];
                }
        }
    }
}

__global__ void permute_rank_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                                    const int32_t* __restrict__ base, int32_t* __restrict__ perm_tok,
                                    int32_t* __restrict__ inv_row) {
    extern __shared__ uint32_t masks[];  // [E][kChunkWords]
    const int c = blockIdx.x;
    for (int q = threadIdx.x; q < E * kChunkWords; q += blockDim.x) masks[q] = 0u;
    __syncthreads();
    const int t0 = c * kChunk;
    const int nt = min(kChunk, T - t0);
    const int na = nt * k;
    const int32_t* ib = idx + (size_t)t0 * k;
    for (int a = threadIdx.x; a < na; a += blockDim.x) {
        const int e = ib[a];
        if (e < 0 || e >= E) continue;  // reported by the hist pass
        const int tl = a / k;
        atomicOr(&masks[e * kChunkWords + (tl >> 5)], 1u << (tl & 31));
    }
    __syncthreads();
    const int32_t* bc = base + (size_t)c * E;
    for (int a = threadIdx.x; a < na; a += blockDim.x) {
        const int e = ib[a];
        if (e < 0 || e >= E) continue;
        const int tl = a / k;
        const uint32_t* m = masks + e * kChunkWords;
        int rank = __popc(m[tl >> 5] & ((1u << (tl & 31)) - 1u));
        for (int q = 0; q < (tl >> 5); ++q) rank += __popc(m[q]);
        const int row = bc[e] + rank;
        const int assign = (t0 + tl) * k + (a % k);
        perm_tok[row] = assign;
        inv_row[assign] = row;
    }
}

// Token t: read its row once (16-byte vectors), write it to its k rows.
__global__ void permute_scatter_kernel(const uint4* __restrict__ x, int vec_per_row, int k,
                                       const int32_t* __restrict__ inv_row, int total_rows, uint4* __restrict__ xp) {
    const int t = blockIdx.x;
    __shared__ int rows[16];
    if (threadIdx.x < k) rows[threadIdx.x] = inv_row[(size_t)t * k + threadIdx.x];
    __syncthreads();
    const uint4* src = x + (size_t)t * vec_per_row;
    constexpr int U = 4;  // vectors loaded per thread before the k stores of each
    for (int v0 = threadIdx.x; v0 < vec_per_row; v0 += blockDim.x * U) {
        uint4 val[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int v = v0 + u * blockDim.x;
            if (v < vec_per_row) val[u] = src[v];
        }
        for (int j = 0; j < k; ++j) {
            const int r = rows[j];
            if ((unsigned)r >= (unsigned)total_rows) continue;
            uint4* dst = xp + (size_t)r * vec_per_row;
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int v = v0 + u * blockDim.x;
                if (v < vec_per_row) dst[v] = val[u];
            }
        }
    }
}

size_t permute_scratch_bytes(int T, int E) {
    const size_t C = (size_t)(T + kChunk - 1) / kChunk;
    return C * (size_t)E * sizeof(int32_t);
}

cudaError_t launch_permute(const void* x, const int32_t* idx, const int32_t* counts, int T, int d, int E, int k,
                           size_t elem_bytes, void* x_perm, int32_t* offsets, int32_t* perm_tok, int32_t* inv_row,
                           int32_t* scratch, int* status, cudaStream_t st) {
    const int C = (T + kChunk - 1) / kChunk;
    int launched = 0;
    if (C > 0) {
        permute_hist_kernel<<<C, 256, E * sizeof(int), st>>>(idx, T, k, E, scratch, status);
        ++launched;
    }
    const int nthr = ((E + 31) / 32) * 32;
    permute_scan_kernel<<<1, nthr < 32 ? 32 : nthr, 0, st>>>(scratch, C, E, counts, offsets, status);
    ++launched;
    if (C > 0) {
        permute_rank_kernel<<<C, 256, (size_t)E * kChunkWords * sizeof(uint32_t), st>>>(idx, T, k, E, scratch,
                                                                                          perm_tok, inv_row);
        ++launched;
        if (x && x_perm) {
            const int vec = (int)((size_t)d * elem_bytes / 16);
            // a block size that divides the row's vectors in U = 4 passes when one does
            int threads = 128;
            for (int c = 256; c >= 64; c -= 32)
                if (vec % (4 * c) == 0) {
                    threads = c;
                    break;
                }
            permute_scatter_kernel<<<T, threads, 0, st>>>(static_cast<const uint4*>(x), vec, k, inv_row, T * k,
                                                           static_cast<uint4*>(x_perm));
            ++launched;
        }
    }
    note_launches(launched);
    return cudaGetLastError();
}

}  // namespace moe
