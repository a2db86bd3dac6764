// Expert-parallel dispatch and return over peer memory ("DeepSeek-V3" page,
// crackai.dev, "How It Works": custom all-to-all kernels for MoE dispatch /
// combine; "DeepSeek V3 Architecture Deep Dive ...", "Throughput on NVIDIA
// H100/H800": tokens of one expert batched together).
//
// W ranks; rank o owns experts [o*E/W, (o+1)*E/W).  Each rank routes and
// permutes its own T tokens (indices only).  From the step's counts of all
// ranks C[s][e], every rank derives the same plan:
//   base[e][s]    row of rank owner(e)'s receive buffer where the rows that
//                 rank s routes to expert e start; a receive buffer holds its
//                 experts in order, each expert's rows by source rank, each
//                 source's rows by token -- the order the single-GPU
//                 permutation of the concatenated batch gives them.
//   src_off[s][e] rank s's own permutation offsets (exclusive scan of C[s]).
//   recv_off[o][i] offsets of rank o's local experts in its receive buffer.
// Dispatch: rank s stores each of its permuted rows straight into the owner's
// receive buffer (peer stores over NVLink).  Return: the owner stores each
// expert output row straight back into the source rank's buffer, at the row's
// place in that rank's own permutation, where the ordinary combine reads it.
// HBM/NVLink bound: one read and one (remote) write of each row.
#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

__global__ void ep_plan_kernel(const int32_t* __restrict__ C, int W, int E, long long cap, int32_t* __restrict__ plan,
                               int* status) {
    // one thread: E * W <= 16K additions
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    const int Epr = E / W;
    int32_t* base = plan;
    int32_t* src_off = plan + E * W;
    int32_t* recv_off = src_off + W * (E + 1);
    int32_t* tail = recv_off + W * (Epr + 1);  // [receive capacity (rows, clamped to int32), overflow flag]
    for (int s = 0; s < W; ++s) {
        int acc = 0;
        for (int e = 0; e < E; ++e) {
            src_off[s * (E + 1) + e] = acc;
            acc += C[s * E + e];
        }
        src_off[s * (E + 1) + E] = acc;
    }
    int overflow = 0;
    for (int o = 0; o < W; ++o) {
        long long row = 0;
        for (int i = 0; i < Epr; ++i) {
            const int e = o * Epr + i;
            recv_off[o * (Epr + 1) + i] = (int)row;
            for (int s = 0; s < W; ++s) {
                base[e * W + s] = (int)row;
                row += C[s * E + e];
            }
        }
        recv_off[o * (Epr + 1) + Epr] = (int)row;
        if (row > cap) overflow = 1;  // some owner would receive more rows than its buffer holds
    }
    tail[0] = (int)(cap < 0x7fffffffLL ? cap : 0x7fffffffLL);
    tail[1] = overflow;
    if (overflow) report(status, kStDeviceCheck);
}

// last index i in [0, n) with a[i] <= v (a non-decreasing, a[0] <= v)
__device__ __forceinline__ int upper_index(const int32_t* a, int n, int v) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a[mid] <= v) lo = mid; else hi = mid - 1;
    }
    return lo;
}

constexpr int kWarps = 8;

__device__ __forceinline__ void copy_row(const uint4* __restrict__ src, uint4* dst, int vec, int lane) {
    for (int v = lane; v < vec; v += 32) dst[v] = src[v];
}

__global__ void __launch_bounds__(kWarps * 32)
    ep_dispatch_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm_tok,
                       const int32_t* __restrict__ plan, int W, int E, int k, int rank, int vec, int T,
                       EpPeers recv, int* status) {
    const int32_t* base = plan;
    const int32_t* tail = plan + E * W + W * (E + 1) + W * (E / W + 1);
    if (tail[1]) return;  // the plan found a receive buffer too small: nothing is sent (status already set)
    const long long cap_recv = tail[0];
    const int32_t* off = plan + E * W + rank * (E + 1);  // this rank's permutation offsets
    const int rows = min(off[E], T * k);  // this rank's rows (the plan must agree with the permutation)
    const int Epr = E / W;
    const int lane = threadIdx.x & 31;
    for (int p = blockIdx.x * kWarps + (threadIdx.x >> 5); p < rows; p += gridDim.x * kWarps) {
        const int e = upper_index(off, E, p);
        const int o = e / Epr;
        const int q = base[e * W + rank] + (p - off[e]);
        const int t = perm_tok[p] / k;
        if (o < 0 || o >= W || q < 0 || (long long)q >= cap_recv || t < 0 || t >= T) {
            if (lane == 0) report(status, kStDeviceCheck);
            continue;
        }
        copy_row(x + (size_t)t * vec, static_cast<uint4*>(recv.p[o]) + (size_t)q * vec, vec, lane);
    }
    __threadfence_system();  // the peer stores are visible before the step's barrier
}

__global__ void __launch_bounds__(kWarps * 32)
    ep_return_kernel(const uint4* __restrict__ y, const int32_t* __restrict__ plan, int W, int E, int rank, int vec,
                     int cap_back, EpPeers back, int* status) {
    const int Epr = E / W;
    const int32_t* tail = plan + E * W + W * (E + 1) + W * (Epr + 1);
    if (tail[1]) return;
    const long long cap_recv = tail[0];
    const int32_t* base = plan;
    const int32_t* src_off = plan + E * W;
    const int32_t* roff = src_off + W * (E + 1) + rank * (Epr + 1);
    const int rows = (long long)roff[Epr] < cap_recv ? roff[Epr] : (int)cap_recv;
    const int lane = threadIdx.x & 31;
    for (int q = blockIdx.x * kWarps + (threadIdx.x >> 5); q < rows; q += gridDim.x * kWarps) {
        const int e = rank * Epr + upper_index(roff, Epr, q);
        const int s = upper_index(base + e * W, W, q);
        const int p = src_off[s * (E + 1) + e] + (q - base[e * W + s]);
        if (p < 0 || p >= cap_back) {
            if (lane == 0) report(status, kStDeviceCheck);
            continue;
        }
        copy_row(y + (size_t)q * vec, static_cast<uint4*>(back.p[s]) + (size_t)p * vec, vec, lane);
    }
    __threadfence_system();
}

}  // namespace

size_t ep_plan_ints(int W, int E) { return (size_t)E * W + (size_t)W * (E + 1) + (size_t)W * (E / W + 1) + 2; }

cudaError_t launch_ep_plan(const int32_t* counts_all, int W, int E, long long recv_capacity, int32_t* plan,
                           int* status, cudaStream_t st) {
    ep_plan_kernel<<<1, 32, 0, st>>>(counts_all, W, E, recv_capacity, plan, status);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_ep_dispatch(const void* x, const int32_t* perm_tok, const int32_t* plan, int W, int E, int k,
                               int rank, int T, size_t row_bytes, const EpPeers& recv, int num_sms, int* status,
                               cudaStream_t st) {
    ep_dispatch_kernel<<<num_sms * 4, kWarps * 32, 0, st>>>(static_cast<const uint4*>(x), perm_tok, plan, W, E, k,
                                                            rank, (int)(row_bytes / 16), T, recv, status);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_ep_return(const void* y, const int32_t* plan, int W, int E, int k, int rank, int T,
                             size_t row_bytes, const EpPeers& back, int num_sms, int* status, cudaStream_t st) {
    ep_return_kernel<<<num_sms * 4, kWarps * 32, 0, st>>>(static_cast<const uint4*>(y), plan, W, E, rank,
                                                          (int)(row_bytes / 16), T * k, back, status);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
