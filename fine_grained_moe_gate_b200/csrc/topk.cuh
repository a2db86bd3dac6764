// Router epilogue shared by the SIMT and tensor-core routers: sigmoid,
// bias-shifted top-k with ties to the lower expert index, unbiased weights
// renormalised in slot order, and the CTA-local load histogram
// ("DeepSeek V3 From Scratch", "In code", route(); "The idea").
#pragma once

#include <float.h>

#include "common.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// Per-thread top-k over one token's E scores, streamed in expert order.
// Keeps the KMAX best (v, s, index) in registers, sorted by descending v;
// a new candidate never displaces an equal v (which has a lower index),
// so equal scores keep ascending index order.
template <int KMAX>
struct TopK {
    float v[KMAX];
    float s[KMAX];
    int id[KMAX];

    __device__ __forceinline__ void init() {
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
            v[j] = -FLT_MAX;
            s[j] = 0.f;
            id[j] = -1;
        }
    }
    // candidate (vi, si, i); i larger than every index pushed before.
    __device__ __forceinline__ void push(float vi, float si, int i) {
        if (!(vi > v[KMAX - 1])) {
            if (!(id[KMAX - 1] < 0 && vi == vi)) return;  // list not full: take any finite score
        }
#pragma unroll
        for (int j = KMAX - 1; j > 0; --j) {
            const bool beats_prev = vi > v[j - 1] || id[j - 1] < 0;
            const bool lands_here = !beats_prev && (vi > v[j] || id[j] < 0);
            if (beats_prev) {
                v[j] = v[j - 1];
                s[j] = s[j - 1];
                id[j] = id[j - 1];
            } else if (lands_here) {
                v[j] = vi;
                s[j] = si;
                id[j] = i;
            }
        }
        if (vi > v[0] || id[0] < 0) {
            v[0] = vi;
            s[0] = si;
            id[0] = i;
        }
    }
};

// Writes idx / w for one token, adds its picks to the CTA histogram.
template <int KMAX>
__device__ __forceinline__ void emit_route(const TopK<KMAX>& tk, int k, int32_t* idx_row, float* w_row,
                                           int* hist_smem, int* status) {
    float den = 0.f;
#pragma unroll
    for (int j = 0; j < KMAX; ++j)
        if (j < k) den = __fadd_rn(den, tk.s[j]);
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
        if (j < k) {
            const int e = tk.id[j];
            if (e < 0) {
                report(status, kStDeviceCheck);  // non-finite scores: fewer than k candidates
                idx_row[j] = -1;
                w_row[j] = 0.f;
                continue;
            }
            idx_row[j] = e;
            w_row[j] = __fdiv_rn(tk.s[j], den);
            atomicAdd(&hist_smem[e], 1);
        }
    }
}

__device__ __forceinline__ float sigmoid_f32(float z) { return __fdiv_rn(1.0f, __fadd_rn(1.0f, expf(-z))); }

}  // namespace moe
