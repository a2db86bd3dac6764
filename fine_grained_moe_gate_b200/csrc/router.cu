// Router and balancing kernels.
//
// Router ("DeepSeek V3 From Scratch", "In code", route(); "The idea"):
//   s = sigmoid(x . W_gate^T) in fp32, v = s + bias, top-k of v with ties to
//   the lower expert index, weights = s of the chosen experts renormalised to
//   sum to 1 (sum in slot order, IEEE division), plus the per-expert count
//   of assignments.
// Bias update ("In code", update_bias(); kbwen.com DeepSeek tag page, "A bias
//   term for each expert"): load = count / T, bias += step * sign(target -
//   load), once per step.
//
// This file holds the SIMT router (fp32 inputs, and bf16 for any shape) and
// the bias update; the top-k / weight / histogram epilogue is shared with
// the tensor-core router (router_tc.cu) through topk.cuh.
#include "common.cuh"
#include "kernels.h"
#include "topk.cuh"

namespace moe {

// ---------------------------------------------------------------------------
// SIMT router.  One CTA = 32 tokens x all E experts, 256 threads.
//  phase 1: thread e accumulates x[t] . W_gate[e] for the CTA's 32 tokens
//           over 32-wide K chunks staged in shared memory (fp32 FFMA).
//  phase 2: sigmoid, scores to shared memory (and to affinity_out).
//  phase 3: warp 0, one thread per token: top-k + weights + histogram.
constexpr int kRtTok = 32;
constexpr int kRtKc = 32;

template <typename Tin, int KMAX>
__global__ void __launch_bounds__(256) router_simt_kernel(const Tin* __restrict__ x, const Tin* __restrict__ wg,
                                                          const float* __restrict__ bias, int T, int d, int E, int k,
                                                          int32_t* __restrict__ idx, float* __restrict__ w,
                                                          int32_t* __restrict__ counts, float* __restrict__ aff,
                                                          int* status) {
    extern __shared__ float sm[];
    const int sstride = E | 1;  // odd row stride: conflict-free column reads
    float* xs = sm;                              // [kRtTok][kRtKc + 1]
    float* ws = xs + kRtTok * (kRtKc + 1);       // [E][kRtKc + 1]
    float* S = ws + E * (kRtKc + 1);             // [kRtTok][sstride]
    float* bs = S + kRtTok * sstride;            // [E]
    int* hist = reinterpret_cast<int*>(bs + E);  // [E]

    const int tid = threadIdx.x;
    const int t0 = blockIdx.x * kRtTok;
    for (int e = tid; e < E; e += blockDim.x) {
        hist[e] = 0;
        bs[e] = bias[e];
    }

    float acc[kRtTok];
#pragma unroll
    for (int t = 0; t < kRtTok; ++t) acc[t] = 0.f;

    for (int c0 = 0; c0 < d; c0 += kRtKc) {
        __syncthreads();
        for (int q = tid; q < kRtTok * kRtKc; q += blockDim.x) {
            const int r = q / kRtKc, c = q % kRtKc;
            const int t = t0 + r;
            xs[r * (kRtKc + 1) + c] = (t < T && c0 + c < d) ? to_f32(x[(size_t)t * d + c0 + c]) : 0.f;
        }
        for (int q = tid; q < E * kRtKc; q += blockDim.x) {
            const int r = q / kRtKc, c = q % kRtKc;
            ws[r * (kRtKc + 1) + c] = (c0 + c < d) ? to_f32(wg[(size_t)r * d + c0 + c]) : 0.f;
        }
        __syncthreads();
        if (tid < E) {
            const float* wr = ws + tid * (kRtKc + 1);
#pragma unroll 4
            for (int c = 0; c < kRtKc; ++c) {
                const float wv = wr[c];
#pragma unroll
                for (int t = 0; t < kRtTok; ++t) acc[t] = fmaf(xs[t * (kRtKc + 1) + c], wv, acc[t]);
            }
        }
    }
    if (tid < E) {
#pragma unroll
        for (int t = 0; t < kRtTok; ++t) {
            const float s = sigmoid_f32(acc[t]);
            S[t * sstride + tid] = s;
            if (aff && t0 + t < T) aff[(size_t)(t0 + t) * E + tid] = s;
        }
    }
    __syncthreads();
    if (tid < kRtTok && t0 + tid < T) {
        const int t = t0 + tid;
        TopK<KMAX> tk;
        tk.init();
        const float* Sr = S + tid * sstride;
        for (int e = 0; e < E; ++e) {
            const float s = Sr[e];
            tk.push(__fadd_rn(s, bs[e]), s, e);
        }
        emit_route<KMAX>(tk, k, idx + (size_t)t * k, w + (size_t)t * k, hist, status);
    }
    __syncthreads();
    for (int e = tid; e < E; e += blockDim.x)
        if (hist[e]) atomicAdd(&counts[e], hist[e]);
}

size_t router_simt_smem(int E) {
    const int sstride = E | 1;
    return sizeof(float) * ((size_t)kRtTok * (kRtKc + 1) + (size_t)E * (kRtKc + 1) + (size_t)kRtTok * sstride + E) +
           sizeof(int) * (size_t)E;
}

template <typename Tin, int KMAX>
static cudaError_t launch_router_simt_t(const void* x, const void* wg, const float* bias, int T, int d, int E, int k,
                                        int32_t* idx, float* w, int32_t* counts, float* aff, int* status,
                                        cudaStream_t st) {
    const size_t smem = router_simt_smem(E);
    auto kern = router_simt_kernel<Tin, KMAX>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const int grid = (T + kRtTok - 1) / kRtTok;
    kern<<<grid, 256, smem, st>>>(static_cast<const Tin*>(x), static_cast<const Tin*>(wg), bias, T, d, E, k, idx,
                                  w, counts, aff, status);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_router_simt(const void* x, const void* wg, const float* bias, int T, int d, int E, int k,
                               bool bf16, int32_t* idx, float* w, int32_t* counts, float* aff, int* status,
                               cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    if (bf16) {
        return k <= 8 ? launch_router_simt_t<__nv_bfloat16, 8>(x, wg, bias, T, d, E, k, idx, w, counts, aff, status, st)
                      : launch_router_simt_t<__nv_bfloat16, 16>(x, wg, bias, T, d, E, k, idx, w, counts, aff, status,
                                                                 st);
    }
    return k <= 8 ? launch_router_simt_t<float, 8>(x, wg, bias, T, d, E, k, idx, w, counts, aff, status, st)
                  : launch_router_simt_t<float, 16>(x, wg, bias, T, d, E, k, idx, w, counts, aff, status, st);
}

// ---------------------------------------------------------------------------
// Bias update: one thread per expert, every operation a single IEEE fp32
// rounding (no contraction), so the result is a deterministic function of
// (counts, bias).
__global__ void bias_update_kernel(const int32_t* __restrict__ counts, int T, int E, int k, float step,
                                   const float* __restrict__ target, float* __restrict__ bias,
                                   float* __restrict__ load_out) {
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= E) return;
    const float load = __fdiv_rn((float)counts[i], (float)T);
    const float tgt = target ? target[i] : __fdiv_rn((float)k, (float)E);
    const float diff = __fsub_rn(tgt, load);
    const float sgn = diff > 0.f ? 1.f : (diff < 0.f ? -1.f : 0.f);
    bias[i] = __fadd_rn(bias[i], __fmul_rn(sgn, step));
    if (load_out) load_out[i] = load;
}

cudaError_t launch_bias_update(const int32_t* counts, int T, int E, int k, float step, const float* target,
                               float* bias, float* load_out, cudaStream_t st) {
    bias_update_kernel<<<(E + 255) / 256, 256, 0, st>>>(counts, T, E, k, step, target, bias, load_out);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
