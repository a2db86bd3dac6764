// Tensor-core router for the bf16 layer ("DeepSeek V3 From Scratch",
// "In code", route(); "The idea"): gate GEMM + sigmoid + bias-shifted top-k
// + unbiased renormalised weights + load histogram in one kernel.
//
// One CTA = 128 tokens.  All E (<= 256) experts fit one tcgen05 MMA: the
// accumulator is 128 TMEM lanes (tokens) x E columns (experts), fp32.  The
// K loop over d streams x and W_gate through a 4-stage TMA ring.  Epilogue
// thread r owns token r: it reads its E scores from TMEM 16 at a time and
// runs the shared top-k (topk.cuh) in registers, so no score matrix is
// written unless the caller asks for the affinities.
#include "common.cuh"
#include "kernels.h"
#include "tmap.h"
#include "topk.cuh"

namespace moe {
namespace {

constexpr int BM = 128, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_STRIDE = 256 * BK * 2;  // room for N <= 256 rows
constexpr int NTHREADS = 192;

struct Ctl {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    float bias[kMaxExperts];
    int hist[kMaxExperts];
};
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * (A_BYTES + B_STRIDE) + sizeof(Ctl);

template <int KMAX>
__global__ void __launch_bounds__(NTHREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const float* __restrict__ bias, int T, int E, int n_pad, uint32_t tmem_cols, int k_blocks,
                     int k, int32_t* __restrict__ idx, float* __restrict__ w, int32_t* __restrict__ counts,
                     float* __restrict__ aff, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = base;
    uint8_t* sB = base + STAGES * A_BYTES;
    Ctl* ctl = reinterpret_cast<Ctl*>(base + STAGES * (A_BYTES + B_STRIDE));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t0 = blockIdx.x * BM;

    for (int e = tid; e < E; e += NTHREADS) {
        ctl->bias[e] = bias[e];
        ctl->hist[e] = 0;
    }
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        mbar_init(&ctl->tfull, 1);
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, tmem_cols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    const uint32_t stage_tx = (uint32_t)(A_BYTES + n_pad * BK * 2);

    if (warp == 0) {
        if (elect_one()) {
            tma_prefetch_desc(&tmX);
            tma_prefetch_desc(&tmW);
            int stage = 0;
            uint32_t phase = 0, issued = 0, iss_phase = 0;
            bool ok = true;
            for (int kb = 0; kb < k_blocks; ++kb) {
                if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, &ctl->abort, status)) {
                    ok = false;
                    break;
                }
                uint64_t* fb = &ctl->full[stage];
                mbar_arrive_expect_tx(fb, stage_tx);
                tma_load_2d(sA + stage * A_BYTES, &tmX, fb, kb * BK, t0, kEvictFirst);
                tma_load_2d(sB + stage * B_STRIDE, &tmW, fb, kb * BK, 0, kEvictLast);
                issued |= 1u << stage;
                iss_phase = (iss_phase & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) {
                for (int s = 0; s < STAGES; ++s)
                    if ((issued >> s) & 1u) mbar_wait_drain(&ctl->full[s], (iss_phase >> s) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (elect_one()) {
            const uint32_t idesc = idesc_bf16_f32(BM, n_pad);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int kb = 0; kb < k_blocks; ++kb) {
                if (!mbar_wait(&ctl->full[stage], phase, &ctl->abort, status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = smem_desc_sw128(smem_u32(sA + stage * A_BYTES));
                const uint64_t bd = smem_desc_sw128(smem_u32(sB + stage * B_STRIDE));
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    tc_mma_bf16(tmem_base, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc,
                                (kb > 0 || kk > 0) ? 1u : 0u);
                tc_commit(&ctl->empty[stage]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) {
                tc_commit(&ctl->tfull);
            } else {
                tc_commit(&ctl->drain);
                mbar_wait_drain(&ctl->drain, 0);
            }
        }
        __syncwarp();
    } else {
        const int q = warp & 3;
        const int r = q * 32 + lane;
        const int t = t0 + r;
        if (mbar_wait(&ctl->tfull, 0, &ctl->abort, status)) {
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
            TopK<KMAX> tk;
            tk.init();
            for (int c = 0; c < n_pad; c += 16) {
                uint32_t v[16];
                tmem_ld16(taddr + (uint32_t)c, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int e = c + i;
                    if (e < E) {
                        const float s = sigmoid_f32(__uint_as_float(v[i]));
                        tk.push(__fadd_rn(s, ctl->bias[e]), s, e);
                        if (aff && t < T) aff[(size_t)t * E + e] = s;
                    }
                }
            }
            if (t < T) emit_route<KMAX>(tk, k, idx + (size_t)t * k, w + (size_t)t * k, ctl->hist, status);
        }
    }
    tc_fence_before();
    __syncthreads();
    for (int e = tid; e < E; e += NTHREADS)
        if (ctl->hist[e]) atomicAdd(&counts[e], ctl->hist[e]);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
}

template <int KMAX>
cudaError_t launch_k(const CUtensorMap& tx, const CUtensorMap& tw, const float* bias, int T, int E, int n_pad,
                     uint32_t cols, int kb, int k, int32_t* idx, float* w, int32_t* counts, float* aff, int* status,
                     cudaStream_t st) {
    auto kern = router_tc_kernel<KMAX>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    const int grid = (T + BM - 1) / BM;
    kern<<<grid, NTHREADS, SMEM_BYTES, st>>>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_tc(const void* x, const void* wg, const float* bias, int T, int d, int E, int k,
                             int32_t* idx, float* w, int32_t* counts, float* aff, int* status, int num_sms,
                             cudaStream_t st) {
    (void)num_sms;
    if (T == 0) return cudaSuccess;
    if (d % BK != 0 || E > kMaxExperts || E <= 0) return cudaErrorInvalidValue;
    const int n_pad = (E + 15) / 16 * 16;  // MMA N: multiple of 16 for M = 128
    uint32_t cols = 32;
    while (cols < (uint32_t)n_pad) cols <<= 1;  // TMEM allocation: power of two >= 32
    CUtensorMap tx, tw;
    if (!make_tmap_2d(&tx, x, d, T, d, BK, BM) || !make_tmap_2d(&tw, wg, d, E, d, BK, n_pad))
        return cudaErrorInvalidValue;
    return k <= 8 ? launch_k<8>(tx, tw, bias, T, E, n_pad, cols, d / BK, k, idx, w, counts, aff, status, st)
                  : launch_k<16>(tx, tw, bias, T, E, n_pad, cols, d / BK, k, idx, w, counts, aff, status, st);
}

}  // namespace moe
