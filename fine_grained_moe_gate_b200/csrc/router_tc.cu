// Tensor-core router for the bf16 layer ("DeepSeek V3 From Scratch",
// "In code", route(); "The idea"): gate GEMM + sigmoid + bias-shifted top-k
// + unbiased renormalised weights + load histogram in one kernel.
//
// A tile = 128 tokens.  All E (<= 256) experts fit one tcgen05 MMA: the
// accumulator is 128 TMEM lanes (tokens) x E columns (experts), fp32.  The
// K loop over d streams x and W_gate through a 4-stage TMA ring.  Small
// batches split K over a cluster of up to 8 CTAs per tile (one CTA per tile
// read all of W_gate alone, 3.7 MB at V3 through one SM); the scores only
// leave shared memory for the caller's optional affinity output.
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
constexpr int RING_BYTES = STAGES * (A_BYTES + B_STRIDE);
constexpr int PS = kMaxExperts + 4;  // row stride (floats) of the score buffers
constexpr int PART_BYTES = BM * PS * 4;

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
// After the K loop the ring is reused for the partial scores of the CTA's K
// slice ([128 tokens][E], fp32) and, with a split K, the reduced scores of the
// tokens this CTA finishes.
constexpr int SCORE_BYTES = PART_BYTES + BM / 2 * PS * 4;
constexpr size_t SMEM_BYTES = 1024 + (size_t)(RING_BYTES > SCORE_BYTES ? RING_BYTES : SCORE_BYTES) + sizeof(Ctl);

__device__ __forceinline__ float4 ld_cluster_f32x4(uint32_t cluster_addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(cluster_addr)
                 : "memory");
    return v;
}

// Split K: the C CTAs of a cluster share one 128-token tile, CTA c running
// the MMA over its slice of d; the slices' fp32 partial scores are summed in
// the fixed order c = 0..C-1 through distributed shared memory (deterministic
// for a given C), CTA c then finishes tokens [c*128/C, (c+1)*128/C) with C
// threads per token, each taking every C-th expert, whose top-k lists are
// merged with warp shuffles.  C = 1 is the plain one-CTA tile.
template <int KMAX, int C>
__global__ void __launch_bounds__(NTHREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const float* __restrict__ bias, int T, int E, int n_pad, uint32_t tmem_cols, int k_blocks,
                     int k, int32_t* __restrict__ idx, float* __restrict__ w, int32_t* __restrict__ counts,
                     float* __restrict__ aff, int* status) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = base;
    uint8_t* sB = base + STAGES * A_BYTES;
    float* part = reinterpret_cast<float*>(base);                 // after the K loop
    float* red = reinterpret_cast<float*>(base + PART_BYTES);     // split K only
    const size_t ring_or_scores = RING_BYTES > SCORE_BYTES ? RING_BYTES : SCORE_BYTES;
    Ctl* ctl = reinterpret_cast<Ctl*>(base + ring_or_scores);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int crank = C > 1 ? (int)cluster_ctarank() : 0;
    const int t0 = (blockIdx.x / C) * BM;
    const int kb0 = crank * k_blocks / C, kb1 = (crank + 1) * k_blocks / C;

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
            for (int kb = kb0; kb < kb1; ++kb) {
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
            for (int kb = kb0; kb < kb1; ++kb) {
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
                                (kb > kb0 || kk > 0) ? 1u : 0u);
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
    } else if (C == 1) {
        // whole K in this CTA: thread r owns token r and streams its scores
        // from TMEM straight into the top-k
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
    } else {
        // partial scores of this K slice: TMEM lane r (token r) -> part[r][0..n_pad)
        const int q = warp & 3;
        const int r = q * 32 + lane;
        if (mbar_wait(&ctl->tfull, 0, &ctl->abort, status)) {
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
            for (int c = 0; c < n_pad; c += 16) {
                uint32_t v[16];
                tmem_ld16(taddr + (uint32_t)c, v);
                tmem_ld_wait();
                float4* dst = reinterpret_cast<float4*>(part + r * PS + c);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                         __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (C > 1) cluster_sync_all();  // every CTA's partial scores are complete and visible

    if (C > 1 && warp >= 2) {
        const int u = tid - 64;             // 0..127
        constexpr int TPC = BM / C;         // tokens this CTA finishes
        const int tl0 = crank * TPC;        // its first token within the tile
        // scores s = sigmoid(sum of the C partials in CTA order), for this CTA's
        // tokens: 128 / TPC threads per token row, four experts per DSMEM load
        // (rows are 16-byte aligned; columns up to n_pad >= E hold MMA results)
        float* sc = red;
        {
            constexpr int TPR = 128 / TPC;
            const int rl = u / TPR, q4 = u - rl * TPR;
            const int r = tl0 + rl;
            const bool keep_aff = aff && t0 + r < T;
#pragma unroll 4
            for (int e = 4 * q4; e < E; e += 4 * TPR) {
                const uint32_t a = smem_u32(part + r * PS + e);
                float4 z = ld_cluster_f32x4(mapa_shared(a, 0));
#pragma unroll
                for (int c = 1; c < C; ++c) {
                    const float4 o = ld_cluster_f32x4(mapa_shared(a, c));
                    z.x = __fadd_rn(z.x, o.x);
                    z.y = __fadd_rn(z.y, o.y);
                    z.z = __fadd_rn(z.z, o.z);
                    z.w = __fadd_rn(z.w, o.w);
                }
                const float zs[4] = {z.x, z.y, z.z, z.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (e + i < E) {
                        const float s = sigmoid_f32(zs[i]);
                        sc[rl * PS + e + i] = s;
                        if (keep_aff) aff[(size_t)(t0 + r) * E + e + i] = s;
                    }
                }
            }
        }
        named_bar_sync(1, 128);
        // top-k: C threads per token, thread `sub` pushes experts sub, sub + C, ...
        const int rl = u / C, sub = u - rl * C;
        const int t = t0 + tl0 + rl;
        TopK<KMAX> tk;
        tk.init();
        for (int e = sub; e < E; e += C) {
            const float s = sc[rl * PS + e];
            tk.push(__fadd_rn(s, ctl->bias[e]), s, e);
        }
        {  // merge the C lists in (v desc, index asc) order
            TopK<KMAX> m;
            m.init();
            int pos = 0;
#pragma unroll
            for (int j = 0; j < KMAX; ++j) {
                float hv = -FLT_MAX, hs = 0.f;
                int hid = 0x7fffffff;
#pragma unroll
                for (int i = 0; i < KMAX; ++i)
                    if (i == pos && tk.id[i] >= 0) {
                        hv = tk.v[i];
                        hs = tk.s[i];
                        hid = tk.id[i];
                    }
                float bv = hv, bs = hs;
                int bid = hid;
#pragma unroll
                for (int o = C / 2; o > 0; o >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    const float os = __shfl_xor_sync(0xffffffffu, bs, o);
                    const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
                    if (ov > bv || (ov == bv && oid < bid)) {
                        bv = ov;
                        bs = os;
                        bid = oid;
                    }
                }
                if (bid != 0x7fffffff) {
                    m.v[j] = bv;
                    m.s[j] = bs;
                    m.id[j] = bid;
                    if (bid == hid) ++pos;
                }
            }
            tk = m;
        }
        if (sub == 0 && t < T) emit_route<KMAX>(tk, k, idx + (size_t)t * k, w + (size_t)t * k, ctl->hist, status);
    }
    __syncthreads();
    for (int e = tid; e < E; e += NTHREADS)
        if (ctl->hist[e]) atomicAdd(&counts[e], ctl->hist[e]);
    if (C > 1) cluster_sync_all();  // no CTA leaves while its partial scores may still be read
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols);
    }
}

template <int KMAX, int C>
cudaError_t launch_kc(const CUtensorMap& tx, const CUtensorMap& tw, const float* bias, int T, int E, int n_pad,
                      uint32_t cols, int kb, int k, int32_t* idx, float* w, int32_t* counts, float* aff, int* status,
                      cudaStream_t st) {
    auto kern = router_tc_kernel<KMAX, C>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(((T + BM - 1) / BM) * C));
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kern, tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status);
    note_launches(1);
    return err == cudaSuccess ? cudaGetLastError() : err;
}

template <int KMAX>
cudaError_t launch_k(const CUtensorMap& tx, const CUtensorMap& tw, const float* bias, int T, int E, int n_pad,
                     uint32_t cols, int kb, int k, int32_t* idx, float* w, int32_t* counts, float* aff, int* status,
                     int split, cudaStream_t st) {
    switch (split) {
        case 8: return launch_kc<KMAX, 8>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, st);
        case 4: return launch_kc<KMAX, 4>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, st);
        case 2: return launch_kc<KMAX, 2>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, st);
        default: return launch_kc<KMAX, 1>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, st);
    }
}

}  // namespace

cudaError_t launch_router_tc(const void* x, const void* wg, const float* bias, int T, int d, int E, int k,
                             int32_t* idx, float* w, int32_t* counts, float* aff, int* status, int num_sms,
                             cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    if (d % BK != 0 || E > kMaxExperts || E <= 0) return cudaErrorInvalidValue;
    const int n_pad = (E + 15) / 16 * 16;  // MMA N: multiple of 16 for M = 128
    uint32_t cols = 32;
    while (cols < (uint32_t)n_pad) cols <<= 1;  // TMEM allocation: power of two >= 32
    CUtensorMap tx, tw;
    if (!make_tmap_2d(&tx, x, d, T, d, BK, BM) || !make_tmap_2d(&tw, wg, d, E, d, BK, n_pad))
        return cudaErrorInvalidValue;
    // K split: as many CTAs per token tile as keep the grid within one wave of SMs
    const int tiles = (T + BM - 1) / BM, kb = d / BK;
    int split = 8;
    while (split > 1 && (tiles * split > num_sms || split > kb)) split >>= 1;
    return k <= 8 ? launch_k<8>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, split, st)
                  : launch_k<16>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, split, st);
}

}  // namespace moe
