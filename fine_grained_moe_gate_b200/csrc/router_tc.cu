// Tensor-core router for the bf16 layer ("DeepSeek V3 From Scratch",
// "In code", route(); "The idea"): gate GEMM + sigmoid + bias-shifted top-k
// + unbiased renormalised weights + load histogram in one kernel.
//
// A tile = 128 tokens in one CTA, or 256 tokens in a CTA pair.  All E (<= 256)
// experts fit one tcgen05 MMA: each CTA's accumulator is 128 TMEM lanes
// (tokens) x E columns (experts), fp32.  The K loop over d streams x and
// W_gate through a TMA ring.  Every token tile reads all of W_gate (3.7 MB at
// V3) from L2, so large batches run the 2-SM form (cta_group::2, M = 256):
// each CTA of a pair loads its 128 tokens and half of W_gate's rows, which
// halves the gate re-reads per token.  Small batches split K over a cluster of
// CTAs (or pairs) per tile so that enough SMs take part; the scores only leave
// shared memory for the caller's optional affinity output.
#include "common.cuh"
#include "kernels.h"
#include "tmap.h"
#include "topk.cuh"

namespace moe {
namespace {

constexpr int BM = 128, BK = 64;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
// One CTA holds all N <= 256 rows of W_gate per stage (4 stages); a CTA of a
// pair holds N/2 <= 128 rows (6 stages).  Both rings take 192 KB.
template <bool PAIR>
__host__ __device__ constexpr int ring_stages() {
    return PAIR ? 6 : 4;
}
template <bool PAIR>
__host__ __device__ constexpr int b_stride() {
    return (PAIR ? 128 : 256) * BK * 2;
}
constexpr int MAX_STAGES = 6;
constexpr int RING_BYTES = 4 * (A_BYTES + 256 * BK * 2);
static_assert(ring_stages<true>() * (A_BYTES + b_stride<true>()) == RING_BYTES, "both rings take the same room");
// Warps: 0 loads the token boxes (and arms the stage barrier), 6 the W_gate
// boxes (one issuing thread paces a TMA ring, so two share it), 1 issues the
// MMAs; after the K loop all warps read the accumulator and finish tokens.
// The sigmoid and the top-k of that finish are latency bound, so the pair
// form, whose finish takes as long as its K loop at V3, runs 16 warps (V3
// routing 55.3 -> 51.2 us against 8); the one-CTA form keeps 8 (16 measured
// 10% slower on the small and decode shapes).
template <bool PAIR>
__host__ __device__ constexpr int n_threads() {
    return PAIR ? 512 : 256;
}
constexpr int kWarpB = 6;
constexpr int PS = kMaxExperts + 4;  // row stride (floats) of the score buffers
constexpr int PART_BYTES = BM * PS * 4;

struct Ctl {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
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

// Split K: the C CTAs (or CTA pairs) of a cluster share one token tile, CTA
// (pair) c running the MMA over its slice of d; the slices' fp32 partial
// scores are summed in the fixed order c = 0..C-1 through distributed shared
// memory (deterministic for a given C), CTA c then finishes tokens
// [c*128/C, (c+1)*128/C) of its 128 with C threads per token, each taking
// every C-th expert, whose top-k lists are merged with warp shuffles.  C = 1
// is the plain tile.  PAIR: a cluster of 2C CTAs, ranks 2c and 2c + 1 forming
// the pair of slice c; the even CTA issues the MMAs, the odd one holds tokens
// 128..255 of the tile and W_gate rows [N/2, N).
template <int KMAX, int C, bool PAIR>
__global__ void __launch_bounds__(n_threads<PAIR>(), 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                     const float* __restrict__ bias, int T, int E, int n_pad, uint32_t tmem_cols, int k_blocks,
                     int k, int32_t* __restrict__ idx, float* __restrict__ w, int32_t* __restrict__ counts,
                     float* __restrict__ aff, int* status) {
    constexpr int STAGES = ring_stages<PAIR>();
    constexpr int BSTR = b_stride<PAIR>();
    constexpr int CL = PAIR ? 2 * C : C;  // CTAs per cluster
    constexpr int NTHREADS = n_threads<PAIR>();
    constexpr int NWARPS = NTHREADS / 32;
    static_assert(NWARPS % 4 == 0 && NWARPS >= 8, "whole TMEM lane quarters per warp group");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = base;
    uint8_t* sB = base + STAGES * A_BYTES;
    float* part = reinterpret_cast<float*>(base);                 // after the K loop
    float* red = reinterpret_cast<float*>(base + PART_BYTES);     // split K only
    const size_t ring_or_scores = RING_BYTES > SCORE_BYTES ? RING_BYTES : SCORE_BYTES;
    Ctl* ctl = reinterpret_cast<Ctl*>(base + ring_or_scores);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int crank = CL > 1 ? (int)cluster_ctarank() : 0;
    const int half = PAIR ? (crank & 1) : 0;        // which 128 tokens of a pair's tile
    const int slice = PAIR ? (crank >> 1) : crank;  // K slice
    const uint32_t leader = (uint32_t)(crank - half);
    const uint16_t pair_mask = (uint16_t)(3u << leader);
    const int t0 = (blockIdx.x / CL) * (PAIR ? 2 * BM : BM) + half * BM;
    const int kb0 = slice * k_blocks / C, kb1 = (slice + 1) * k_blocks / C;
    const int n_rows = PAIR ? n_pad / 2 : n_pad;  // W_gate rows this CTA loads per stage

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
        if (PAIR) {
            tmem_alloc_pair(&ctl->tmem_base, tmem_cols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(&ctl->tmem_base, tmem_cols);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    if (PAIR)
        cluster_sync_all();  // the leader's barriers are initialised before the peer's loads count on them
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    // bytes landing on a stage's full barrier: both CTAs' parts for a pair
    const uint32_t stage_tx = (uint32_t)(PAIR ? 2 : 1) * (uint32_t)(A_BYTES + n_rows * BK * 2);

    if (warp == 0 || warp == kWarpB) {
        // token boxes (warp 0, which also arms the stage barrier) or W_gate boxes
        const bool tok = warp == 0;
        if (elect_one()) {
            tma_prefetch_desc(tok ? &tmX : &tmW);
            const uint32_t leader_full = PAIR ? mapa_shared(smem_u32(&ctl->full[0]), leader) : 0u;
            int stage = 0;
            uint32_t phase = 0, issued = 0, iss_phase = 0;
            bool ok = true;
            for (int kb = kb0; kb < kb1; ++kb) {
                if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, &ctl->abort, status)) {
                    ok = false;
                    break;
                }
                if (PAIR) {
                    if (tok && half == 0) mbar_arrive_expect_tx(&ctl->full[stage], stage_tx);
                    const uint32_t fb = leader_full + 8u * (uint32_t)stage;
                    if (tok)
                        tma_load_2d_pair(sA + stage * A_BYTES, &tmX, fb, kb * BK, t0, kEvictFirst);
                    else
                        tma_load_2d_pair(sB + stage * BSTR, &tmW, fb, kb * BK, half * n_rows, kEvictLast);
                } else {
                    uint64_t* fb = &ctl->full[stage];
                    if (tok) {
                        mbar_arrive_expect_tx(fb, stage_tx);
                        tma_load_2d(sA + stage * A_BYTES, &tmX, fb, kb * BK, t0, kEvictFirst);
                    } else {
                        tma_load_2d(sB + stage * BSTR, &tmW, fb, kb * BK, 0, kEvictLast);
                    }
                }
                issued |= 1u << stage;
                iss_phase = (iss_phase & ~(1u << stage)) | (phase << stage);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) {
                if (PAIR) {
                    settle_inflight_loads();
                } else {
                    for (int s = 0; s < STAGES; ++s)
                        if ((issued >> s) & 1u) mbar_wait_drain(&ctl->full[s], (iss_phase >> s) & 1u);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if ((!PAIR || half == 0) && elect_one()) {
            const uint32_t idesc = idesc_bf16_f32(PAIR ? 2 * BM : BM, n_pad);
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
                const uint64_t bd = smem_desc_sw128(smem_u32(sB + stage * BSTR));
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint32_t acc = (kb > kb0 || kk > 0) ? 1u : 0u;
                    if (PAIR)
                        tc_mma_bf16_pair(tmem_base, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, acc);
                    else
                        tc_mma_bf16(tmem_base, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, acc);
                }
                if (PAIR)
                    tc_commit_pair(&ctl->empty[stage], pair_mask);
                else
                    tc_commit(&ctl->empty[stage]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (ok) {
                if (PAIR)
                    tc_commit_pair(&ctl->tfull, pair_mask);
                else
                    tc_commit(&ctl->tfull);
            } else {
                if (PAIR)
                    tc_commit_pair(&ctl->drain, (uint16_t)(1u << leader));
                else
                    tc_commit(&ctl->drain);
                mbar_wait_drain(&ctl->drain, 0);
            }
        }
        __syncwarp();
    } else if (C == 1 && warp >= 2 && warp < 6) {
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
            // Scores into shared memory (the operand ring is free now), column e of token r at
            // sbuf[e * BM + r], with the maxima of v = s + b over the KMAX expert classes e % KMAX: those
            // are KMAX >= k distinct experts, so the token's k-th largest v is at least their minimum and
            // experts below it cannot be chosen.  The pushes then take only the experts at or above it,
            // popped from a bit mask in expert order (pushing every expert ran the sorted-list insertion
            // for the whole warp whenever one lane needed it).
            float* sbuf = part;
            float gmax[KMAX];
#pragma unroll
            for (int j = 0; j < KMAX; ++j) gmax[j] = -FLT_MAX;
            for (int c = 0; c < n_pad; c += 16) {
                uint32_t v[16];
                tmem_ld16(taddr + (uint32_t)c, v);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int e = c + i;
                    if (e < E) {
                        const float s = sigmoid_f32(__uint_as_float(v[i]));
                        sbuf[e * BM + r] = s;
                        gmax[i % KMAX] = fmaxf(gmax[i % KMAX], __fadd_rn(s, ctl->bias[e]));
                        if (aff && t < T) aff[(size_t)t * E + e] = s;
                    }
                }
            }
            float th = gmax[0];
#pragma unroll
            for (int j = 1; j < KMAX; ++j) th = fminf(th, gmax[j]);
            if (E < KMAX) th = -FLT_MAX;  // a class without experts: no bound
            for (int e0 = 0; e0 < E; e0 += 32) {
                uint32_t mask = 0u;
                for (int i = 0; i < 32 && e0 + i < E; ++i)
                    if (__fadd_rn(sbuf[(e0 + i) * BM + r], ctl->bias[e0 + i]) >= th) mask |= 1u << i;
                while (mask) {
                    const int e = e0 + __ffs(mask) - 1;
                    mask &= mask - 1u;
                    const float s = sbuf[e * BM + r];
                    tk.push(__fadd_rn(s, ctl->bias[e]), s, e);
                }
            }
            if (t < T) emit_route<KMAX>(tk, k, idx + (size_t)t * k, w + (size_t)t * k, ctl->hist, status);
        }
    }
    if (C > 1) {
        // partial scores of this K slice: TMEM lane r (token r) -> part[r][0..n_pad);
        // warp w reads lane quarter w % 4, column chunk w / 4 of NWARPS / 4 (multiples of 16)
        const int q = warp & 3;
        const int r = q * 32 + lane;
        constexpr int NCH = NWARPS / 4;
        const int ch = warp >> 2, n16 = n_pad >> 4;
        const int c_lo = (n16 * ch / NCH) << 4, c_hi = (n16 * (ch + 1) / NCH) << 4;
        if (mbar_wait(&ctl->tfull, 0, &ctl->abort, status)) {
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16);
            for (int c = c_lo; c < c_hi; c += 16) {
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

    if (C > 1) {
        const int u = tid;                  // all threads of the CTA
        constexpr int TPC = BM / C;         // tokens this CTA finishes
        constexpr int P = NTHREADS / TPC;   // threads per token
        static_assert(P <= 32 && (P & (P - 1)) == 0, "a token's threads are a power-of-two group of one warp");
        const int tl0 = slice * TPC;        // its first token within the CTA's 128
        // scores s = sigmoid(sum of the C partials in CTA order), for this CTA's
        // tokens: P threads per token row, four experts per DSMEM load
        // (rows are 16-byte aligned; columns up to n_pad >= E hold MMA results)
        float* sc = red;
        {
            constexpr int TPR = P;
            const int rl = u / TPR, q4 = u - rl * TPR;
            const int r = tl0 + rl;
            const bool keep_aff = aff && t0 + r < T;
#pragma unroll 4
            for (int e = 4 * q4; e < E; e += 4 * TPR) {
                const uint32_t a = smem_u32(part + r * PS + e);
                float4 z = ld_cluster_f32x4(mapa_shared(a, (uint32_t)half));
#pragma unroll
                for (int c = 1; c < C; ++c) {
                    const float4 o = ld_cluster_f32x4(mapa_shared(a, (uint32_t)(PAIR ? 2 * c + half : c)));
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
        __syncthreads();
        // top-k: P threads per token, thread `sub` takes experts sub, sub + P, ...
        const int rl = u / P, sub = u - rl * P;
        const int t = t0 + tl0 + rl;
        TopK<KMAX> tk;
        tk.init();
        if (P >= k && E <= 32 * P) {
            // The P threads' largest v are P >= k distinct experts, so the k-th
            // largest v of the token is at least their minimum: experts below it
            // cannot be chosen.  Each thread marks its experts at or above it in a
            // bit mask and pushes only those, in expert order; without the mask
            // the warp ran the insertion for every expert that any lane inserted.
            float vmax = -FLT_MAX;
            for (int e = sub; e < E; e += P) vmax = fmaxf(vmax, __fadd_rn(sc[rl * PS + e], ctl->bias[e]));
            float th = vmax;
#pragma unroll
            for (int o = P / 2; o > 0; o >>= 1) th = fminf(th, __shfl_xor_sync(0xffffffffu, th, o));
            uint32_t mask = 0u;
            for (int e = sub, j = 0; e < E; e += P, ++j)
                if (__fadd_rn(sc[rl * PS + e], ctl->bias[e]) >= th) mask |= 1u << j;
            while (mask) {
                const int e = sub + (__ffs(mask) - 1) * P;
                mask &= mask - 1u;
                const float s = sc[rl * PS + e];
                tk.push(__fadd_rn(s, ctl->bias[e]), s, e);
            }
        } else {
            for (int e = sub; e < E; e += P) {
                const float s = sc[rl * PS + e];
                tk.push(__fadd_rn(s, ctl->bias[e]), s, e);
            }
        }
        {  // merge the P lists in (v desc, index asc) order
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
                for (int o = P / 2; o > 0; o >>= 1) {
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
    // no CTA leaves while its partial scores may still be read, or while its
    // pair leader's MMAs may still read its shared memory
    if (CL > 1) cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        if (PAIR)
            tmem_dealloc_pair(tmem_base, tmem_cols);
        else
            tmem_dealloc(tmem_base, tmem_cols);
    }
}

template <int KMAX, int C, bool PAIR>
cudaError_t launch_kc(const CUtensorMap& tx, const CUtensorMap& tw, const float* bias, int T, int E, int n_pad,
                      uint32_t cols, int kb, int k, int32_t* idx, float* w, int32_t* counts, float* aff, int* status,
                      cudaStream_t st) {
    auto kern = router_tc_kernel<KMAX, C, PAIR>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    constexpr int CL = PAIR ? 2 * C : C;
    const int tile = PAIR ? 2 * BM : BM;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(((T + tile - 1) / tile) * CL));
    cfg.blockDim = dim3(n_threads<PAIR>());
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kern, tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status);
    note_launches(1);
    return err == cudaSuccess ? cudaGetLastError() : err;
}

template <int KMAX, bool PAIR>
cudaError_t launch_k(const CUtensorMap& tx, const CUtensorMap& tw, const float* bias, int T, int E, int n_pad,
                     uint32_t cols, int kb, int k, int32_t* idx, float* w, int32_t* counts, float* aff, int* status,
                     int split, cudaStream_t st) {
    switch (split) {
        case 8:
            if (!PAIR)  // a pair cluster of 16 CTAs is not portable
                return launch_kc<KMAX, 8, false>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status,
                                                 st);
            return cudaErrorInvalidValue;
        case 4: return launch_kc<KMAX, 4, PAIR>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, st);
        case 2: return launch_kc<KMAX, 2, PAIR>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, st);
        default:
            return launch_kc<KMAX, 1, PAIR>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, st);
    }
}

}  // namespace

cudaError_t launch_router_tc(const void* x, const void* wg, const float* bias, int T, int d, int E, int k,
                             int32_t* idx, float* w, int32_t* counts, float* aff, int* status, int num_sms,
                             cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    if (d % BK != 0 || E > kMaxExperts || E <= 0) return cudaErrorInvalidValue;
    const int n_pad = (E + 15) / 16 * 16;  // MMA N: a multiple of 16 (N/2 rows per CTA of a pair: 8-row atoms)
    uint32_t cols = 32;
    while (cols < (uint32_t)n_pad) cols <<= 1;  // TMEM allocation: power of two >= 32
    // Large batches: CTA pairs of 256 tokens (half the W_gate rows per CTA);
    // the one-CTA form only while its K split would still reach 4 or more.
    const int tiles1 = (T + BM - 1) / BM, kb = d / BK;
    const bool pair = T > 2 * BM && tiles1 * 4 > num_sms;
    CUtensorMap tx, tw;
    if (!make_tmap_2d(&tx, x, d, T, d, BK, BM) || !make_tmap_2d(&tw, wg, d, E, d, BK, pair ? n_pad / 2 : n_pad))
        return cudaErrorInvalidValue;
    // K split: as many CTAs per token tile as keep the grid within one wave of SMs
    const int tiles = pair ? (T + 2 * BM - 1) / (2 * BM) : tiles1, per = pair ? 2 : 1;
    int split = pair ? 4 : 8;  // clusters of at most 8 CTAs
    while (split > 1 && (tiles * split * per > num_sms || split > kb)) split >>= 1;
    if (pair)
        return k <= 8 ? launch_k<8, true>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, split, st)
                      : launch_k<16, true>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, split,
                                           st);
    return k <= 8 ? launch_k<8, false>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, split, st)
                  : launch_k<16, false>(tx, tw, bias, T, E, n_pad, cols, kb, k, idx, w, counts, aff, status, split, st);
}

}  // namespace moe
