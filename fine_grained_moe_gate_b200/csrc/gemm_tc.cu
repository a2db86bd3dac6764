// Grouped expert GEMMs on the sm_100a tensor cores (tcgen05 + TMEM + TMA)
// for the bf16 layer ("Scaling Efficiency: A Deep Dive into the DeepSeek-V3
// Architecture", DeepSeekMoE sketch: one MLP per expert over the tokens
// routed to it; "DeepSeek V3 Architecture Deep Dive ...", "Throughput on
// NVIDIA H100/H800": tokens of one expert batched together).
//
//   up:   h[r][n]  = silu(A[r] . W1_g[n]) * (A[r] . W3_g[n])   (SwiGLU fused)
//   down: Y[r][n]  = h[r] . W2_g[n]
//
// One persistent CTA per SM walks a device-side tile list built from the
// expert offsets (no host read-back).  Tile = 128 rows x 256 accumulator
// columns; for the up projection the 256 columns are 128 gate rows of W1
// and the matching 128 rows of W3, loaded by two TMA boxes into one
// 256-row operand so gate and up land side by side in TMEM and the SwiGLU
// is an epilogue over one accumulator.  Weights stay in their natural
// [out][in] layout; no packing pass.
//
// Warp roles (192 threads):
//   warp 0      TMA producer (one lane): A box 64x128, B boxes into a
//               4-stage ring of 48 KB stages, 128-byte swizzle.
//   warp 1      TMEM owner; one lane issues tcgen05.mma (M=128, N=256,
//               K=16, bf16 -> fp32) and commits to the ring / accumulator
//               barriers.
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x 16 columns, SwiGLU or
//               plain bf16 conversion, stores.  Two TMEM accumulators
//               (2 x 256 columns) let the epilogue of tile i overlap the
//               main loop of tile i+1.
// Every wait is bounded (common.cuh); on a timeout the CTA raises its abort
// flag, drains the copies and MMAs it issued, frees TMEM and exits.
#include "common.cuh"
#include "kernels.h"
#include "tmap.h"

namespace moe {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;  // 16 KB
constexpr int B_BYTES = BN * BK * 2;  // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int NTHREADS = 192;

struct Ctl {
    uint64_t full[STAGES];
    uint64_t empty[STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
struct Tables {
    int rowstart[kMaxGroups];
    int rows[kMaxGroups];
    int mtiles[kMaxGroups];
    int prefix[kMaxGroups + 1];
};
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + sizeof(Ctl) + sizeof(Tables);

struct Params {
    const int32_t* offsets;
    int G, M;
    int n_tiles, k_blocks;
    int w_rows;     // up: rows of W1/W3 per group (I)
    int kseg, nseg; // down: W2 block geometry along K
    void* out;
    int ldo, n_limit;
    int n_fastest;
    long long a_rows;  // rows of A and of the output; every group must lie inside
    int* status;
};

__device__ __forceinline__ void tile_coords(const Tables* tb, int G, int n_tiles, bool n_fastest, int tile, int& g,
                                            int& mt, int& nt) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {  // last group whose first tile is <= tile (never an empty one)
        const int mid = (lo + hi + 1) >> 1;
        if (tb->prefix[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    g = lo;
    const int q = tile - tb->prefix[g];
    if (n_fastest) {
        mt = q / n_tiles;
        nt = q - mt * n_tiles;
    } else {
        const int m = tb->mtiles[g];
        nt = q / m;
        mt = q - nt * m;
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&b);
}

template <bool UP>
__global__ void __launch_bounds__(NTHREADS, 1)
    tc_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                           const __grid_constant__ CUtensorMap tmB1, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sA = base;
    uint8_t* sB = base + STAGES * A_BYTES;
    Ctl* ctl = reinterpret_cast<Ctl*>(base + STAGES * STAGE_BYTES);
    Tables* tb = reinterpret_cast<Tables*>(ctl + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int G = p.G;

    for (int g = tid; g < G; g += NTHREADS) {
        const int rs = p.offsets ? p.offsets[g] : 0;
        const int re = p.offsets ? p.offsets[g + 1] : p.M;
        int rows = re - rs;
        if (rs < 0 || rows < 0 || (long long)re > p.a_rows) {  // corrupt offsets: skip the group
            report(p.status, kStDeviceCheck);
            rows = 0;
        }
        tb->rowstart[g] = rows > 0 ? rs : 0;
        tb->rows[g] = rows;
        tb->mtiles[g] = (rows + BM - 1) / BM;
    }
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&ctl->tfull[a], 1);
            mbar_init(&ctl->tempty[a], 128);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&ctl->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefix of per-group tile counts
        int carry = 0;
        for (int b = 0; b < G; b += 32) {
            const int g = b + lane;
            const int v = g < G ? tb->mtiles[g] * p.n_tiles : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n;
            }
            if (g < G) tb->prefix[g] = carry + incl - v;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) tb->prefix[G] = carry;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    const int total = tb->prefix[G];
    const bool n_fastest = p.n_fastest != 0;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB0);
            if (UP) tma_prefetch_desc(&tmB1);
            int stage = 0;
            uint32_t phase = 0, issued = 0, iss_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                int g, mt, nt;
                tile_coords(tb, G, p.n_tiles, n_fastest, tile, g, mt, nt);
                const int arow = tb->rowstart[g] + mt * BM;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, &ctl->abort, p.status)) {
                        ok = false;
                        break;
                    }
                    uint64_t* fb = &ctl->full[stage];
                    mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    tma_load_2d(sA + stage * A_BYTES, &tmA, fb, kb * BK, arow, kEvictNormal);
                    if (UP) {
                        const int brow = g * p.w_rows + nt * (BN / 2);
                        tma_load_2d(sB + stage * B_BYTES, &tmB0, fb, kb * BK, brow, kEvictNormal);
                        tma_load_2d(sB + stage * B_BYTES + B_BYTES / 2, &tmB1, fb, kb * BK, brow, kEvictNormal);
                    } else {
                        const int kk = kb * BK;
                        const int seg = kk / p.kseg;
                        tma_load_3d(sB + stage * B_BYTES, &tmB0, fb, kk - seg * p.kseg, nt * BN, g * p.nseg + seg,
                                    kEvictNormal);
                    }
                    issued |= 1u << stage;
                    iss_phase = (iss_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                for (int s = 0; s < STAGES; ++s)
                    if ((issued >> s) & 1u) mbar_wait_drain(&ctl->full[s], (iss_phase >> s) & 1u);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (elect_one()) {
            constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                if (!mbar_wait(&ctl->tempty[acc], acc_phase ^ 1u, &ctl->abort, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&ctl->full[stage], phase, &ctl->abort, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_sw128(smem_u32(sA + stage * A_BYTES));
                    const uint64_t bd = smem_desc_sw128(smem_u32(sB + stage * B_BYTES));
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)  // +32 bytes along K per step
                        tc_mma_bf16(d_tmem, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc,
                                    (kb > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(&ctl->empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(&ctl->tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok) {
                tc_commit(&ctl->drain);
                mbar_wait_drain(&ctl->drain, 0);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int r = q * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            int g, mt, nt;
            tile_coords(tb, G, p.n_tiles, n_fastest, tile, g, mt, nt);
            if (!mbar_wait(&ctl->tfull[acc], acc_phase, &ctl->abort, p.status)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
            const int mrow = mt * BM + r;
            const bool valid = mrow < tb->rows[g];
            const size_t grow = (size_t)(tb->rowstart[g] + mrow);
            if (UP) {
                __nv_bfloat16* dst = out + grow * p.ldo + nt * (BN / 2);
#pragma unroll 1
                for (int c = 0; c < BN / 2; c += 16) {
                    uint32_t gv[16], uv[16];
                    tmem_ld16(taddr + c, gv);
                    tmem_ld16(taddr + BN / 2 + c, uv);
                    tmem_ld_wait();
                    if (valid) {
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float h0 = silu_f32(__uint_as_float(gv[2 * i])) * __uint_as_float(uv[2 * i]);
                            const float h1 =
                                silu_f32(__uint_as_float(gv[2 * i + 1])) * __uint_as_float(uv[2 * i + 1]);
                            pk[i] = pack_bf16x2(h0, h1);
                        }
                        uint4* d4 = reinterpret_cast<uint4*>(dst + c);
                        d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    }
                }
            } else {
                __nv_bfloat16* dst = out + grow * p.ldo + nt * BN;
#pragma unroll 1
                for (int c = 0; c < BN; c += 16) {
                    uint32_t v[16];
                    tmem_ld16(taddr + c, v);
                    tmem_ld_wait();
                    if (valid && nt * BN + c < p.n_limit) {
                        uint32_t pk[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) pk[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                        uint4* d4 = reinterpret_cast<uint4*>(dst + c);
                        d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                        d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&ctl->tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

template <bool UP>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const Params& p, int num_sms,
                   cudaStream_t st) {
    auto kern = tc_grouped_gemm_kernel<UP>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    kern<<<num_sms, NTHREADS, SMEM_BYTES, st>>>(a, b0, b1, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_up(const TcUpArgs& a, int* status, int num_sms, cudaStream_t st) {
    if (a.G <= 0 || a.G > kMaxGroups || a.d % BK != 0 || a.I % (BN / 2) != 0) return cudaErrorInvalidValue;
    CUtensorMap tA, tB0, tB1;
    if (!make_tmap_2d(&tA, a.A, a.d, a.A_rows, a.d, BK, BM) || !make_tmap_2d(&tB0, a.W1, a.d, a.W_rows, a.d, BK, BN / 2) ||
        !make_tmap_2d(&tB1, a.W3, a.d, a.W_rows, a.d, BK, BN / 2))
        return cudaErrorInvalidValue;
    Params p{};
    p.offsets = a.offsets;
    p.G = a.G;
    p.M = a.M;
    p.n_tiles = a.I / (BN / 2);
    p.k_blocks = a.d / BK;
    p.w_rows = a.I;
    p.kseg = a.d;
    p.nseg = 1;
    p.out = a.H;
    p.ldo = a.I;
    p.n_limit = a.I;
    // one large group (the shared experts): walk N fastest so a band of A
    // rows stays in L2 while every weight tile passes over it
    p.n_fastest = (a.offsets == nullptr && a.M > 8 * BM) ? 1 : 0;
    p.a_rows = a.A_rows;
    p.status = status;
    return launch<true>(tA, tB0, tB1, p, num_sms, st);
}

cudaError_t launch_tc_down(const TcDownArgs& a, int* status, int num_sms, cudaStream_t st) {
    if (a.G <= 0 || a.G > kMaxGroups || a.K % BK != 0 || a.kseg % BK != 0 || a.d % BK != 0)
        return cudaErrorInvalidValue;
    CUtensorMap tA, tB;
    if (!make_tmap_2d(&tA, a.H, a.K, a.H_rows, a.K, BK, BM) ||
        !make_tmap_3d(&tB, a.W2, a.kseg, a.d, (unsigned long long)a.G * a.nseg, BK, BN))
        return cudaErrorInvalidValue;
    Params p{};
    p.offsets = a.offsets;
    p.G = a.G;
    p.M = a.M;
    p.n_tiles = (a.d + BN - 1) / BN;
    p.k_blocks = a.K / BK;
    p.w_rows = 0;
    p.kseg = a.kseg;
    p.nseg = a.nseg;
    p.out = a.Y;
    p.ldo = a.d;
    p.n_limit = a.d;
    p.n_fastest = (a.offsets == nullptr && a.M > 8 * BM) ? 1 : 0;
    p.a_rows = a.H_rows;
    p.status = status;
    return launch<false>(tA, tB, tB, p, num_sms, st);
}

}  // namespace moe
