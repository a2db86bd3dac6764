// Grouped expert GEMMs on the sm_100a tensor cores (tcgen05 + TMEM + TMA)
// for the bf16 layer ("Scaling Efficiency: A Deep Dive into the DeepSeek-V3
// Architecture", DeepSeekMoE sketch: one MLP per expert over the tokens
// routed to it; "DeepSeek V3 Architecture Deep Dive ...", "Throughput on
// NVIDIA H100/H800": tokens of one expert batched together).
//
//   up:   h[t][f] = silu(W1_g[f] . a[t]) * (W3_g[f] . a[t])   (SwiGLU fused)
//   down: y[t][o] = W2_g[o] . h[t]
//
// Weights are the MMA's M operand (128 output features per tile) and the
// expert's tokens the N operand.  N only has to be a multiple of 16, so the
// last token tile of an expert is trimmed to its real rows rounded up to 16
// instead of padding a 128-row M tile: with ~256 rows per expert the
// padded MMA work drops from ~25% to ~3%.
//
//   up tile:   128 features of W1 and the same 128 of W3 x up to 128 tokens;
//              two MMAs per K step into TMEM columns [0,128) (gate) and
//              [128,256) (up), so one thread holds gate and up of its feature
//              and SwiGLU is an epilogue over the accumulator.
//   down tile: 128 features of W2 x up to 256 tokens, one MMA per K step.
// Both use 48 KB smem stages (4-stage TMA ring, 128-byte swizzle) and two
// 256-column TMEM accumulators, so the epilogue of one tile overlaps the
// main loop of the next.  Weights stay in their natural [out][in] layout.
//
// One persistent CTA per SM walks a device-side tile list built from the
// expert offsets (no host read-back); per expert, token tiles are walked
// fastest so the CTAs working on one weight tile at the same time share it
// in L2, and the expert's token rows stay in L2 across its feature tiles.
//
// Warp roles (192 threads):
//   warp 0      TMA producer (one lane)
//   warp 1      TMEM owner; one lane issues tcgen05.mma (kind::f16, M=128,
//               N = trimmed token count) and commits to the barriers
//   warps 2..5  epilogue: tcgen05.ld (32 lanes = 32 features x 16 tokens),
//               SwiGLU / bf16 conversion, transpose through a 1 KB per-warp
//               shared buffer into token-major rows, 32-byte vector stores.
// Every wait is bounded (common.cuh); on a timeout the CTA raises its abort
// flag, drains the copies and MMAs it issued, frees TMEM and exits.
#include "common.cuh"
#include "kernels.h"
#include "tmap.h"

namespace moe {
namespace {

constexpr int BF = 128;  // weight rows (output features) per tile = MMA M
constexpr int BK = 64;   // K per stage: one 128-byte swizzle row of bf16
constexpr int STAGES = 4;
constexpr int W_BYTES = BF * BK * 2;  // 16 KB per weight operand
constexpr int STAGE_BYTES = 48 * 1024;
constexpr int SMALL_ROWS = 32;        // token box for tiles of <= 32 tokens
constexpr uint32_t ACC_COLS = 256;    // one accumulator buffer
constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
constexpr int NTHREADS = 192;
constexpr int EPI_BUF = 16 * 32 * 2;  // per-warp transpose buffer: 16 tokens x 32 features

template <bool UP>
struct Geo {
    static constexpr int NT = UP ? 128 : 256;              // tokens per tile
    static constexpr int A_BYTES = UP ? 2 * W_BYTES : W_BYTES;
    static constexpr int B_BYTES = NT * BK * 2;
    static_assert(A_BYTES + B_BYTES == STAGE_BYTES, "stage layout");
};

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
    int ttiles[kMaxGroups];  // token tiles per group
    int prefix[kMaxGroups + 1];
};
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 4 * EPI_BUF + sizeof(Ctl) + sizeof(Tables);

struct Params {
    const int32_t* offsets;
    int G, M;
    int f_tiles;       // feature tiles per group
    int k_blocks;
    int w_rows;        // up: rows of W1/W3 per group (I)
    int kseg, nseg;    // down: W2 block geometry along K
    void* out;
    int ldo;           // output row pitch (elements)
    int f_limit;       // valid output features
    long long a_rows;  // rows of the token operand and of the output
    int* status;
};

struct TileCoord {
    int g, ft, tt;
};

__device__ __forceinline__ TileCoord tile_coords(const Tables* tb, int G, int tile) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {  // last group whose first tile is <= tile (never an empty one)
        const int mid = (lo + hi + 1) >> 1;
        if (tb->prefix[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int q = tile - tb->prefix[lo];
    const int nt = tb->ttiles[lo];
    return {lo, q / nt, q - (q / nt) * nt};
}

__device__ __forceinline__ uint16_t bf16_bits(float v) {
    const __nv_bfloat16 b = __float2bfloat16_rn(v);
    return *reinterpret_cast<const uint16_t*>(&b);
}

template <bool UP>
__global__ void __launch_bounds__(NTHREADS, 1)
    tc_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmW0, const __grid_constant__ CUtensorMap tmW1,
                           const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmXs,
                           const Params p) {
    using GE = Geo<UP>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* ring = base;
    uint8_t* epi = base + STAGES * STAGE_BYTES;
    Ctl* ctl = reinterpret_cast<Ctl*>(epi + 4 * EPI_BUF);
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
        tb->ttiles[g] = (rows + GE::NT - 1) / GE::NT;
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
            const int v = g < G ? tb->ttiles[g] * p.f_tiles : 0;
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

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (elect_one()) {
            tma_prefetch_desc(&tmW0);
            if (UP) tma_prefetch_desc(&tmW1);
            tma_prefetch_desc(&tmX);
            tma_prefetch_desc(&tmXs);
            int stage = 0;
            uint32_t phase = 0, issued = 0, iss_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const TileCoord tc = tile_coords(tb, G, tile);
                const int tok0 = tb->rowstart[tc.g] + tc.tt * GE::NT;
                const int ntok = min(GE::NT, tb->rows[tc.g] - tc.tt * GE::NT);
                const bool small = ntok <= SMALL_ROWS;
                const uint32_t tx = GE::A_BYTES + (small ? SMALL_ROWS : GE::NT) * BK * 2;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, &ctl->abort, p.status)) {
                        ok = false;
                        break;
                    }
                    uint64_t* fb = &ctl->full[stage];
                    uint8_t* sa = ring + stage * STAGE_BYTES;
                    uint8_t* sb = sa + GE::A_BYTES;
                    mbar_arrive_expect_tx(fb, tx);
                    if (UP) {
                        const int wrow = tc.g * p.w_rows + tc.ft * BF;
                        tma_load_2d(sa, &tmW0, fb, kb * BK, wrow, kEvictNormal);
                        tma_load_2d(sa + W_BYTES, &tmW1, fb, kb * BK, wrow, kEvictNormal);
                    } else {
                        const int kk = kb * BK;
                        const int seg = kk / p.kseg;
                        tma_load_3d(sa, &tmW0, fb, kk - seg * p.kseg, tc.ft * BF, tc.g * p.nseg + seg, kEvictNormal);
                    }
                    tma_load_2d(sb, small ? &tmXs : &tmX, fb, kb * BK, tok0, kEvictNormal);
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
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
                const TileCoord tc = tile_coords(tb, G, tile);
                const int ntok = min(GE::NT, tb->rows[tc.g] - tc.tt * GE::NT);
                const int n_mma = (ntok + 15) & ~15;
                const uint32_t idesc = idesc_bf16_f32(BF, n_mma);
                if (!mbar_wait(&ctl->tempty[acc], acc_phase ^ 1u, &ctl->abort, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * ACC_COLS;
                for (int kb = 0; kb < p.k_blocks; ++kb) {
                    if (!mbar_wait(&ctl->full[stage], phase, &ctl->abort, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t* sa = ring + stage * STAGE_BYTES;
                    const uint64_t ad0 = smem_desc_sw128(smem_u32(sa));
                    const uint64_t bd = smem_desc_sw128(smem_u32(sa + GE::A_BYTES));
                    if (UP) {
                        const uint64_t ad1 = smem_desc_sw128(smem_u32(sa + W_BYTES));
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {  // +32 bytes along K per step
                            const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
                            tc_mma_bf16(d_tmem, ad0 + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, accum);
                            tc_mma_bf16(d_tmem + GE::NT, ad1 + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc,
                                        accum);
                        }
                    } else {
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            tc_mma_bf16(d_tmem, ad0 + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc,
                                        (kb > 0 || kk > 0) ? 1u : 0u);
                    }
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
        const int q = warp & 3;  // TMEM lane quarter: features 32q .. 32q+31 of the tile
        uint16_t* buf = reinterpret_cast<uint16_t*>(epi + q * EPI_BUF);  // [16 tokens][32 features]
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
            const TileCoord tc = tile_coords(tb, G, tile);
            const int tok0 = tb->rowstart[tc.g] + tc.tt * GE::NT;
            const int ntok = min(GE::NT, tb->rows[tc.g] - tc.tt * GE::NT);
            const int f0 = tc.ft * BF + q * 32;  // first feature of this warp
            if (!mbar_wait(&ctl->tfull[acc], acc_phase, &ctl->abort, p.status)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * ACC_COLS;
            // this lane's share of a 16-token x 32-feature block: token lane/2, 16 features
            const int my_tok = lane >> 1;
            const int my_half = (lane & 1) * 16;
            const bool feat_ok = f0 + my_half < p.f_limit;  // f_limit is a multiple of 16
#pragma unroll 1
            for (int c = 0; c < ntok; c += 16) {
                float v[16];
                if (UP) {
                    uint32_t gv[16], uv[16];
                    tmem_ld16(taddr + (uint32_t)c, gv);
                    tmem_ld16(taddr + (uint32_t)(GE::NT + c), uv);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = silu_f32(__uint_as_float(gv[i])) * __uint_as_float(uv[i]);
                } else {
                    uint32_t r[16];
                    tmem_ld16(taddr + (uint32_t)c, r);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
                }
                // transpose: buf[token i][feature lane]
#pragma unroll
                for (int i = 0; i < 16; ++i) buf[i * 32 + lane] = bf16_bits(v[i]);
                __syncwarp();
                if (c + my_tok < ntok && feat_ok) {
                    const uint4* src = reinterpret_cast<const uint4*>(buf + my_tok * 32 + my_half);
                    uint4* dst = reinterpret_cast<uint4*>(out + (size_t)(tok0 + c + my_tok) * p.ldo + f0 + my_half);
                    dst[0] = src[0];
                    dst[1] = src[1];
                }
                __syncwarp();
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
cudaError_t launch(const CUtensorMap& w0, const CUtensorMap& w1, const CUtensorMap& x, const CUtensorMap& xs,
                   const Params& p, int num_sms, cudaStream_t st) {
    auto kern = tc_grouped_gemm_kernel<UP>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    kern<<<num_sms, NTHREADS, SMEM_BYTES, st>>>(w0, w1, x, xs, p);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_up(const TcUpArgs& a, int* status, int num_sms, cudaStream_t st) {
    if (a.G <= 0 || a.G > kMaxGroups || a.d % BK != 0 || a.I % BF != 0) return cudaErrorInvalidValue;
    CUtensorMap tW1, tW3, tX, tXs;
    if (!make_tmap_2d(&tW1, a.W1, a.d, a.W_rows, a.d, BK, BF) || !make_tmap_2d(&tW3, a.W3, a.d, a.W_rows, a.d, BK, BF) ||
        !make_tmap_2d(&tX, a.A, a.d, a.A_rows, a.d, BK, Geo<true>::NT) ||
        !make_tmap_2d(&tXs, a.A, a.d, a.A_rows, a.d, BK, SMALL_ROWS))
        return cudaErrorInvalidValue;
    Params p{};
    p.offsets = a.offsets;
    p.G = a.G;
    p.M = a.M;
    p.f_tiles = a.I / BF;
    p.k_blocks = a.d / BK;
    p.w_rows = a.I;
    p.kseg = a.d;
    p.nseg = 1;
    p.out = a.H;
    p.ldo = a.I;
    p.f_limit = a.I;
    p.a_rows = a.A_rows;
    p.status = status;
    return launch<true>(tW1, tW3, tX, tXs, p, num_sms, st);
}

cudaError_t launch_tc_down(const TcDownArgs& a, int* status, int num_sms, cudaStream_t st) {
    if (a.G <= 0 || a.G > kMaxGroups || a.K % BK != 0 || a.kseg % BK != 0 || a.d % 16 != 0)
        return cudaErrorInvalidValue;
    CUtensorMap tW2, tX, tXs;
    if (!make_tmap_3d(&tW2, a.W2, a.kseg, a.d, (unsigned long long)a.G * a.nseg, BK, BF) ||
        !make_tmap_2d(&tX, a.H, a.K, a.H_rows, a.K, BK, Geo<false>::NT) ||
        !make_tmap_2d(&tXs, a.H, a.K, a.H_rows, a.K, BK, SMALL_ROWS))
        return cudaErrorInvalidValue;
    Params p{};
    p.offsets = a.offsets;
    p.G = a.G;
    p.M = a.M;
    p.f_tiles = (a.d + BF - 1) / BF;
    p.k_blocks = a.K / BK;
    p.w_rows = 0;
    p.kseg = a.kseg;
    p.nseg = a.nseg;
    p.out = a.Y;
    p.ldo = a.d;
    p.f_limit = a.d;
    p.a_rows = a.H_rows;
    p.status = status;
    return launch<false>(tW2, tW2, tX, tXs, p, num_sms, st);
}

}  // namespace moe
