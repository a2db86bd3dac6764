// Grouped GEMMs of the layer backward on the sm_100a tensor cores (2-SM
// tcgen05 MMA, TMEM accumulators, TMA), bf16 operands, fp32 accumulation and
// fp32 results ("Scaling Efficiency: A Deep Dive into the DeepSeek-V3
// Architecture", DeepSeekMoE sketch: one MLP per expert over the tokens
// routed to it -- its gradients are the same contractions transposed).
//
// Two kinds of launch, both over the groups (experts, or one shared group)
// of a padded row layout: group g owns rows [start[g], start[g] + rows[g]) of
// every per-row operand, and every group's segment is padded with zero rows
// up to a multiple of 64 (the rows past rows[g] are never written).
//
//   rows (input gradients): out[r][m] (+)= sum_k A_g(m, k) B(r, k) for the
//     rows r of group g -- the weight of the group is the MMA's M operand
//     (256 of its output features per CTA pair), the group's rows the N
//     operand (token tiles of <= 256 rows, as in the forward).  A is read
//     MN-major (u = dy W2, dx = da W1 + dg W3: the weights read along their
//     output dimension from their natural [out][in] layout, no transposed
//     copy); for dx the contraction runs over W1's rows and then W3's (two
//     tensor maps).  The template keeps the K-major form of A as well; the
//     recompute of a = x W1^T and g = x W3^T, which read it so, runs in the
//     forward's gate/up kernel instead (h comes out of the same launch).
//   wgrad (weight gradients): out_g[m][n] = sum_{r in g} A(r, m) B(r, n) --
//     M and N the weight's two dimensions (256 x 256 tiles per CTA pair), the
//     contraction over the group's padded rows (64 per stage, the zero rows
//     add nothing); both operands MN-major straight from the per-row
//     matrices (dW2 = do^T h, dW1 = da^T x, dW3 = dg^T x).  A group without
//     rows gets a zero gradient.
//
// MN-major operand tiles are loaded as boxes of 64 K-rows x 64 M (or N)
// elements (128-byte swizzle), two per CTA for 128 M rows: the shared-memory
// descriptor's leading byte offset steps between those 64-element atoms and
// its stride byte offset between 8-row groups along K; an MMA of K = 16 then
// starts 16 rows (2 KB) further.  K-major tiles are those of the forward.
//
// Warp roles per CTA: 0 loads A (the leader's lane also arms the stage
// barrier with both CTAs' bytes), 1 owns TMEM and in the leader issues the
// MMAs, 2-5 are the epilogue, 6 loads B.  Tiles are dealt to the CTA pairs
// round-robin; every role walks the same sequence.  Every wait is bounded
// (common.cuh); on a timeout the CTA raises its abort flag, drains and exits.
#include "common.cuh"
#include "kernels.h"
#include "tmap.h"

namespace moe {
namespace {

constexpr int BK = 64;
constexpr int MAX_STAGES = 6;
constexpr int A_BYTES = 128 * BK * 2;
constexpr int B_BYTES = 128 * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NT = 256;
constexpr int NXBOX = 8;  // token boxes of 16, 32, ..., 128 rows (K-major B)
constexpr uint32_t ACC_COLS = 256;
constexpr uint32_t TMEM_COLS = 512;
// The weight-gradient kind has short K loops (a group's rows) and 128 KB of
// fp32 results per CTA and tile: it runs eight epilogue warps (each quarter
// of TMEM lanes read by two, one per column half) and four stages; the rows
// kind four epilogue warps and six stages.
template <bool WG>
__host__ __device__ constexpr int n_epi() {
    return WG ? 8 : 4;
}
template <bool WG>
__host__ __device__ constexpr int n_stages() {
    return WG ? 4 : 6;
}
template <bool WG>
__host__ __device__ constexpr int n_threads() {
    return 32 * (3 + n_epi<WG>());
}
constexpr int XS = 132;
constexpr int XBUF_BYTES = 16 * XS * 4;
constexpr int kMaxBwdGroups = kMaxGroups + 1;

struct Ctl {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
struct Tables {
    int rowstart[kMaxBwdGroups];
    int rows[kMaxBwdGroups];
    int ttiles[kMaxBwdGroups];  // rows: token tiles; wgrad: 1
    int prefix[kMaxBwdGroups + 1];
};
// epilogue staging: rows, two exchange buffers; wgrad, two 4 KB output boxes per epilogue warp
template <bool WG>
__host__ __device__ constexpr size_t xbuf_bytes() {
    return WG ? (size_t)n_epi<WG>() * 2 * 4096 : 2 * (size_t)XBUF_BYTES;
}
template <bool WG>
__host__ __device__ constexpr size_t smem_bytes() {
    return 1024 + (size_t)n_stages<WG>() * STAGE_BYTES + xbuf_bytes<WG>() + sizeof(Ctl) + sizeof(Tables);
}
static_assert(smem_bytes<false>() <= 232448 && smem_bytes<true>() <= 232448, "shared memory budget");
static_assert(n_stages<false>() <= MAX_STAGES && n_stages<true>() <= MAX_STAGES, "ring depth");

struct Maps {
    CUtensorMap a0, a1;   // A: the weights (rows) or the per-row matrix (wgrad); a1: dx's W3
    CUtensorMap b;        // wgrad: MN-major B
    CUtensorMap bx[NXBOX];  // rows: K-major token boxes
    CUtensorMap o;        // wgrad: the fp32 output [G][M_total][N_total], stored in 32 x 32 boxes
};

struct BwdParams {
    int G;
    const int32_t* start;   // group row starts (padded layout); null: one group of M_rows rows from 0
    const int32_t* rows;    // group row counts
    int M_rows;
    long long op_rows;      // rows of the per-row operands (bounds of start/rows)
    int M_total;            // rows: output features; wgrad: dW rows
    int N_total;            // wgrad: dW columns
    int m_tiles, n_tiles;   // 256-wide tiles over M_total (and N_total)
    int k_blocks;           // rows: K / 64
    int k_split;            // rows with two A maps: K blocks read from a0 (then a1); 0 = all from a0
    long long a_grow;       // rows, K-major A: map row of group g = g * a_grow + m; MN-major A: K row = g * a_grow + k
    float* out;
    long long out_gstride;  // wgrad: elements between groups' gradients
    int ldo;                // output row pitch (elements)
    int accumulate;         // rows: out += result
    int* status;
};

__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)(8192u >> 4) << 16;  // next 64-element atom along M / N
    d |= (uint64_t)(1024u >> 4) << 32;  // next 8 rows along K
    d |= 1ull << 46;
    d |= 2ull << 61;
    return d;
}

// 32 lanes x 32 bits, 32 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void token_tile(int rows, int ntt, int tt, int& start, int& len) {
    const int q = rows / ntt, r = rows - q * ntt;
    start = tt * q + min(tt, r);
    len = q + (tt < r ? 1 : 0);
}

struct Tile {
    int g, a, b;  // rows: (group, feature tile, token tile); wgrad: (group, m tile, n tile)
};
__device__ __forceinline__ Tile tile_of(const Tables* tb, int G, int per_group_a, int tile) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tb->prefix[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int q = tile - tb->prefix[lo];
    const int nb = tb->ttiles[lo];
    (void)per_group_a;
    return {lo, q / nb, q - (q / nb) * nb};
}

__device__ __forceinline__ bool wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag, int* status) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0;; ++it) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (ok) return true;
        if ((it & 63u) == 63u) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                *abort_flag = 1;
                report(status, kStTimeout);
                return false;
            }
        }
    }
}

__device__ __forceinline__ void settle_loads() {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) {
    }
}

// Per tile, what every role needs: K blocks and, for the rows kind, the
// token tile.
struct TileInfo {
    int kb;      // K blocks
    int tok0;    // rows: first row of the tile; wgrad: first row of the group
    int ntok;    // rows: rows of the tile; wgrad: N columns of the tile (<= 256)
    int m0;      // first M row of the pair's tile
    int n0;      // wgrad: first N column
};

template <bool WG>
__device__ __forceinline__ TileInfo tile_info(const Tables* tb, const BwdParams& p, const Tile& t) {
    TileInfo ti;
    ti.m0 = t.a * 256;
    if (WG) {
        ti.kb = (tb->rows[t.g] + BK - 1) / BK;
        ti.tok0 = tb->rowstart[t.g];
        ti.n0 = t.b * 256;
        ti.ntok = min(256, p.N_total - ti.n0);
    } else {
        ti.kb = p.k_blocks;
        int ts, len;
        token_tile(tb->rows[t.g], tb->ttiles[t.g], t.b, ts, len);
        ti.tok0 = tb->rowstart[t.g] + ts;
        ti.ntok = len;
        ti.n0 = 0;
    }
    return ti;
}

template <bool AMN, bool BMN, bool WG>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(n_threads<WG>(), 1)
    tc_bwd_gemm_kernel(const __grid_constant__ Maps mp, const BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* ring = base;
    constexpr int STAGES = n_stages<WG>();
    constexpr int NEPI = n_epi<WG>();
    constexpr int NTHREADS = n_threads<WG>();
    float* xbuf = reinterpret_cast<float*>(base + STAGES * STAGE_BYTES);
    Ctl* ctl = reinterpret_cast<Ctl*>(base + STAGES * STAGE_BYTES + xbuf_bytes<WG>());
    Tables* tb = reinterpret_cast<Tables*>(ctl + 1);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int G = p.G;

    for (int g = tid; g < G; g += NTHREADS) {
        int rs = p.start ? p.start[g] : 0;
        int rows = p.start ? p.rows[g] : p.M_rows;
        if (rs < 0 || rows < 0 || (long long)rs + rows > p.op_rows) {
            report(p.status, kStDeviceCheck);
            rs = 0;
            rows = 0;
        }
        tb->rowstart[g] = rs;
        tb->rows[g] = rows;
        tb->ttiles[g] = WG ? p.n_tiles : (rows + NT - 1) / NT;
    }
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&ctl->tfull[a], 1);
            mbar_init(&ctl->tempty[a], 2 * NEPI);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&ctl->tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    __syncthreads();
    if (warp == 0) {  // exclusive prefix of per-group tile counts (wgrad: m tiles x n tiles per group)
        int carry = 0;
        for (int b = 0; b < G; b += 32) {
            const int g = b + lane;
            const int v = g < G ? tb->ttiles[g] * p.m_tiles : 0;
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
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    const int total = tb->prefix[G];
    const uint32_t leader_full = mapa_shared(smem_u32(&ctl->full[0]), 0);

    if (warp == 0) {
        // ------------------------------------------------ A producer (both CTAs)
        if (lane == 0) {
            tma_prefetch_desc(&mp.a0);
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued = false;
            for (int tile = pair; tile < total && ok; tile += npairs) {
                const Tile t = tile_of(tb, G, p.m_tiles, tile);
                const TileInfo ti = tile_info<WG>(tb, p, t);
                const int mrow = ti.m0 + (int)rank * 128;  // this CTA's first M row
                // bytes of both CTAs per stage: A 16 KB each, B by kind
                uint32_t bbytes;
                if (WG) {
                    const int ncta = ((ti.ntok + 127) / 128) * 64;  // N columns per CTA (64 or 128)
                    bbytes = (uint32_t)ncta * 128u;
                } else {
                    const int half = ((ti.ntok + 15) & ~15) >> 1;
                    bbytes = (uint32_t)((half + 15) & ~15) * 128u;
                }
                const uint32_t tx = 2u * ((uint32_t)A_BYTES + bbytes);
                for (int kb = 0; kb < ti.kb; ++kb) {
                    if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, &ctl->abort, p.status)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&ctl->full[stage], tx);
                    uint8_t* sa = ring + stage * STAGE_BYTES;
                    const uint32_t fb = leader_full + 8u * (uint32_t)stage;
                    if (AMN) {
                        // K rows: the weights' rows (rows kind: W2 rows o, or W1 then W3 rows i of group g),
                        // or the group's operand rows (wgrad); M columns: this CTA's 128, two 64-wide atoms
                        const CUtensorMap* am = &mp.a0;
                        int kb_local = kb;
                        if (!WG && p.k_split > 0 && kb >= p.k_split) {
                            am = &mp.a1;
                            kb_local = kb - p.k_split;
                        }
                        const int krow = WG ? ti.tok0 + kb * BK : (int)((long long)t.g * p.a_grow) + kb_local * BK;
                        tma_load_2d_pair(sa, am, fb, mrow, krow, kEvictNormal);
                        tma_load_2d_pair(sa + 8192, am, fb, mrow + 64, krow, kEvictNormal);
                    } else {
                        tma_load_2d_pair(sa, &mp.a0, fb, kb * BK, (int)((long long)t.g * p.a_grow) + mrow,
                                         kEvictNormal);
                    }
                    issued = true;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && issued) settle_loads();
        }
        __syncwarp();
    } else if (warp == 2 + NEPI) {
        // ------------------------------------------------ B producer (both CTAs)
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true, issued = false;
            for (int tile = pair; tile < total && ok; tile += npairs) {
                const Tile t = tile_of(tb, G, p.m_tiles, tile);
                const TileInfo ti = tile_info<WG>(tb, p, t);
                for (int kb = 0; kb < ti.kb; ++kb) {
                    if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, &ctl->abort, p.status)) {
                        ok = false;
                        break;
                    }
                    uint8_t* sb = ring + stage * STAGE_BYTES + A_BYTES;
                    const uint32_t fb = leader_full + 8u * (uint32_t)stage;
                    if (WG) {  // MN-major: N columns of this CTA, 64 per box
                        const int ncta = ((ti.ntok + 127) / 128) * 64;
                        const int ncol = ti.n0 + (int)rank * ncta;
                        for (int j = 0; j < ncta; j += 64)
                            tma_load_2d_pair(sb + (j / 64) * 8192, &mp.b, fb, ncol + j, ti.tok0 + kb * BK,
                                             kEvictNormal);
                    } else {  // K-major token rows: this CTA's half of the tile
                        const int half = ((ti.ntok + 15) & ~15) >> 1;
                        const int hb = ((half + 15) & ~15) / 16 - 1;
                        tma_load_2d_pair(sb, &mp.bx[hb], fb, kb * BK, ti.tok0 + (int)rank * half, kEvictNormal);
                    }
                    issued = true;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && issued) settle_loads();
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader CTA)
        if (rank == 0 && elect_one()) {
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int tile = pair; tile < total; tile += npairs) {
                const Tile t = tile_of(tb, G, p.m_tiles, tile);
                const TileInfo ti = tile_info<WG>(tb, p, t);
                int n_mma;
                if (WG) n_mma = ((ti.ntok + 127) / 128) * 128;
                else n_mma = (ti.ntok + 15) & ~15;
                const uint32_t idesc = idesc_bf16(256, n_mma, AMN, BMN);
                if (!wait_cluster(&ctl->tempty[acc], acc_phase ^ 1u, &ctl->abort, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * ACC_COLS;
                for (int kb = 0; kb < ti.kb; ++kb) {
                    if (!mbar_wait(&ctl->full[stage], phase, &ctl->abort, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(ring + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {  // K = 16 per MMA
                        const uint64_t ad = AMN ? desc_mn_sw128(sa + (uint32_t)kk * 2048u)
                                                : smem_desc_sw128(sa) + (uint64_t)(2 * kk);
                        const uint64_t bd = BMN ? desc_mn_sw128(sb + (uint32_t)kk * 2048u)
                                                : smem_desc_sw128(sb) + (uint64_t)(2 * kk);
                        tc_mma_bf16_pair(d_tmem, ad, bd, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit_pair(&ctl->empty[stage], 0x3);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit_pair(&ctl->tfull[acc], 0x3);  // also with no MMA: the epilogue then writes zeros
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok) {
                tc_commit_pair(&ctl->drain, 0x1);
                mbar_wait_drain(&ctl->drain, 0);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (both CTAs, warps 2 .. 1 + NEPI)
        const int q = warp & 3;  // TMEM lane quarter
        const int e = tid - 64;  // 0..127
        const int my_tok = e >> 3, part = e & 7;
        const uint32_t leader_tempty = mapa_shared(smem_u32(&ctl->tempty[0]), 0);
        int acc = 0, xb = 0;
        uint32_t acc_phase = 0;
        for (int tile = pair; tile < total; tile += npairs) {
            const Tile t = tile_of(tb, G, p.m_tiles, tile);
            const TileInfo ti = tile_info<WG>(tb, p, t);
            if (!mbar_wait(&ctl->tfull[acc], acc_phase, &ctl->abort, p.status)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * ACC_COLS;
            const int mcta = ti.m0 + (int)rank * 128;  // this CTA's first M row
            if (WG) {
                // D[m][n]: lane = m, column = n; warp w reads lane quarter w % 4, column half (w - 2) / 4.
                // Per 32 columns the warp's 32 x 32 block goes through one of its two 4 KB shared-memory
                // boxes (128-byte swizzled rows: 16-byte chunk j of row r at j ^ (r % 8)) and leaves as one
                // TMA store, whole 128-byte lines; rows past M_total are clipped by the map.  The TMEM
                // read of the next 32 columns and the store of the previous box run meanwhile.
                const int ew = warp - 2;
                const int c_lo = (ew >> 2) * 128, c_hi = min(c_lo + 128, ti.ntok);
                const int mq = mcta + q * 32;
                uint32_t r0[32], r1[32];
                const auto store32 = [&](int c, const uint32_t (&v)[32]) {
                    float* sb = xbuf + ew * 2048 + xb * 1024;
                    if (lane == 0) bulk_wait_group_read<1>();  // the store that last used this box has read it
                    __syncwarp();
                    float4* srow = reinterpret_cast<float4*>(sb + lane * 32);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        srow[i ^ (lane & 7)] =
                            ti.kb > 0 ? make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                    __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]))
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(&mp.o, sb, ti.n0 + c, mq, t.g);
                        bulk_commit_group();
                    }
                    xb ^= 1;
                };
                const bool live = mq < p.M_total && c_lo < c_hi;  // warp-uniform: nothing of this warp's to store
                if (live && ti.kb > 0) tmem_ld32(taddr + (uint32_t)c_lo, r0);
                for (int c = c_lo; live && c < c_hi; c += 64) {  // the tile's columns come in multiples of 128
                    if (ti.kb > 0) {
                        tmem_ld_wait();
                        tmem_ld32(taddr + (uint32_t)(c + 32), r1);
                    }
                    store32(c, r0);
                    if (ti.kb > 0) {
                        tmem_ld_wait();
                        if (c + 64 < c_hi) tmem_ld32(taddr + (uint32_t)(c + 64), r0);
                    }
                    store32(c + 32, r1);
                }
            } else {
                // D[m][token]: 16-token chunks through shared memory, token-major fp32 rows
                const int ntok = ti.ntok;
                for (int c = 0; c < ntok; c += 16) {
                    uint32_t r[16];
                    tmem_ld16(taddr + (uint32_t)c, r);
                    tmem_ld_wait();
                    float* xs = xbuf + xb * (XBUF_BYTES / 4);
#pragma unroll
                    for (int i = 0; i < 16; ++i) xs[i * XS + q * 32 + lane] = __uint_as_float(r[i]);
                    named_bar_sync(1, 128);
                    const int fj = part * 16;
                    if (c + my_tok < ntok && mcta + fj < p.M_total) {
                        const float* row = xs + my_tok * XS + fj;
                        float4* dst = reinterpret_cast<float4*>(p.out + (size_t)(ti.tok0 + c + my_tok) * p.ldo +
                                                                mcta + fj);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            float4 v = *reinterpret_cast<const float4*>(row + 4 * i);
                            if (p.accumulate) {
                                const float4 o = dst[i];
                                v.x += o.x;
                                v.y += o.y;
                                v.z += o.z;
                                v.w += o.w;
                            }
                            dst[i] = v;
                        }
                    }
                    xb ^= 1;  // the next chunk writes the other buffer; its barrier orders the reuse
                }
            }
            tc_fence_before();
            __syncwarp();
            // the accumulator's tcgen05.ld have completed (wait::ld above): a relaxed arrive frees it (a
            // cluster-scope release here cost about 1 us per tile and warp)
            if (lane == 0) mbar_arrive_relaxed_cluster(leader_tempty + 8u * (uint32_t)acc);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
    }

    if (WG && warp >= 2 && warp < 2 + NEPI && lane == 0) bulk_wait_group<0>();  // the output boxes are written
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

template <bool AMN, bool BMN, bool WG>
cudaError_t launch_bwd(const Maps& m, const BwdParams& p, int num_sms, cudaStream_t st) {
    auto kern = tc_bwd_gemm_kernel<AMN, BMN, WG>;
    constexpr size_t SMEM_BYTES = smem_bytes<WG>();
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (err != cudaSuccess) return err;
    const int grid = (num_sms / 2) * 2;
    kern<<<grid, n_threads<WG>(), SMEM_BYTES, st>>>(m, p);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace

// rows kind, A MN-major: out[r][m] (+)= sum_k W(k, m) X[r][k] with W(k, m) =
//   W0[g * a_grow + k][m] for k < K0, then W1[g * a_grow + k - K0][m];
//   W0/W1: [Wrows][M_total] bf16 (rows along K), X: [op_rows][K0 + K1] bf16.
cudaError_t launch_bwd_rows_mnmajor(const BwdRowsArgs& a, int* status, int num_sms, cudaStream_t st) {
    Maps m{};
    if (a.K % BK != 0 || a.M_total % 128 != 0 || (a.W1 && a.K0 % BK != 0)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&m.a0, a.W, a.M_total, a.W_rows, a.M_total, 64, 64) ||
        !make_tmap_2d(&m.a1, a.W1 ? a.W1 : a.W, a.M_total, a.W_rows, a.M_total, 64, 64))
        return cudaErrorInvalidValue;
    for (int b = 0; b < NXBOX; ++b)
        if (!make_tmap_2d(&m.bx[b], a.X, a.K, a.op_rows, a.K, 64, 16 * (b + 1))) return cudaErrorInvalidValue;
    m.b = m.a0;
    BwdParams p{};
    p.G = a.G;
    p.start = a.start;
    p.rows = a.rows;
    p.M_rows = a.M_rows;
    p.op_rows = a.op_rows;
    p.M_total = a.M_total;
    p.m_tiles = (a.M_total + 255) / 256;
    p.n_tiles = 1;
    p.k_blocks = a.K / BK;
    p.k_split = a.W1 ? a.K0 / BK : 0;
    p.a_grow = a.a_grow;
    p.out = a.out;
    p.ldo = a.ldo;
    p.accumulate = a.accumulate ? 1 : 0;
    p.status = status;
    return launch_bwd<true, false, false>(m, p, num_sms, st);
}

// wgrad kind: out[g][m][n] = sum over group g's padded rows r of A[r][a_col0 + m] * B[r][b_col0 + n]
//   A: [op_rows][lda] bf16, B: [op_rows][ldb] bf16, out: [G][M_total][N_total] fp32.
cudaError_t launch_bwd_wgrad(const BwdWgradArgs& a, int* status, int num_sms, cudaStream_t st) {
    Maps m{};
    // M: the 64-wide boxes past M_total read zeros and those rows are not stored; N: whole 128-column halves
    if (a.M_total % 8 != 0 || a.N_total % 128 != 0) return cudaErrorInvalidValue;
    // the boxes start at column a_col0 + m (b_col0 + n): a view that begins there keeps the 16-byte rule
    const uint16_t* A = static_cast<const uint16_t*>(a.A) + a.a_col0;
    const uint16_t* B = static_cast<const uint16_t*>(a.B) + a.b_col0;
    if ((reinterpret_cast<uintptr_t>(A) & 15u) || (reinterpret_cast<uintptr_t>(B) & 15u)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&m.a0, A, a.M_total, a.op_rows, a.lda, 64, 64) ||
        !make_tmap_2d(&m.b, B, a.N_total, a.op_rows, a.ldb, 64, 64))
        return cudaErrorInvalidValue;
    m.a1 = m.a0;
    for (int b = 0; b < NXBOX; ++b) m.bx[b] = m.b;
    if ((reinterpret_cast<uintptr_t>(a.out) & 15u) ||
        !make_tmap_3d_f32(&m.o, a.out, a.N_total, a.M_total, a.G, a.N_total, (unsigned long long)a.M_total * a.N_total,
                          32, 32))
        return cudaErrorInvalidValue;
    BwdParams p{};
    p.G = a.G;
    p.start = a.start;
    p.rows = a.rows;
    p.M_rows = a.M_rows;
    p.op_rows = a.op_rows;
    p.M_total = a.M_total;
    p.N_total = a.N_total;
    p.m_tiles = (a.M_total + 255) / 256;
    p.n_tiles = (a.N_total + 255) / 256;
    p.k_blocks = 0;
    p.k_split = 0;
    p.a_grow = 0;
    p.out = a.out;
    p.out_gstride = (long long)a.M_total * a.N_total;
    p.ldo = a.N_total;
    p.accumulate = 0;
    p.status = status;
    return launch_bwd<true, true, true>(m, p, num_sms, st);
}

}  // namespace moe
