// Grouped expert GEMMs on the sm_100a tensor cores (2-SM tcgen05 MMA, TMEM,
// TMA) for bf16 and block-scaled E4M3 experts ("Scaling Efficiency: A Deep Dive into the
// DeepSeek-V3 Architecture", DeepSeekMoE sketch: one MLP per expert over the
// tokens routed to it; "DeepSeek V3 Architecture Deep Dive ...", "Throughput
// on NVIDIA H100/H800": tokens of one expert batched together).
//
//   up:   h[t][f] = silu(W1_g[f] . a[t]) * (W3_g[f] . a[t])   (SwiGLU fused)
//   down: y[t][o] = W2_g[o] . h[t]
//
// Swap-AB: the expert's weights are the MMA's M operand and its tokens the N
// operand.  N only has to be a multiple of 16, so an expert's tokens are cut
// into ceil(rows / 256) tiles of equal size, each rounded up to 16, instead
// of padding 128-row M tiles (padded MMA work on the V3 routing drops from
// ~25% to a few percent).
//
// Each tile runs on a cluster of two CTAs (two SMs) sharing one
// cta_group::2 MMA of M = 256 weight rows (128 in each CTA's shared memory)
// by N <= 256 tokens (N/2 rows in each CTA); each CTA's TMEM receives its 128
// rows of the result.  Per SM and K step that is 16 KB of weights + 16 KB of
// tokens for 128 x 256 x 64 MMA work -- a third fewer operand bytes per FLOP
// than a one-SM 128 x 256 tile, and 32 KB stages allow a 6-deep TMA ring.
//
//   up tile:   each CTA holds 64 rows of W1 and the same 64 rows of W3, so
//              its TMEM lanes 0-63 hold gate and 64-127 up of its 64 output
//              features; the epilogue pairs them through shared memory.
//   down tile: each CTA holds 128 rows of W2 (its 128 output features).
// The weights stay in their natural [out][in] layout (no packing pass).
//
// One persistent cluster per SM pair takes tiles from a device-side tile list
// built from the expert offsets (no host read-back), in list order, through
// a global atomic counter: the tiles in flight are always a window of about
// one tile per cluster, so the clusters sharing an expert's token rows (its
// feature tiles) or a weight tile (its token tiles) run at the same time and
// find them in L2, and the last tiles spread over the clusters that are free.
// Per expert, token tiles are walked fastest, then feature tiles.
//
// Warp roles per CTA (bf16 up: 12 warps, down: 7; E4M3 up: 13, down: 12):
//   warp 0      weight producer (one lane), both CTAs: loads this CTA's
//               weight rows (up: the W1 half), completion counted on the
//               leader CTA's stage barrier, which the leader's lane arms with
//               both CTAs' bytes.  The leader's warp 0 also takes tiles from
//               the counter and posts them in a small tile queue in both
//               CTAs' shared memory for every other role, one tile ahead of
//               its own loads (the atomic's round trip overlaps the current
//               tile's loads).
//   warp 1      TMEM owner (paired allocation); in the leader (even) CTA one
//               lane issues the MMAs and commits to both CTAs' barriers.
//   warps 2..   epilogue (up and E4M3 down: 8 warps, bf16 down: 4): tcgen05.ld 32 lanes x 16
//               tokens into shared memory, SwiGLU / bf16 conversion,
//               token-major vector stores.  Two 256-column TMEM accumulators
//               let the epilogue of one tile overlap the main loop of the next.
//   then        the token-operand producer, and for up the W3-half producer:
//               they follow the tile queue and fill their part of each stage.
//               A thread that issues a TMA tile load stalls for roughly as
//               long as the unit takes to accept its bytes, so one thread
//               issuing all of a stage's loads left the tensor pipe waiting;
//               spreading a stage's loads over warps measured the up
//               projection 13-15% and the V3 step 7% faster.  E4M3: one
//               more warp loads each stage's tile scales (weight atom and
//               token image) onto the same stage barrier.
// Every wait is bounded (common.cuh); on a timeout the CTA raises its abort
// flag, drains what it issued, frees TMEM and exits (the peer then times out
// on its next wait and does the same).
#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "tmap.h"

namespace moe {
namespace {

constexpr int BK = 64;                  // bf16 K per stage: one 128-byte swizzle row
// K elements per stage for the operand type: 64 bf16 or 128 E4M3 (128 bytes either way)
template <bool F8>
__host__ __device__ constexpr int bk_elems() { return F8 ? 128 : 64; }
// Ring depth of the operand tiles (an E4M3 stage also carries its tile scales)
template <bool UP, bool F8>
__host__ __device__ constexpr int n_stages() { return 6; }
constexpr int A_BYTES = 128 * BK * 2;   // this CTA's 128 weight rows
constexpr int B_ROWS = 128;             // this CTA's half of <= 256 tokens
constexpr int B_BYTES = B_ROWS * BK * 2;
// Token rows are loaded with one box per K step whose height is the CTA's
// half of the tile rounded up to 16 rows (16, 32, ..., 128: one tensor map
// each); a fixed 128-row box would bring in up to 60% rows of no use on
// balanced tiles.
constexpr int NXBOX = B_ROWS / 16;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 32 KB
constexpr uint32_t ACC_COLS = 256;      // one accumulator buffer
constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
// E4M3 with per-tile scales (block-scaled MMA): the scales of a stage sit in
// tensor memory beside the accumulators, so the second accumulator gives up
// 16 columns and holds tiles of at most 240 tokens (larger ones use the
// first).  Every ring stage has a scale slot of its own: this CTA's 128
// weight rows x 4 tiles (one 512-byte atom, 4 columns) and the tile's token
// image (up to 256 tokens x 4 tiles, 1024 bytes, 8 columns), both brought by
// TMA onto the stage's full barrier, so the MMA issuer waits once per stage
// for operands and scales alike.
constexpr uint32_t ACC1_COLS_F8 = 240;
constexpr uint32_t SFA_COL = 496, SFB_COL = 504;
constexpr int SFA_BYTES = 512, SFB_BYTES = 1024, SF_STAGE_BYTES = SFA_BYTES + SFB_BYTES;
// Epilogue warps come in groups of four (one per TMEM lane quarter); groups
// take the tile's 16-token chunks in turn.  The gate/up epilogue (SwiGLU on
// every element) runs two groups with one exchange buffer each.  The bf16
// down epilogue, a plain conversion, runs one group with two buffers: a
// second group there took issue slots from the producer lanes and measured
// 10% slower on the V3 down projection.  The E4M3 down projection (16 K steps
// of 128 per tile at I = 2048) runs two groups: with one, its epilogue paced
// the launch (the MMA issuer waited for a free accumulator 28% of its time).
template <bool UP, bool F8>
__host__ __device__ constexpr int n_epi_warps() { return UP || F8 ? 8 : 4; }
template <bool UP, bool F8>
__host__ __device__ constexpr int n_xbuf_per_group() { return UP || F8 ? 1 : 2; }
// producer warps after the epilogue warps: the token operand (both), the W3 half (up),
// the tile scales (E4M3)
template <bool UP, bool F8>
__host__ __device__ constexpr int n_extra_producers() { return (UP ? 2 : 1) + (F8 ? 1 : 0); }
template <bool UP, bool F8>
__host__ __device__ constexpr int n_threads() { return 32 * (2 + n_epi_warps<UP, F8>() + n_extra_producers<UP, F8>()); }
constexpr int XS = 132;                 // row stride (floats) of the epilogue exchange buffer
constexpr int XBUF_BYTES = 16 * XS * 4; // 16 tokens x 128 lanes (+pad), fp32
// L2 policy of the two operands' loads.  Marking the weights evict-first
// (each weight box is read by at most two clusters) and the token rows
// evict-last (re-read by every feature tile of the expert) measured 3.5%
// slower on the V3 step than the normal policy for both.
constexpr uint64_t W_HINT = kEvictNormal;
constexpr uint64_t X_HINT = kEvictNormal;
constexpr int TQ = 8;                   // tile queue slots
// readers of a queue slot, in each CTA: the epilogue warps, the extra producers, and
// the MMA issuer (leader) or the weight producer (peer)
template <bool UP, bool F8>
__host__ __device__ constexpr uint32_t tq_readers() {
    return 2u * (1u + (uint32_t)n_epi_warps<UP, F8>() + (uint32_t)n_extra_producers<UP, F8>());
}

// Tile counters: one {next, done} pair per launch slot.  A launch takes the
// next slot round-robin on the host; the last cluster to finish resets its
// pair to zero, so every launch starts from a zero counter without a memset.
// Two launches share a pair only if 1024 launches were enqueued in between
// while the first is still running.
constexpr int kSchedSlots = 1024;
__device__ unsigned int g_tile_sched[kSchedSlots][2];


constexpr int MAX_STAGES = 6;
struct Ctl {
    uint64_t full[MAX_STAGES];
    uint64_t empty[MAX_STAGES];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t tq_full[TQ];   // in both CTAs: slot holds the next tile
    uint64_t tq_empty[TQ];  // leader only: every reader has taken the slot's tile
    uint64_t drain;
    int tq[TQ];             // tile index, or -1 when the list is exhausted
    uint32_t tmem_base;
    int abort;
};
constexpr int kMaxTcGroups = kMaxGroups + 1;  // routed experts + the shared set
struct Tables {
    int rowstart[kMaxTcGroups];
    int rows[kMaxTcGroups];
    int ttiles[kMaxTcGroups];  // token tiles per group
    int fgroup[kMaxTcGroups];  // > 0: the group's tiles run in groups of this many feature tiles (see tile_coords)
    int tbase[kMaxTcGroups];   // routed groups: index of the group's first token tile among all routed groups
    int prefix[kMaxTcGroups + 1];
};
// The shared set's gate/up tiles (every token x S * Is features: 32 token
// tiles x 16 feature tiles at V3) run in groups of SHARED_FGROUP feature
// tiles, token tile by token tile inside a group, so the clusters in flight
// share 8 weight tiles (29 MB) and a few token tiles, and the token rows
// (x, 117 MB) are streamed twice instead of once per feature tile: V3 gate/up
// DRAM reads 18.4 -> 17.3 GB, the skewed batch's gate/up 4.5% faster.
constexpr int SHARED_FGROUP = 8;
constexpr size_t XBUF_TOTAL = 2 * (size_t)XBUF_BYTES;  // groups x buffers per group = 2 either way
static_assert(n_epi_warps<true, false>() / 4 * n_xbuf_per_group<true, false>() == 2, "exchange buffers");
static_assert(n_epi_warps<true, true>() / 4 * n_xbuf_per_group<true, true>() == 2, "exchange buffers");
static_assert(n_epi_warps<false, false>() / 4 * n_xbuf_per_group<false, false>() == 2, "exchange buffers");
static_assert(n_epi_warps<false, true>() / 4 * n_xbuf_per_group<false, true>() == 2, "exchange buffers");
// ring, tile scales (E4M3), epilogue exchange buffers, control, tables
template <bool UP, bool F8>
__host__ __device__ constexpr size_t sf_region_bytes() { return F8 ? (size_t)n_stages<UP, F8>() * SF_STAGE_BYTES : 0; }
template <bool UP, bool F8>
__host__ __device__ constexpr size_t smem_bytes() {
    return 1024 + (size_t)n_stages<UP, F8>() * STAGE_BYTES + sf_region_bytes<UP, F8>() + XBUF_TOTAL + sizeof(Ctl) +
           sizeof(Tables);
}
static_assert(smem_bytes<false, false>() <= 232448 && smem_bytes<false, true>() <= 232448 &&
                  smem_bytes<true, false>() <= 232448 && smem_bytes<true, true>() <= 232448,
              "shared memory budget");
static_assert(n_stages<false, false>() <= MAX_STAGES && n_stages<false, true>() <= MAX_STAGES &&
                  n_stages<true, false>() <= MAX_STAGES && n_stages<true, true>() <= MAX_STAGES,
              "ring depth");


// Tensor maps of one expert set: weights (w1 only for the up projection),
// the token operand with box heights 16 * (i + 1) rows, and (E4M3) the tile
// scales.
struct SetMaps {
    CUtensorMap w0, w1;
    CUtensorMap x[NXBOX];
    CUtensorMap sfw, sfx;  // E4M3: weight scale atoms (512-byte rows), token images (1024-byte rows)
};

// One expert set in a launch: set 0 = the routed experts (groups [0, G0),
// rows from offsets), set 1 = the shared experts (group G0, rows [0, M)).
struct SetParams {
    int f_tiles;       // feature tiles (per CTA pair) per group
    int k_blocks;
    int w_rows;        // rows of one weight block: up I (W1/W3 per group), down d (W2 per block)
    int kseg, nseg;    // down: W2 block geometry along K
    void* out;
    int ldo;           // output row pitch (elements)
    int f_limit;       // valid output features
    long long a_rows;  // rows the groups may index (token operand rows, or gathered rows) = output rows
    // E4M3 operands only: the tile scales come through the set's scale maps
    // (SetMaps::sfw, sfx).  Weight atom row of the CTA's rows: up, unit
    // (g * w_rows + f) / 64 of the joint W1/W3 units; down, atom
    // (g * w_rows + f) / 128; row y = atom row * k_blocks + kb.  Token images:
    // row (tile image index) * k_blocks + kb.
    // down only, weighted combine fused into the epilogue: each output row is
    // scaled by its routing weight and added (fp32 atomics) into acc [T][ldo];
    // routed set: row r holds assignment a = row_tok[r], token a / row_k,
    // weight row_w[a]; shared set (row_tok null): row r is token r, weight 1.
    float* acc;
    const int32_t* row_tok;
    const float* row_w;
    int row_k;
    // up, E4M3 only, optional: h leaves as E4M3 codes q_out [rows][ldo] with
    // its tile scales as the down projection's token images q_img (same
    // tiles: image of tile i, stage s at q_img + (i * ldo / 128 + s) * 256
    // words), exactly what quantizing the bf16 h would give; out is then
    // unused.
    uint8_t* q_out;
    uint32_t* q_img;
    // up, bf16 only, optional: the fp32 pre-activations (gate rows into a_out,
    // up rows into g_out, [rows][ldo]) beside h.
    float* a_out;
    float* g_out;
};
struct Params {
    const int32_t* offsets;
    int G0;            // routed groups
    int has_shared;    // 1: group G0 is the shared set
    int M;             // rows of the shared set
    SetParams set[2];
    const int32_t* gather;  // up, routed set, optional: row r reads token row gather[r] / gather_div
    int gather_div;
    int sched_slot;         // this launch's tile counter pair
    int* status;
};

struct TileCoord {
    int g, ft, tt;
};

// Tile order inside a group: the token tiles of a feature tile run back to
// back, so the clusters that share a weight tile read it at about the same
// time and DRAM sees it once; the shared set's gate/up group runs in groups
// of feature tiles (fgroup, SHARED_FGROUP above).  (Running the feature tiles
// of one token tile back to back for every group with more token tiles than
// feature tiles cut the V3 gate/up DRAM reads to 17.5 GB but measured 12%
// slower on the skewed batch, whose hot experts have many token tiles.)
__device__ __forceinline__ TileCoord tile_coords(const Tables* tb, int G, int tile) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {  // last group whose first tile is <= tile (never an empty one)
        const int mid = (lo + hi + 1) >> 1;
        if (tb->prefix[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int q = tile - tb->prefix[lo];
    const int nt = tb->ttiles[lo];
    const int fg = tb->fgroup[lo];
    if (fg > 0) {  // groups of fg feature tiles; inside one, token tile by token tile
        const int nft = (tb->prefix[lo + 1] - tb->prefix[lo]) / nt;
        const int b = q / (fg * nt), r = q - b * (fg * nt);
        const int bf = min(fg, nft - b * fg);  // feature tiles in this group
        return {lo, b * fg + (r - (r / bf) * bf), r / bf};
    }
    return {lo, q / nt, q - (q / nt) * nt};
}

// Token tile tt of a group with `rows` tokens split into `ntt` tiles of
// near-equal size (<= kTokTile each, token_tile_split).  Equal sizes keep the
// clusters that share a weight tile at the same pace, so the weight tile is
// still in L2 when the slower one reads it (a small tail tile would run ahead
// and let L2 evict).
__device__ __forceinline__ void token_tile(int rows, int ntt, int tt, int& start, int& len) {
    token_tile_split(rows, ntt, tt, start, len);
}

// silu(a) = a / (1 + e^-a) with the hardware exponential and division: the
// result is rounded to bf16 right after, so their few-ulp fp32 error is far
// below the output's own rounding.
__device__ __forceinline__ float silu_fast(float a) { return __fdividef(a, 1.0f + __expf(-a)); }

// Four fp32 additions into global memory (16-byte aligned), no return value.
__device__ __forceinline__ void red_add_v4(float* p, float a, float b, float c, float d) {
    asm volatile("red.relaxed.gpu.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
                 "f"(d)
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&b);
}

// Bounded wait with cluster-scope acquire (for barriers the peer CTA arrives on).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  int* status) {
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

// Tile queue signalling.  No cluster-scope release is issued by the TMA
// producer or the MMA issuer: on B200 one such arrive per tile measured about
// 1 us of producer stall per tile (the loads of the next tile start late).
// The peer's slot is written with st.async, whose byte count completes the
// peer's barrier (armed by a relaxed remote expect-tx arrive), and readers
// free a slot with a relaxed arrive issued after the tile index was consumed.
__device__ __forceinline__ void st_async_u32(uint32_t cluster_addr, int v, uint32_t cluster_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];" ::"r"(cluster_addr),
                 "r"(v), "r"(cluster_bar)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx_remote(uint32_t cluster_bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.relaxed.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(cluster_bar),
                 "r"(bytes)
                 : "memory");
}

// Reader side of the tile queue: wait for slot j, take its tile, free the
// slot for the leader's producer.  Returns false on a timeout or abort.
__device__ __forceinline__ bool tq_take(Ctl* ctl, int j, uint32_t ph, uint32_t leader_tq_empty, int* tile,
                                        int* status) {
    if (!mbar_wait_cluster(&ctl->tq_full[j], ph, &ctl->abort, status)) return false;
    const int t = reinterpret_cast<volatile int*>(ctl->tq)[j];
    *tile = t;
    mbar_arrive_relaxed_cluster(leader_tq_empty + 8u * (uint32_t)j);
    return true;
}

// A producer other than warp 0: follows the tile queue; per tile, begin(tc)
// returns the tile's K steps; per K step it waits until the stage is free and
// load(kb, stage, leader_full_bar) issues this producer's part.  kWarp: the
// whole warp runs the loop (lane 0 waits, every lane may load); otherwise
// lane 0 alone calls it.  The stage barrier may see these bytes land before
// warp 0 arms it: its transaction count then stays negative until the
// arming, and the phase cannot complete before the arrive that comes with it.
template <int STAGES, bool kWarp, typename Begin, typename Load>
__device__ __forceinline__ void follow_tiles(Ctl* ctl, const Tables* tb, int G, uint32_t leader_tq_empty, int* status,
                                             uint8_t* ring, int lane, Begin&& begin, Load&& load) {
    const uint32_t leader_full = mapa_shared(smem_u32(&ctl->full[0]), 0);
    int stage = 0, j = 0;
    uint32_t phase = 0, tq_ph = 0;
    bool ok = true, issued_any = false;
    for (;;) {
        int tile = -1, got = 1;
        if (!kWarp || lane == 0) got = tq_take(ctl, j, tq_ph, leader_tq_empty, &tile, status) ? 1 : 0;
        if (kWarp) {
            got = __shfl_sync(0xffffffffu, got, 0);
            tile = __shfl_sync(0xffffffffu, tile, 0);
        }
        if (!got) {
            ok = false;
            break;
        }
        if (tile < 0) break;
        if (++j == TQ) {
            j = 0;
            tq_ph ^= 1u;
        }
        const int k_blocks = begin(tile_coords(tb, G, tile));
        for (int kb = 0; kb < k_blocks; ++kb) {
            int free_ = 1;
            if (!kWarp || lane == 0) free_ = mbar_wait(&ctl->empty[stage], phase ^ 1u, &ctl->abort, status) ? 1 : 0;
            if (kWarp) free_ = __shfl_sync(0xffffffffu, free_, 0);
            if (!free_) {
                ok = false;
                break;
            }
            load(kb, ring + stage * STAGE_BYTES, leader_full + 8u * (uint32_t)stage);
            issued_any = true;
            if (++stage == STAGES) {
                stage = 0;
                phase ^= 1u;
            }
        }
        if (!ok) break;
    }
    if (!ok && issued_any && lane == 0) settle_inflight_loads();
    if (kWarp) __syncwarp();
}

// Accumulator of the tile that follows one in accumulator `prev`: the other
// one, except that with tile scales in tensor memory the second holds at most
// ACC1_COLS_F8 tokens.  The MMA issuer and the epilogue both follow it.
template <bool F8>
__device__ __forceinline__ int next_acc(int prev, int n_mma) {
    const int a = prev ^ 1;
    return (F8 && a == 1 && n_mma > (int)ACC1_COLS_F8) ? 0 : a;
}

template <bool UP, bool F8>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(n_threads<UP, F8>(), 1)
    tc_grouped_gemm_kernel(const __grid_constant__ SetMaps ma, const __grid_constant__ SetMaps mb,
                           const __grid_constant__ CUtensorMap tmXg, const Params p) {
    constexpr int STAGES = n_stages<UP, F8>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* ring = base;
    uint8_t* sfr = base + STAGES * STAGE_BYTES;  // tile scales of each stage (E4M3)
    float* xbuf = reinterpret_cast<float*>(sfr + sf_region_bytes<UP, F8>());
    Ctl* ctl = reinterpret_cast<Ctl*>(reinterpret_cast<uint8_t*>(xbuf) + XBUF_TOTAL);
    constexpr int NEPI = n_epi_warps<UP, F8>();
    constexpr int NXB = n_xbuf_per_group<UP, F8>();
    constexpr int NTHREADS = n_threads<UP, F8>();
    Tables* tb = reinterpret_cast<Tables*>(ctl + 1);

    constexpr int BKE = bk_elems<F8>();
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = cluster_ctarank();  // 0 = leader (issues the MMAs)
    const int npairs = gridDim.x >> 1;
    const int G = p.G0 + p.has_shared;

    for (int g = tid; g < G; g += NTHREADS) {
        const bool sh = g >= p.G0;
        const int rs = sh ? 0 : p.offsets[g];
        const int re = sh ? p.M : p.offsets[g + 1];
        int rows = re - rs;
        if (rs < 0 || rows < 0 || (long long)re > p.set[sh ? 1 : 0].a_rows) {  // corrupt offsets: skip the group
            report(p.status, kStDeviceCheck);
            rows = 0;
        }
        tb->rowstart[g] = rows > 0 ? rs : 0;
        tb->rows[g] = rows;
        tb->ttiles[g] = token_tiles(rows);
        tb->fgroup[g] = UP && sh ? SHARED_FGROUP : 0;
    }
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&ctl->tfull[a], 1);
            mbar_init(&ctl->tempty[a], 2 * NEPI);  // every epilogue warp of both CTAs
        }
        for (int j = 0; j < TQ; ++j) {
            mbar_init(&ctl->tq_full[j], 1);
            mbar_init(&ctl->tq_empty[j], tq_readers<UP, F8>());
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
    if (warp == 0) {  // exclusive prefixes of per-group tile counts: all tiles, and the token tiles
        int carry = 0, tcarry = 0;
        for (int b = 0; b < G; b += 32) {
            const int g = b + lane;
            const int tt = g < G ? tb->ttiles[g] : 0;
            const int v = tt * p.set[g >= p.G0 ? 1 : 0].f_tiles;
            int incl = v, tincl = tt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n = __shfl_up_sync(0xffffffffu, incl, o);
                const int tn = __shfl_up_sync(0xffffffffu, tincl, o);
                if (lane >= o) {
                    incl += n;
                    tincl += tn;
                }
            }
            if (g < G) {
                tb->prefix[g] = carry + incl - v;
                tb->tbase[g] = g < p.G0 ? tcarry + tincl - tt : 0;
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
            tcarry += __shfl_sync(0xffffffffu, tincl, 31);
        }
        if (lane == 0) tb->prefix[G] = carry;
    }
    tc_fence_before();
    cluster_sync_all();  // both CTAs' barriers initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    const int total = tb->prefix[G];
    const uint32_t leader_tq_empty = mapa_shared(smem_u32(&ctl->tq_empty[0]), 0);

    constexpr int kTokWarp = 2 + NEPI;  // token-operand producer
    constexpr int kW3Warp = 3 + NEPI;   // up: W3-half producer
    constexpr int kSfWarp = (UP ? 4 : 3) + NEPI;  // E4M3: tile-scale producer
    const bool gather = UP && p.gather != nullptr;  // routed set only

    if (warp == 0) {
        // ------------------------------------------------ weight producer (both CTAs, lane 0)
        // The K loop is kept to a wait, the arming, one load and a few
        // additions: this lane paces the ring (an integer division per K step
        // here measured 10% on the down projection).
        if (lane == 0) {
            if (p.G0 > 0) tma_prefetch_desc(&ma.w0);
            if (p.has_shared) tma_prefetch_desc(&mb.w0);
            const uint32_t leader_full = mapa_shared(smem_u32(&ctl->full[0]), 0);
            const uint32_t peer_tq = mapa_shared(smem_u32(&ctl->tq[0]), 1);
            const uint32_t peer_tq_full = mapa_shared(smem_u32(&ctl->tq_full[0]), 1);
            unsigned int* sched = g_tile_sched[p.sched_slot];
            int stage = 0, tq_j = 0, post_j = 0;
            uint32_t phase = 0, tq_ph = 0, post_ph = 0;
            bool ok = true, issued_any = false;
            // leader: post a tile (index, or -1 = no more) to both CTAs' queue slot post_j
            auto post = [&](int t) -> bool {
                if (!mbar_wait_cluster(&ctl->tq_empty[post_j], post_ph ^ 1u, &ctl->abort, p.status)) return false;
                ctl->tq[post_j] = t;
                mbar_arrive(&ctl->tq_full[post_j]);  // CTA-scope release of the store above
                mbar_arrive_expect_tx_remote(peer_tq_full + 8u * (uint32_t)post_j, 4u);
                st_async_u32(peer_tq + 4u * (uint32_t)post_j, t, peer_tq_full + 8u * (uint32_t)post_j);
                if (++post_j == TQ) {
                    post_j = 0;
                    post_ph ^= 1u;
                }
                return true;
            };
            const auto take = [&](unsigned int t) { return t < (unsigned int)total ? (int)t : -1; };
            int cur = -1;
            unsigned int t_next = 0;
            if (rank == 0) {
                cur = take(atomicAdd(&sched[0], 1u));
                ok = post(cur);
                if (ok && cur >= 0) t_next = atomicAdd(&sched[0], 1u);
            }
            for (;;) {
                int tile = -1;
                if (rank == 0) {  // cur is posted; post the next one before loading cur
                    tile = ok ? cur : -1;
                    if (ok && cur >= 0) {
                        cur = take(t_next);
                        ok = post(cur);
                        if (ok && cur >= 0) t_next = atomicAdd(&sched[0], 1u);
                    }
                } else {
                    ok = tq_take(ctl, tq_j, tq_ph, leader_tq_empty, &tile, p.status);
                    if (++tq_j == TQ) {
                        tq_j = 0;
                        tq_ph ^= 1u;
                    }
                }
                if (!ok || tile < 0) break;
                const TileCoord tc = tile_coords(tb, G, tile);
                const int si = tc.g >= p.G0 ? 1 : 0;
                const SetParams& sp = p.set[si];
                const CUtensorMap* wmap = &(si ? mb : ma).w0;
                const int wg = si ? 0 : tc.g;  // weight block index of the group inside its set
                const bool gat = gather && si == 0;
                int tstart, ntok;
                token_tile(tb->rows[tc.g], tb->ttiles[tc.g], tc.tt, tstart, ntok);
                const int half = ((ntok + 15) & ~15) >> 1;
                const int xrows = gat ? half : (half + 15) & ~15;  // token rows a CTA loads per K step
                // both CTAs' bytes (E4M3: with the stage's scale slot)
                const uint32_t tx = 2u * ((uint32_t)A_BYTES + (uint32_t)xrows * 128u + (F8 ? (uint32_t)SF_STAGE_BYTES : 0u));
                const int k_blocks = sp.k_blocks;
                // weight box coordinates: up, this CTA's 64 W1 rows of the tile; down, its 128
                // W2 rows, moving to the next W2 block (d rows further) every kseg columns
                const int kseg = UP ? 0x7fffffff : sp.kseg;
                const int next_block = UP ? 0 : sp.w_rows;
                int col = 0;
                int row = UP ? wg * sp.w_rows + tc.ft * 128 + (int)rank * 64
                             : wg * sp.nseg * sp.w_rows + tc.ft * 256 + (int)rank * 128;
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, &ctl->abort, p.status)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&ctl->full[stage], tx);
                    tma_load_2d_pair(ring + stage * STAGE_BYTES, wmap, leader_full + 8u * (uint32_t)stage, col, row,
                                     W_HINT);
                    issued_any = true;
                    col += BKE;
                    if (col == kseg) {
                        col = 0;
                        row += next_block;
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
            }
            if (rank == 0) {  // this cluster takes no more tiles; the last one resets the counter
                __threadfence();
                if (atomicAdd(&sched[1], 1u) == (unsigned int)npairs - 1u) {
                    __threadfence();
                    atomicExch(&sched[0], 0u);
                    atomicExch(&sched[1], 0u);
                }
            }
            if (!ok && issued_any) settle_inflight_loads();
        }
        __syncwarp();
    } else if (warp == kTokWarp) {
        // ------------------------------------------------ token-operand producer (both CTAs)
        // One lane loads this CTA's half of the tile's token rows per K step;
        // with a gather index the whole warp runs the loop and every lane
        // fetches four token rows (tile::gather4), so the operand is read
        // straight from x in expert order.
        if (lane == 0) {
            if (p.G0 > 0) tma_prefetch_desc(gather ? &tmXg : &ma.x[NXBOX - 1]);
            if (p.has_shared) tma_prefetch_desc(&mb.x[NXBOX - 1]);
        }
        const CUtensorMap* xmap = nullptr;
        bool gat = false;
        int half = 0, tok0 = 0;
        int src[4] = {0, 0, 0, 0};
        const auto begin = [&](const TileCoord& tc) {
            const int si = tc.g >= p.G0 ? 1 : 0;
            gat = gather && si == 0;
            int tstart, ntok;
            token_tile(tb->rows[tc.g], tb->ttiles[tc.g], tc.tt, tstart, ntok);
            half = ((ntok + 15) & ~15) >> 1;
            const int row0 = tb->rowstart[tc.g] + tstart;  // first row of the tile
            tok0 = row0 + (int)rank * half;                // first row of this CTA's half
            xmap = &(si ? mb : ma).x[((half + 15) & ~15) / 16 - 1];
            if (gat) {  // this lane's four rows; rows past the tile's tokens repeat its first row
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int jr = (int)rank * half + 4 * lane + i;
                    src[i] = p.gather[row0 + (jr < ntok ? jr : 0)] / p.gather_div;
                }
            }
            return p.set[si].k_blocks;
        };
        const auto load = [&](int kb, uint8_t* stage, uint32_t fb) {
            uint8_t* sb = stage + A_BYTES;
            if (!gat && lane == 0) tma_load_2d_pair(sb, xmap, fb, kb * BKE, tok0, X_HINT);
            if (gat && 4 * lane < half)
                tma_gather4_pair(sb + 4 * lane * 128, &tmXg, fb, kb * BKE, src[0], src[1], src[2], src[3], X_HINT);
        };
        if (gather) {
            follow_tiles<STAGES, true>(ctl, tb, G, leader_tq_empty, p.status, ring, lane, begin, load);
        } else {
            if (lane == 0) follow_tiles<STAGES, false>(ctl, tb, G, leader_tq_empty, p.status, ring, lane, begin, load);
            __syncwarp();
        }
    } else if (UP && warp == kW3Warp) {
        // ------------------------------------------------ W3-half producer (up, both CTAs)
        if (lane == 0) {
            if (p.G0 > 0) tma_prefetch_desc(&ma.w1);
            if (p.has_shared) tma_prefetch_desc(&mb.w1);
        }
        const CUtensorMap* wmap = nullptr;
        int wrow = 0;
        if (lane == 0)
            follow_tiles<STAGES, false>(
                ctl, tb, G, leader_tq_empty, p.status, ring, lane,
                [&](const TileCoord& tc) {
                    const int si = tc.g >= p.G0 ? 1 : 0;
                    wmap = &(si ? mb : ma).w1;
                    wrow = (si ? 0 : tc.g) * p.set[si].w_rows + tc.ft * 128 + (int)rank * 64;
                    return p.set[si].k_blocks;
                },
                [&](int kb, uint8_t* stage, uint32_t fb) {
                    tma_load_2d_pair(stage + A_BYTES / 2, wmap, fb, kb * BKE, wrow, W_HINT);
                });

        __syncwarp();
    } else if (F8 && warp == kSfWarp) {
        // ------------------------------------------------ tile-scale producer (E4M3, both CTAs, lane 0)
        // Per stage, into the stage's scale slot: this CTA's weight-row atom
        // (512 bytes) and the tile's token image (1024 bytes), onto the
        // leader's full barrier of the stage like the operand boxes.
        if (lane == 0) {
            if (p.G0 > 0) {
                tma_prefetch_desc(&ma.sfw);
                tma_prefetch_desc(&ma.sfx);
            }
            if (p.has_shared) {
                tma_prefetch_desc(&mb.sfw);
                tma_prefetch_desc(&mb.sfx);
            }
            const CUtensorMap* wmap = nullptr;
            const CUtensorMap* xmap = nullptr;
            int wy = 0, xy = 0;
            follow_tiles<STAGES, false>(
                ctl, tb, G, leader_tq_empty, p.status, ring, lane,
                [&](const TileCoord& tc) {
                    const int si = tc.g >= p.G0 ? 1 : 0;
                    const SetParams& sp = p.set[si];
                    wmap = &(si ? mb : ma).sfw;
                    xmap = &(si ? mb : ma).sfx;
                    const int wg = si ? 0 : tc.g;
                    const long long f0 = UP ? (long long)wg * sp.w_rows + tc.ft * 128 + (int)rank * 64
                                            : (long long)wg * sp.w_rows + tc.ft * 256 + (int)rank * 128;
                    wy = (int)((UP ? f0 >> 6 : f0 >> 7) * sp.k_blocks);
                    xy = ((si ? 0 : tb->tbase[tc.g]) + tc.tt) * sp.k_blocks;
                    return sp.k_blocks;
                },
                [&](int kb, uint8_t* stage, uint32_t fb) {
                    uint8_t* slot = sfr + (size_t)((stage - ring) / STAGE_BYTES) * SF_STAGE_BYTES;
                    tma_load_2d_pair(slot, wmap, fb, 0, wy + kb, W_HINT);
                    tma_load_2d_pair(slot + SFA_BYTES, xmap, fb, 0, xy + kb, X_HINT);
                });
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (leader CTA only)
        if (rank == 0 && elect_one()) {
            int stage = 0, acc = 1, j = 0;  // acc: the previous tile's accumulator
            uint32_t phase = 0, tq_ph = 0;
            uint32_t acc_ph = 0u;  // bit a: phase of accumulator a
            bool ok = true;
            for (;;) {
                int tile;
                if (!tq_take(ctl, j, tq_ph, leader_tq_empty, &tile, p.status)) {
                    ok = false;
                    break;
                }
                if (++j == TQ) {
                    j = 0;
                    tq_ph ^= 1u;
                }
                if (tile < 0) break;
                const TileCoord tc = tile_coords(tb, G, tile);
                const int kblocks = p.set[tc.g >= p.G0 ? 1 : 0].k_blocks;
                int tstart, ntok;
                token_tile(tb->rows[tc.g], tb->ttiles[tc.g], tc.tt, tstart, ntok);
                const int n_mma = (ntok + 15) & ~15;
                const uint32_t idesc = idesc_bf16_f32(256, n_mma);
                acc = next_acc<F8>(acc, n_mma);
                if (!mbar_wait_cluster(&ctl->tempty[acc], ((acc_ph >> acc) & 1u) ^ 1u, &ctl->abort, p.status)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)acc * ACC_COLS;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&ctl->full[stage], phase, &ctl->abort, p.status)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t* sa = ring + stage * STAGE_BYTES;
                    const uint64_t ad = smem_desc_sw128(smem_u32(sa));
                    const uint64_t bd = smem_desc_sw128(smem_u32(sa + A_BYTES));
                    if (F8) {
                        // the stage's tile scales into tensor memory (one slot, reused every stage: the
                        // copies and MMAs of this thread execute in issue order), then 4 MMAs of K = 32,
                        // each reading byte kk of its rows' scale words
                        const uint32_t sfa = smem_u32(sfr + stage * SF_STAGE_BYTES);
                        tc_cp_32x128b_x4_pair(tmem_base + SFA_COL, smem_desc_plain(sfa));
                        tc_cp_32x128b_x4_pair(tmem_base + SFB_COL, smem_desc_plain(sfa + SFA_BYTES));
                        if (n_mma > 128)
                            tc_cp_32x128b_x4_pair(tmem_base + SFB_COL + 4u, smem_desc_plain(sfa + SFA_BYTES + 512));
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            tc_mma_mx_pair(d_tmem, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk),
                                           idesc_mx_e4m3(256, n_mma, (uint32_t)kk, (uint32_t)kk),
                                           (tmem_base + SFA_COL) | ((uint32_t)kk << 30),
                                           (tmem_base + SFB_COL) | ((uint32_t)kk << 30), (kb > 0 || kk > 0) ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)  // 4 MMAs of K = 16 (32 bytes)
                            tc_mma_bf16_pair(d_tmem, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc,
                                             (kb > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit_pair(&ctl->empty[stage], 0x3);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit_pair(&ctl->tfull[acc], 0x3);
                acc_ph ^= 1u << acc;
            }
            if (!ok) {  // wait for the pair MMAs already issued (same cta_group as the MMAs)
                tc_commit_pair(&ctl->drain, 0x1);
                mbar_wait_drain(&ctl->drain, 0);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue (both CTAs)
        // Two groups of four warps (one per TMEM lane quarter each) take the
        // tile's 16-token chunks in turn: group eg handles chunks eg, eg+2, ...
        const int q = warp & 3;           // TMEM lane quarter this warp may read
        const int eg = (warp - 2) >> 2;   // epilogue group
        const int e = tid - 64 - 128 * eg;  // 0..127 within the group
        const int my_tok = e >> 3;        // token (0..15) of a 16-token chunk this thread stores
        const int part = e & 7;
        const uint32_t leader_tempty = mapa_shared(smem_u32(&ctl->tempty[0]), 0);
        int acc = 1, xb = 0, j = 0;  // acc: the previous tile's accumulator (next_acc, as the MMA issuer)
        uint32_t acc_ph = 0u, tq_ph = 0;  // acc_ph bit a: phase of accumulator a
        for (;;) {
            int tile = -1, got = 1;
            if (lane == 0) got = tq_take(ctl, j, tq_ph, leader_tq_empty, &tile, p.status) ? 1 : 0;
            got = __shfl_sync(0xffffffffu, got, 0);
            tile = __shfl_sync(0xffffffffu, tile, 0);
            if (!got || tile < 0) break;
            if (++j == TQ) {
                j = 0;
                tq_ph ^= 1u;
            }
            const TileCoord tc = tile_coords(tb, G, tile);
            const SetParams& sp = p.set[tc.g >= p.G0 ? 1 : 0];
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(sp.out);
            int tstart, ntok;
            token_tile(tb->rows[tc.g], tb->ttiles[tc.g], tc.tt, tstart, ntok);
            const int tok0 = tb->rowstart[tc.g] + tstart;
            const int qimg = (tc.g >= p.G0 ? 0 : tb->tbase[tc.g]) + tc.tt;  // E4M3 h: the tile's scale image
            // first output feature of this CTA
            const int fcta = UP ? tc.ft * 128 + (int)rank * 64 : tc.ft * 256 + (int)rank * 128;
            acc = next_acc<F8>(acc, (ntok + 15) & ~15);
            if (!mbar_wait(&ctl->tfull[acc], (acc_ph >> acc) & 1u, &ctl->abort, p.status)) break;
            tc_fence_after();
            const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)acc * ACC_COLS;
            // TMEM reads run one chunk ahead of the exchange below
            constexpr int CSTEP = 16 * (NEPI / 4);
            uint32_t r[16];
            if (16 * eg < ntok) tmem_ld16(taddr + (uint32_t)(16 * eg), r);
#pragma unroll 1
            for (int c = 16 * eg; c < ntok; c += CSTEP) {
                tmem_ld_wait();
                float v16[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v16[i] = __uint_as_float(r[i]);
                if (c + CSTEP < ntok) tmem_ld16(taddr + (uint32_t)(c + CSTEP), r);
                float* xs = xbuf + (NXB * eg + xb) * (XBUF_BYTES / 4);
#pragma unroll
                for (int i = 0; i < 16; ++i) xs[i * XS + q * 32 + lane] = v16[i];
                named_bar_sync(1 + eg, 128);
                const bool tok_ok = c + my_tok < ntok;
                const float* row = xs + my_tok * XS;
                if (UP) {  // lanes 0-63: gate, 64-127: up of the same 64 features
                    const int fj = part * 8;
                    float4 g0 = *reinterpret_cast<const float4*>(row + fj);
                    float4 g1 = *reinterpret_cast<const float4*>(row + fj + 4);
                    float4 u0 = *reinterpret_cast<const float4*>(row + 64 + fj);
                    float4 u1 = *reinterpret_cast<const float4*>(row + 64 + fj + 4);
                    if (NXB == 1) named_bar_sync(1 + eg, 128);  // the single buffer is free for the next chunk
                    if (F8 && sp.q_out) {
                        // h rounded to bf16 (as the plain output), then its 1x32 tiles to E4M3: the four lanes
                        // of a token's 32 features share the tile's largest magnitude
                        float hv[8] = {silu_fast(g0.x) * u0.x, silu_fast(g0.y) * u0.y, silu_fast(g0.z) * u0.z,
                                       silu_fast(g0.w) * u0.w, silu_fast(g1.x) * u1.x, silu_fast(g1.y) * u1.y,
                                       silu_fast(g1.z) * u1.z, silu_fast(g1.w) * u1.w};
                        float amax = 0.0f;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            hv[i] = __bfloat162float(__float2bfloat16_rn(hv[i]));
                            amax = fmaxf(amax, fabsf(hv[i]));
                        }
                        if (!tok_ok) amax = 0.0f;
                        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
                        const int ex = mx_tile_exponent(amax);
                        const float mul = mx_inv_scale(ex);
                        const uint32_t sbyte = (uint32_t)(ex + 127);
                        const uint32_t sother = __shfl_xor_sync(0xffffffffu, sbyte, 4);  // the CTA's other tile
                        if (tok_ok) {
                            const size_t orow = (size_t)(tok0 + c + my_tok);
                            const uint32_t c0 = e4m3x2(__fmul_rn(hv[0], mul), __fmul_rn(hv[1], mul)) |
                                                (e4m3x2(__fmul_rn(hv[2], mul), __fmul_rn(hv[3], mul)) << 16);
                            const uint32_t c1 = e4m3x2(__fmul_rn(hv[4], mul), __fmul_rn(hv[5], mul)) |
                                                (e4m3x2(__fmul_rn(hv[6], mul), __fmul_rn(hv[7], mul)) << 16);
                            *reinterpret_cast<uint2*>(sp.q_out + orow * sp.ldo + fcta + fj) = make_uint2(c0, c1);
                        }
                        if (part == 0) {  // tiles fcta / 32 and the next: bytes j, j + 1 of the token's stage word
                            // (tokens of the last chunk past the tile get scale 1: the down MMA's padding columns)
                            uint8_t* wd = reinterpret_cast<uint8_t*>(
                                sp.q_img + ((size_t)qimg * (size_t)(sp.ldo >> 7) + (size_t)(fcta >> 7)) * 256u +
                                tile_image_word(c + my_tok));
                            *reinterpret_cast<uint16_t*>(wd + ((fcta & 127) >> 5)) = (uint16_t)(sbyte | (sother << 8));
                        }
                    } else if (tok_ok) {
                        uint4 v;
                        v.x = pack_bf16x2(silu_fast(g0.x) * u0.x, silu_fast(g0.y) * u0.y);
                        v.y = pack_bf16x2(silu_fast(g0.z) * u0.z, silu_fast(g0.w) * u0.w);
                        v.z = pack_bf16x2(silu_fast(g1.x) * u1.x, silu_fast(g1.y) * u1.y);
                        v.w = pack_bf16x2(silu_fast(g1.z) * u1.z, silu_fast(g1.w) * u1.w);
                        *reinterpret_cast<uint4*>(out + (size_t)(tok0 + c + my_tok) * sp.ldo + fcta + fj) = v;
                        if (!F8 && sp.a_out) {
                            const size_t o = (size_t)(tok0 + c + my_tok) * sp.ldo + fcta + fj;
                            float4* ad = reinterpret_cast<float4*>(sp.a_out + o);
                            float4* gd = reinterpret_cast<float4*>(sp.g_out + o);
                            ad[0] = g0;
                            ad[1] = g1;
                            gd[0] = u0;
                            gd[1] = u1;
                        }
                    }
                } else {
                    const int fj = part * 16;
                    const bool st_ok = tok_ok && fcta + fj < sp.f_limit;
                    float f[16];
                    if (st_ok) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float4 t = *reinterpret_cast<const float4*>(row + fj + 4 * i);
                            f[4 * i] = t.x;
                            f[4 * i + 1] = t.y;
                            f[4 * i + 2] = t.z;
                            f[4 * i + 3] = t.w;
                        }
                    }
                    if (NXB == 1) named_bar_sync(1 + eg, 128);  // the single buffer is free for the next chunk
                    if (st_ok) {
                        const int orow = tok0 + c + my_tok;
                        if (sp.acc) {  // fused weighted combine
                            int t = orow;
                            float wt = 1.0f;
                            if (sp.row_tok) {
                                const int a = sp.row_tok[orow];
                                t = a / sp.row_k;
                                wt = sp.row_w[a];
                            }
                            float* dst = sp.acc + (size_t)t * sp.ldo + fcta + fj;
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                red_add_v4(dst + 4 * i, f[4 * i] * wt, f[4 * i + 1] * wt, f[4 * i + 2] * wt,
                                           f[4 * i + 3] * wt);
                        } else {
                            uint4* dst = reinterpret_cast<uint4*>(out + (size_t)orow * sp.ldo + fcta + fj);
                            dst[0] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                                pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7]));
                            dst[1] = make_uint4(pack_bf16x2(f[8], f[9]), pack_bf16x2(f[10], f[11]),
                                                pack_bf16x2(f[12], f[13]), pack_bf16x2(f[14], f[15]));
                        }
                    }
                }
                if (NXB == 2) xb ^= 1;  // the next chunk writes the other buffer; its barrier orders the reuse
            }
            tc_fence_before();
            __syncwarp();
            // the accumulator's tcgen05.ld have completed (wait::ld above): a relaxed arrive frees it (a
            // cluster-scope release here cost about 1 us per tile and warp)
            if (lane == 0) mbar_arrive_relaxed_cluster(leader_tempty + 8u * (uint32_t)acc);
            acc_ph ^= 1u << acc;
        }
    }

    tc_fence_before();
    cluster_sync_all();  // no CTA leaves while its peer's MMAs may still read its shared memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

std::atomic<unsigned int> g_sched_seq{0};

template <bool UP, bool F8>
cudaError_t launch(const SetMaps& a, const SetMaps& b, const CUtensorMap& xg, Params p, int num_sms, cudaStream_t st) {
    auto kern = tc_grouped_gemm_kernel<UP, F8>;
    p.sched_slot = (int)(g_sched_seq.fetch_add(1u, std::memory_order_relaxed) % (unsigned int)kSchedSlots);
    constexpr size_t SMEM = smem_bytes<UP, F8>();
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM);
    constexpr int NTHREADS = n_threads<UP, F8>();
    if (err != cudaSuccess) return err;
    const int grid = (num_sms / 2) * 2;  // whole CTA pairs, one CTA per SM
    kern<<<grid, NTHREADS, SMEM, st>>>(a, b, xg, p);
    note_launches(1);
    return cudaGetLastError();
}

bool token_maps(SetMaps& m, const void* base, int cols, long long rows, unsigned eb) {
    for (int b = 0; b < NXBOX; ++b)
        if (!make_tmap_2d(&m.x[b], base, cols, rows, cols, 128 / eb, 16 * (b + 1), eb)) return false;
    return true;
}

bool up_set(const TcUpArgs& a, SetMaps& m, SetParams& sp) {
    const unsigned eb = a.f8 ? 1 : 2;
    const int bke = 128 / (int)eb;
    if (a.d % bke != 0 || a.I % 128 != 0) return false;
    if (a.f8 && (!a.w13s || !a.xs || a.xs_tiles <= 0 || a.d % 128 != 0 || a.W_rows % 64 != 0)) return false;
    if (!make_tmap_2d(&m.w0, a.W1, a.d, a.W_rows, a.d, bke, 64, eb) ||
        !make_tmap_2d(&m.w1, a.W3, a.d, a.W_rows, a.d, bke, 64, eb) || !token_maps(m, a.A, a.d, a.A_rows, eb))
        return false;
    sp.f_tiles = a.I / 128;
    sp.k_blocks = a.d / bke;
    if (a.f8 && (!make_tmap_rows_u32(&m.sfw, a.w13s, SFA_BYTES / 4, (unsigned long long)(a.W_rows / 64) * sp.k_blocks) ||
                 !make_tmap_rows_u32(&m.sfx, a.xs, SFB_BYTES / 4, (unsigned long long)a.xs_tiles * sp.k_blocks)))
        return false;
    sp.w_rows = a.I;
    sp.kseg = a.d;
    sp.nseg = 1;
    sp.out = a.H;
    sp.ldo = a.I;
    sp.f_limit = a.I;
    sp.a_rows = a.gather ? a.gather_rows : a.A_rows;
    sp.q_out = a.f8 ? a.hq : nullptr;
    sp.q_img = a.f8 ? a.hq_img : nullptr;
    if (sp.q_out && !sp.q_img) return false;
    sp.a_out = a.f8 ? nullptr : a.pre_a;
    sp.g_out = a.f8 ? nullptr : a.pre_g;
    if (!sp.a_out != !sp.g_out) return false;
    return true;
}

bool down_set(const TcDownArgs& a, SetMaps& m, SetParams& sp) {
    const unsigned eb = a.f8 ? 1 : 2;
    const int bke = 128 / (int)eb;
    if (a.K % bke != 0 || a.kseg % bke != 0 || a.d % 16 != 0) return false;
    if (a.f8 && (!a.w2s || !a.hs || a.hs_tiles <= 0 || a.K % 128 != 0 || a.kseg % 128 != 0 || a.d % 128 != 0))
        return false;
    // W2 blocks [G * nseg][d][kseg] viewed as one matrix of G * nseg * d rows: a 2D map fed
    // the down projection ~10% faster than the same boxes through a 3D map.  Rows past d of
    // a feature tile read the next block's rows (or zero past the end); their outputs are
    // never stored.
    if (!make_tmap_2d(&m.w0, a.W2, a.kseg, (unsigned long long)a.G * a.nseg * a.d, a.kseg, bke, 128, eb) ||
        !token_maps(m, a.H, a.K, a.H_rows, eb))
        return false;
    m.w1 = m.w0;
    sp.f_tiles = (a.d + 255) / 256;
    sp.k_blocks = a.K / bke;
    if (a.f8 && (!make_tmap_rows_u32(&m.sfw, a.w2s, SFA_BYTES / 4, (unsigned long long)a.G * a.d / 128 * sp.k_blocks) ||
                 !make_tmap_rows_u32(&m.sfx, a.hs, SFB_BYTES / 4, (unsigned long long)a.hs_tiles * sp.k_blocks)))
        return false;
    sp.acc = a.acc;
    sp.row_tok = a.row_tok;
    sp.row_w = a.row_w;
    sp.row_k = a.row_k > 0 ? a.row_k : 1;
    sp.w_rows = a.d;
    sp.kseg = a.kseg;
    sp.nseg = a.nseg;
    sp.out = a.Y;
    sp.ldo = a.d;
    sp.f_limit = a.d;
    sp.a_rows = a.H_rows;
    return true;
}

}  // namespace

// routed: groups from offsets (may be null to launch the shared set alone);
// shared: one group of M rows (may be null).  Both sets share one launch.
cudaError_t launch_tc_up(const TcUpArgs* routed, const TcUpArgs* shared, int* status, int num_sms, cudaStream_t st) {
    if (!routed && !shared) return cudaSuccess;
    SetMaps ma{}, mb{};
    Params p{};
    CUtensorMap xg{};
    if (routed) {
        if (routed->G <= 0 || routed->G > kMaxGroups || !routed->offsets || !up_set(*routed, ma, p.set[0]))
            return cudaErrorInvalidValue;
        const unsigned eb = routed->f8 ? 1 : 2;
        if (!make_tmap_2d(&xg, routed->A, routed->d, routed->A_rows, routed->d, 128 / eb, 1, eb))  // tile::gather4 box
            return cudaErrorInvalidValue;
        p.offsets = routed->offsets;
        p.G0 = routed->G;
        p.gather = routed->gather;
        p.gather_div = routed->gather_div > 0 ? routed->gather_div : 1;
    }
    if (shared) {
        if (shared->M <= 0 || !up_set(*shared, mb, p.set[1])) return cudaErrorInvalidValue;
        p.has_shared = 1;
        p.M = shared->M;
        if (!routed) xg = mb.x[NXBOX - 1];
    }
    if (routed && shared && routed->f8 != shared->f8) return cudaErrorInvalidValue;
    if (!routed) ma = mb;
    if (!shared) mb = ma;
    p.status = status;
    const bool f8 = routed ? routed->f8 : shared->f8;
    return f8 ? launch<true, true>(ma, mb, xg, p, num_sms, st) : launch<true, false>(ma, mb, xg, p, num_sms, st);
}

cudaError_t launch_tc_down(const TcDownArgs* routed, const TcDownArgs* shared, int* status, int num_sms,
                           cudaStream_t st) {
    if (!routed && !shared) return cudaSuccess;
    SetMaps ma{}, mb{};
    Params p{};
    if (routed) {
        if (routed->G <= 0 || routed->G > kMaxGroups || !routed->offsets || !down_set(*routed, ma, p.set[0]))
            return cudaErrorInvalidValue;
        p.offsets = routed->offsets;
        p.G0 = routed->G;
    }
    if (shared) {
        if (shared->M <= 0 || !down_set(*shared, mb, p.set[1])) return cudaErrorInvalidValue;
        p.has_shared = 1;
        p.M = shared->M;
    }
    if (routed && shared && routed->f8 != shared->f8) return cudaErrorInvalidValue;
    if (!routed) ma = mb;
    if (!shared) mb = ma;
    p.gather = nullptr;
    p.gather_div = 1;
    p.status = status;
    const bool f8 = routed ? routed->f8 : shared->f8;
    return f8 ? launch<false, true>(ma, mb, ma.x[NXBOX - 1], p, num_sms, st)
              : launch<false, false>(ma, mb, ma.x[NXBOX - 1], p, num_sms, st);
}

}  // namespace moe
