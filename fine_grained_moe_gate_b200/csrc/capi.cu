// C ABI entry points (moe_gate.h): host-side validation, workspace carving
// and kernel launches.  Nothing here allocates device memory.
#include "../../include/moe_gate.h"
#include "kernels.h"

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

namespace {

// Per-device status word written by kernels on an anomaly.
__device__ int g_status_word;

constexpr int kMaxDevices = 64;
std::atomic<unsigned long long> g_launches{0};
int* g_status_ptr[kMaxDevices];
int g_num_sms[kMaxDevices];
std::mutex g_setup_mu;

// Per-device set-up, once: the status word's device address and SM count.
moe_status device_setup(int* dev_out, int** status_out, int* sms_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_setup_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return MOE_ERR_CUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return MOE_ERR_CUDA;
        g_num_sms[dev] = sms;
        g_status_ptr[dev] = static_cast<int*>(p);
    }
    *dev_out = dev;
    *status_out = g_status_ptr[dev];
    *sms_out = g_num_sms[dev];
    return MOE_OK;
}

inline size_t align256(size_t n) { return (n + 255) & ~size_t(255); }
// bytes per element of the token rows moe_permute moves (E4M3 rows for MOE_FP8_E4M3)
inline size_t esize(const moe_shape& sh) { return sh.dtype == MOE_F32 ? 4 : sh.dtype == MOE_BF16 ? 2 : 1; }
inline bool is_fp8(const moe_shape& sh) { return sh.dtype == MOE_FP8_E4M3; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status validate_shape(const moe_shape& sh) {
    if (sh.dtype != MOE_F32 && sh.dtype != MOE_BF16 && sh.dtype != MOE_FP8_E4M3) return MOE_ERR_INVALID_ARG;
    if (sh.T < 0 || sh.d <= 0 || sh.E <= 0 || sh.k <= 0 || sh.I <= 0 || sh.S < 0) return MOE_ERR_INVALID_ARG;
    if (sh.S > 0 && sh.Is <= 0) return MOE_ERR_INVALID_ARG;
    if (sh.k > sh.E) return MOE_ERR_INVALID_ARG;
    if (sh.k > 16 || sh.E > moe::kMaxExperts) return MOE_ERR_UNSUPPORTED;
    if (sh.d % 8 != 0) return MOE_ERR_UNSUPPORTED;
    // 32-bit row coordinates (tensor maps, row indices)
    if ((long long)sh.T * sh.k >= (1ll << 31) || (long long)sh.E * sh.I >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
    if (sh.dtype != MOE_F32) {
        if (sh.d % (is_fp8(sh) ? 128 : 64) != 0 || sh.I % 128 != 0) return MOE_ERR_UNSUPPORTED;
        if (sh.S > 0 && sh.Is % 128 != 0) return MOE_ERR_UNSUPPORTED;
    }
    return MOE_OK;
}

// Calls that take bf16 (or fp32) expert weights.
moe_status validate_dense_weights(const moe_shape& sh) {
    const moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    return is_fp8(sh) ? MOE_ERR_UNSUPPORTED : MOE_OK;
}

#define MOE_REQUIRE(cond, code) \
    do {                        \
        if (!(cond)) return (code); \
    } while (0)

#define MOE_CUDA(call)                                   \
    do {                                                 \
        if ((call) != cudaSuccess) return MOE_ERR_CUDA;  \
    } while (0)

size_t permute_ws(const moe_shape& sh) { return align256(moe::permute_scratch_bytes(sh.T, sh.E)); }
size_t swiglu_ws(const moe_shape& sh) {
    const size_t eb = esize(sh);
    return align256((size_t)sh.T * sh.k * sh.I * eb) + align256((size_t)sh.T * sh.S * (size_t)sh.Is * eb);
}

// ---- internal stages (arguments already validated) -----------------------

moe_status do_route(const void* x, const void* w_gate, const float* bias, const moe_shape& sh, int32_t* idx,
                    float* w, int32_t* counts, float* aff, int* status, int sms, cudaStream_t st) {
    MOE_CUDA(cudaMemsetAsync(counts, 0, sizeof(int32_t) * sh.E, st));
    if (sh.T == 0) return MOE_OK;
    cudaError_t err;
    if (sh.dtype != MOE_F32)  // x and W_gate are bf16 for MOE_FP8_E4M3 too
        err = moe::launch_router_tc(x, w_gate, bias, sh.T, sh.d, sh.E, sh.k, idx, w, counts, aff, status, sms, st);
    else
        err = moe::launch_router_simt(x, w_gate, bias, sh.T, sh.d, sh.E, sh.k, false, idx, w, counts, aff, status,
                                      st);
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status do_permute(const void* x, const int32_t* idx, const int32_t* counts, const moe_shape& sh, void* x_perm,
                      int32_t* offsets, int32_t* perm, int32_t* inv, void* ws, int* status, cudaStream_t st) {
    cudaError_t err = moe::launch_permute(x, idx, counts, sh.T, sh.d, sh.E, sh.k, esize(sh), x_perm, offsets, perm,
                                          inv, static_cast<int32_t*>(ws), status, st);
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Tensor-core argument blocks of one expert set: the routed set has a group
// per expert (rows from offsets), the shared set is one group of T rows whose
// S weight blocks are stacked into one [S*Is][d] matrix.
moe::TcUpArgs tc_up_args(const void* a, const int32_t* gather, const int32_t* offsets, const void* w1,
                         const void* w3, const moe_shape& sh, bool shared, void* h) {
    const long long rows = shared ? sh.T : (long long)sh.T * sh.k;
    const int Ig = shared ? sh.S * sh.Is : sh.I;
    if (shared) gather = nullptr;
    return moe::TcUpArgs{a, gather ? sh.T : rows, gather, sh.k, rows, w1, w3,
                         shared ? (long long)Ig : (long long)sh.E * sh.I, h, sh.d, Ig, shared ? nullptr : offsets,
                         shared ? 1 : sh.E, shared ? sh.T : 0};
}

moe::TcDownArgs tc_down_args(const void* h, const int32_t* offsets, const void* w2, const moe_shape& sh, bool shared,
                             void* y) {
    const long long rows = shared ? sh.T : (long long)sh.T * sh.k;
    return moe::TcDownArgs{h, rows, w2, shared ? sh.S : 1, shared ? sh.Is : sh.I, y, sh.d,
                           shared ? sh.S * sh.Is : sh.I, shared ? nullptr : offsets, shared ? 1 : sh.E,
                           shared ? sh.T : 0};
}

// gather (routed set only, may be null): group row r reads row gather[r] / k
// of `a` (= x, unpermuted); without it `a` is x_perm itself.
moe_status do_expert_up(const void* a, const int32_t* gather, const int32_t* offsets, const void* w1, const void* w3,
                        const moe_shape& sh, bool shared, void* h, int* status, int sms, cudaStream_t st) {
    if (sh.T == 0) return MOE_OK;
    const long long rows = shared ? sh.T : (long long)sh.T * sh.k;  // rows the groups index (= rows of h)
    const int Ig = shared ? sh.S * sh.Is : sh.I;  // S stacked [Is][d] blocks = one [S*Is][d] matrix
    if (shared) gather = nullptr;
    cudaError_t err;
    if (sh.dtype == MOE_BF16) {
        const moe::TcUpArgs up = tc_up_args(a, gather, offsets, w1, w3, sh, shared, h);
        err = moe::launch_tc_up(shared ? nullptr : &up, shared ? &up : nullptr, status, sms, st);
    } else {
        moe::GemmArgs up{a, sh.d, w1, w3, shared ? 0 : (long long)sh.I * sh.d, sh.d, sh.d, 0, h, Ig, Ig, sh.d,
                         shared ? nullptr : offsets, shared ? 1 : sh.E, (int)rows, gather, sh.k};
        err = moe::launch_simt_gemm(up, false, true, sms, st);
    }
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status do_expert_down(const void* h, const int32_t* offsets, const void* w2, const moe_shape& sh, bool shared,
                          void* y, int* status, int sms, cudaStream_t st) {
    if (sh.T == 0) return MOE_OK;
    const long long rows = shared ? sh.T : (long long)sh.T * sh.k;
    const int kseg = shared ? sh.Is : sh.I;
    const int K = shared ? sh.S * sh.Is : sh.I;
    cudaError_t err;
    if (sh.dtype == MOE_BF16) {
        const moe::TcDownArgs dn = tc_down_args(h, offsets, w2, sh, shared, y);
        err = moe::launch_tc_down(shared ? nullptr : &dn, shared ? &dn : nullptr, status, sms, st);
    } else {
        // element (n, kk) of W2 block g: (kk / kseg) * d * kseg + n * kseg + kk % kseg
        moe::GemmArgs dn{h, K, w2, nullptr, shared ? 0 : (long long)sh.d * sh.I, kseg, kseg,
                         (long long)sh.d * kseg, y, sh.d, sh.d, K, shared ? nullptr : offsets, shared ? 1 : sh.E,
                         (int)rows, nullptr, 1};
        err = moe::launch_simt_gemm(dn, false, false, sms, st);
    }
    return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Both expert sets, one launch per projection on the tensor-core path.
moe_status do_ffn_up(const void* x_perm, const int32_t* offsets, const void* w1, const void* w3, const void* x,
                     const void* ws1, const void* ws3, const moe_shape& sh, void* h, void* hs, int* status, int sms,
                     cudaStream_t st) {
    if (sh.T == 0) return MOE_OK;
    const bool shared = x && sh.S > 0;
    if (sh.dtype == MOE_BF16) {
        const moe::TcUpArgs ur = tc_up_args(x_perm, nullptr, offsets, w1, w3, sh, false, h);
        const moe::TcUpArgs us = tc_up_args(x, nullptr, nullptr, ws1, ws3, sh, true, hs);
        return moe::launch_tc_up(&ur, shared ? &us : nullptr, status, sms, st) == cudaSuccess ? MOE_OK
                                                                                                : MOE_ERR_CUDA;
    }
    moe_status v = do_expert_up(x_perm, nullptr, offsets, w1, w3, sh, false, h, status, sms, st);
    if (v == MOE_OK && shared) v = do_expert_up(x, nullptr, nullptr, ws1, ws3, sh, true, hs, status, sms, st);
    return v;
}

moe_status do_ffn_down(const void* h, const int32_t* offsets, const void* w2, const void* hs, const void* ws2,
                       const moe_shape& sh, void* y_perm, void* shared_out, int* status, int sms, cudaStream_t st) {
    if (sh.T == 0) return MOE_OK;
    const bool shared = hs && sh.S > 0;
    if (sh.dtype == MOE_BF16) {
        const moe::TcDownArgs dr = tc_down_args(h, offsets, w2, sh, false, y_perm);
        const moe::TcDownArgs ds = tc_down_args(hs, nullptr, ws2, sh, true, shared_out);
        return moe::launch_tc_down(&dr, shared ? &ds : nullptr, status, sms, st) == cudaSuccess ? MOE_OK
                                                                                                  : MOE_ERR_CUDA;
    }
    moe_status v = do_expert_down(h, offsets, w2, sh, false, y_perm, status, sms, st);
    if (v == MOE_OK && shared) v = do_expert_down(hs, nullptr, ws2, sh, true, shared_out, status, sms, st);
    return v;
}

// Down projection with the weighted combine fused into its epilogue (tensor
// cores): routed rows scaled by topk_w[perm_tok[r]] and added into acc at
// token perm_tok[r] / k; shared rows (hs) added with weight 1.
moe_status do_ffn_down_combine(const void* h, const int32_t* offsets, const void* w2, const void* hs,
                               const void* ws2, const int32_t* perm_tok, const float* topk_w, const moe_shape& sh,
                               float* acc, int* status, int sms, cudaStream_t st) {
    if (sh.T == 0) return MOE_OK;
    const bool shared = hs && sh.S > 0;
    moe::TcDownArgs dr = tc_down_args(h, offsets, w2, sh, false, nullptr);
    dr.acc = acc;
    dr.row_tok = perm_tok;
    dr.row_w = topk_w;
    dr.row_k = sh.k;
    moe::TcDownArgs ds = tc_down_args(hs, nullptr, ws2, sh, true, nullptr);
    ds.acc = acc;
    return moe::launch_tc_down(&dr, shared ? &ds : nullptr, status, sms, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status do_swiglu(const void* x_perm, const int32_t* offsets, const void* w1, const void* w3, const void* w2,
                     const void* x, const void* ws1, const void* ws3, const void* ws2, const moe_shape& sh,
                     void* y_perm, void* shared_out, void* ws, int* status, int sms, cudaStream_t st) {
    const size_t eb = esize(sh);
    const long long rows = (long long)sh.T * sh.k;
    char* h = static_cast<char*>(ws);
    char* hs = h + align256((size_t)rows * sh.I * eb);
    const bool shared = x && sh.S > 0 && shared_out;
    moe_status v = do_ffn_up(x_perm, offsets, w1, w3, shared ? x : nullptr, ws1, ws3, sh, h, hs, status, sms, st);
    if (v != MOE_OK) return v;
    return do_ffn_down(h, offsets, w2, shared ? hs : nullptr, ws2, sh, y_perm, shared_out, status, sms, st);
}

// ---- FP8 experts -----------------------------------------------------------


moe_status do_ffn_up_fp8(const uint8_t* xq_perm, const void* x_tiles, const int32_t* offsets, const uint8_t* xq,
                         const void* xsh_tiles, const moe_fp8_experts* w, const moe_shape& sh, void* h, void* hs,
                         int* status, int sms, cudaStream_t st, uint8_t* hq = nullptr, void* h_tiles = nullptr,
                         uint8_t* hsq = nullptr, void* hs_tiles = nullptr) {
    if (sh.T == 0) return MOE_OK;
    const bool shared = xq && sh.S > 0;
    moe::TcUpArgs ur = tc_up_args(xq_perm, nullptr, offsets, w->w1, w->w3, sh, false, h);
    ur.f8 = true;
    ur.w13s = static_cast<const uint8_t*>(w->w13_scale);
    ur.xs = static_cast<const uint32_t*>(x_tiles);
    ur.xs_tiles = moe::mx_tile_images((long long)sh.T * sh.k, sh.E);
    ur.hq = hq;
    ur.hq_img = static_cast<uint32_t*>(h_tiles);
    moe::TcUpArgs us = tc_up_args(xq, nullptr, nullptr, w->ws1, w->ws3, sh, true, hs);
    us.f8 = true;
    us.w13s = static_cast<const uint8_t*>(w->ws13_scale);
    us.xs = static_cast<const uint32_t*>(xsh_tiles);
    us.xs_tiles = moe::mx_tile_images(sh.T, 1);
    us.hq = hsq;
    us.hq_img = static_cast<uint32_t*>(hs_tiles);
    return moe::launch_tc_up(&ur, shared ? &us : nullptr, status, sms, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status do_ffn_down_fp8(const uint8_t* hq, const void* h_tiles, const int32_t* offsets, const uint8_t* hsq,
                           const void* hs_tiles, const moe_fp8_experts* w, const moe_shape& sh, void* y_perm,
                           void* shared_out, int* status, int sms, cudaStream_t st) {
    if (sh.T == 0) return MOE_OK;
    const bool shared = hsq && sh.S > 0;
    moe::TcDownArgs dr = tc_down_args(hq, offsets, w->w2, sh, false, y_perm);
    dr.f8 = true;
    dr.w2s = static_cast<const uint8_t*>(w->w2_scale);
    dr.hs = static_cast<const uint32_t*>(h_tiles);
    dr.hs_tiles = moe::mx_tile_images((long long)sh.T * sh.k, sh.E);
    moe::TcDownArgs ds = tc_down_args(hsq, nullptr, w->ws2, sh, true, shared_out);
    ds.f8 = true;
    ds.w2s = static_cast<const uint8_t*>(w->ws2_scale);
    ds.hs = static_cast<const uint32_t*>(hs_tiles);
    ds.hs_tiles = moe::mx_tile_images(sh.T, 1);
    return moe::launch_tc_down(&dr, shared ? &ds : nullptr, status, sms, st) == cudaSuccess ? MOE_OK
                                                                                              : MOE_ERR_CUDA;
}

bool fp8_weights_ok(const moe_fp8_experts* w, const moe_shape& sh) {
    if (!w || !w->w1 || !w->w3 || !w->w2 || !w->w13_scale || !w->w2_scale) return false;
    if (sh.S > 0 && (!w->ws1 || !w->ws3 || !w->ws2 || !w->ws13_scale || !w->ws2_scale)) return false;
    return true;
}

bool fp8_weights_aligned(const moe_fp8_experts* w) {
    return aligned16(w->w1) && aligned16(w->w3) && aligned16(w->w2) && aligned16(w->ws1) && aligned16(w->ws3) &&
           aligned16(w->ws2) && aligned16(w->w13_scale) && aligned16(w->w2_scale) && aligned16(w->ws13_scale) &&
           aligned16(w->ws2_scale);
}

// Workspace of moe_layer_forward_fp8, carved in this order.
struct Fp8Work {
    int32_t* offsets;
    int32_t* perm;
    int32_t* inv;
    void* pws;
    uint8_t* xq;
    void* xs;
    uint8_t* xq_perm;
    void* x_tiles;    // token images of xq_perm's tiles
    void* xsh_tiles;  // token images of xq's tiles (shared experts)
    uint8_t* hq;
    void* h_tiles;
    uint8_t* hsq;
    void* hs_tiles;
    void* y_perm;
    void* shared_out;
};

// Bytes of the token images of `rows` rows in `groups` groups, K columns.
size_t tile_image_bytes(long long rows, int groups, int K) {
    return (size_t)moe::mx_tile_images(rows, groups) * (size_t)(K / 128) * 1024;
}

size_t fp8_work(const moe_shape& sh, char* base, Fp8Work* o) {
    const size_t T = (size_t)sh.T, rows = T * sh.k, SI = (size_t)sh.S * sh.Is, d = (size_t)sh.d, I = (size_t)sh.I;
    const bool S = sh.S > 0;
    // token-layout tile scales of x: one 32-bit word per row and 128 columns
    const size_t sizes[15] = {(size_t)(sh.E + 1) * 4, rows * 4, rows * 4, permute_ws(sh), T * d, T * (d / 128) * 4,
                              rows * d, tile_image_bytes((long long)rows, sh.E, sh.d),
                              S ? tile_image_bytes(sh.T, 1, sh.d) : 0, rows * I,
                              tile_image_bytes((long long)rows, sh.E, sh.I), T * SI,
                              S ? tile_image_bytes(sh.T, 1, (int)SI) : 0, rows * d * 2, T * d * 2};
    void* ptrs[15];
    size_t off = 0;
    for (int i = 0; i < 15; ++i) {
        ptrs[i] = base ? base + off : nullptr;
        off += align256(sizes[i]);
    }
    if (o) {
        o->offsets = static_cast<int32_t*>(ptrs[0]);
        o->perm = static_cast<int32_t*>(ptrs[1]);
        o->inv = static_cast<int32_t*>(ptrs[2]);
        o->pws = ptrs[3];
        o->xq = static_cast<uint8_t*>(ptrs[4]);
        o->xs = ptrs[5];
        o->xq_perm = static_cast<uint8_t*>(ptrs[6]);
        o->x_tiles = ptrs[7];
        o->xsh_tiles = ptrs[8];
        o->hq = static_cast<uint8_t*>(ptrs[9]);
        o->h_tiles = ptrs[10];
        o->hsq = static_cast<uint8_t*>(ptrs[11]);
        o->hs_tiles = ptrs[12];
        o->y_perm = ptrs[13];
        o->shared_out = ptrs[14];
    }
    return off;
}

}  // namespace

namespace moe {
void note_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }
}  // namespace moe

extern "C" {

uint64_t moe_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int moe_abi_version(void) { return 100; }

const char* moe_status_string(moe_status s) {
    switch (s) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case MOE_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_CUDA: return "CUDA runtime error";
        case MOE_ERR_DEVICE_CHECK: return "device-side consistency check failed";
        case MOE_ERR_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

size_t moe_permute_workspace_size(moe_shape sh) {
    if (validate_shape(sh) != MOE_OK) return 0;
    return permute_ws(sh);
}

size_t moe_grouped_swiglu_workspace_size(moe_shape sh) {
    if (validate_dense_weights(sh) != MOE_OK) return 0;
    return swiglu_ws(sh);
}

size_t moe_workspace_size(moe_shape sh) {
    if (validate_shape(sh) != MOE_OK) return 0;
    if (is_fp8(sh)) return fp8_work(sh, nullptr, nullptr);
    const size_t rows = (size_t)sh.T * sh.k;
    return align256((sh.E + 1) * sizeof(int32_t)) + 2 * align256(rows * sizeof(int32_t)) + permute_ws(sh) +
           align256(rows * sh.d * esize(sh)) + swiglu_ws(sh) + align256((size_t)sh.T * sh.d * esize(sh));
}

moe_status moe_route(const void* x, const void* w_gate, const float* bias, moe_shape sh, int32_t* topk_idx,
                     float* topk_w, int32_t* counts, float* affinity_out, void* stream) {
    moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(w_gate && bias && counts, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (x && topk_idx && topk_w), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(x) && aligned16(w_gate) && aligned16(bias) && aligned16(topk_idx) && aligned16(topk_w) &&
                    aligned16(counts) && aligned16(affinity_out),
                MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return do_route(x, w_gate, bias, sh, topk_idx, topk_w, counts, affinity_out, status, sms,
                    static_cast<cudaStream_t>(stream));
}

moe_status moe_load_and_bias_update(const int32_t* counts, moe_shape sh, float step, const float* target, float* bias,
                                    float* load_out, void* stream) {
    moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(sh.T > 0, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(counts && bias, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(step == step, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(counts) && aligned16(bias) && aligned16(target) && aligned16(load_out), MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return moe::launch_bias_update(counts, sh.T, sh.E, sh.k, step, target, bias, load_out,
                                   static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_permute(const void* x, const int32_t* topk_idx, const int32_t* counts, moe_shape sh, void* x_perm,
                       int32_t* offsets, int32_t* perm_tok, int32_t* inv_row, void* workspace, size_t ws_bytes,
                       void* stream) {
    moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(offsets, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (topk_idx && perm_tok && inv_row), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(!x_perm || sh.T == 0 || x, MOE_ERR_INVALID_ARG);  // x_perm null: index outputs only
    MOE_REQUIRE(aligned16(x) && aligned16(topk_idx) && aligned16(counts) && aligned16(x_perm) && aligned16(offsets) &&
                    aligned16(perm_tok) && aligned16(inv_row),
                MOE_ERR_ALIGNMENT);
    MOE_REQUIRE(ws_bytes >= permute_ws(sh) && (workspace || permute_ws(sh) == 0), MOE_ERR_WORKSPACE);
    MOE_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return do_permute(x, topk_idx, counts, sh, x_perm, offsets, perm_tok, inv_row, workspace, status,
                      static_cast<cudaStream_t>(stream));
}

moe_status moe_grouped_swiglu(const void* x_perm, const int32_t* offsets, const void* w1, const void* w3,
                              const void* w2, const void* x, const void* ws1, const void* ws3, const void* ws2,
                              moe_shape sh, void* y_perm, void* shared_out, void* workspace, size_t ws_bytes,
                              void* stream) {
    moe_status v = validate_dense_weights(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(offsets && w1 && w3 && w2, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (x_perm && y_perm), MOE_ERR_INVALID_ARG);
    const bool shared = x != nullptr && sh.S > 0;
    MOE_REQUIRE(!shared || (ws1 && ws3 && ws2 && shared_out), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(x_perm) && aligned16(offsets) && aligned16(w1) && aligned16(w3) && aligned16(w2) &&
                    aligned16(x) && aligned16(ws1) && aligned16(ws3) && aligned16(ws2) && aligned16(y_perm) &&
                    aligned16(shared_out),
                MOE_ERR_ALIGNMENT);
    MOE_REQUIRE(ws_bytes >= swiglu_ws(sh) && (workspace || swiglu_ws(sh) == 0), MOE_ERR_WORKSPACE);
    MOE_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return do_swiglu(x_perm, offsets, w1, w3, w2, shared ? x : nullptr, ws1, ws3, ws2, sh, y_perm, shared_out,
                     workspace, status, sms, static_cast<cudaStream_t>(stream));
}

moe_status moe_expert_up(const void* a, const int32_t* gather_idx, const int32_t* offsets, const void* w1,
                         const void* w3, moe_shape sh, int32_t set, void* h, void* stream) {
    moe_status v = validate_dense_weights(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(set == MOE_ROUTED || set == MOE_SHARED, MOE_ERR_INVALID_ARG);
    const bool shared = set == MOE_SHARED;
    MOE_REQUIRE(!shared || sh.S > 0, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(w1 && w3 && (shared || offsets), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (a && h), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(!shared || !gather_idx, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(a) && aligned16(gather_idx) && aligned16(offsets) && aligned16(w1) && aligned16(w3) &&
                    aligned16(h),
                MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return do_expert_up(a, gather_idx, offsets, w1, w3, sh, shared, h, status, sms,
                        static_cast<cudaStream_t>(stream));
}

moe_status moe_expert_down(const void* h, const int32_t* offsets, const void* w2, moe_shape sh, int32_t set, void* y,
                           void* stream) {
    moe_status v = validate_dense_weights(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(set == MOE_ROUTED || set == MOE_SHARED, MOE_ERR_INVALID_ARG);
    const bool shared = set == MOE_SHARED;
    MOE_REQUIRE(!shared || sh.S > 0, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(w2 && (shared || offsets), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (h && y), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(h) && aligned16(offsets) && aligned16(w2) && aligned16(y), MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return do_expert_down(h, offsets, w2, sh, shared, y, status, sms, static_cast<cudaStream_t>(stream));
}

moe_status moe_ffn_up(const void* x_perm, const int32_t* offsets, const void* w1, const void* w3, const void* x,
                      const void* ws1, const void* ws3, moe_shape sh, void* h, void* hs, void* stream) {
    moe_status v = validate_dense_weights(sh);
    if (v != MOE_OK) return v;
    const bool shared = x != nullptr && sh.S > 0;
    MOE_REQUIRE(offsets && w1 && w3, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (x_perm && h), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(!shared || (ws1 && ws3 && (sh.T == 0 || hs)), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(x_perm) && aligned16(offsets) && aligned16(w1) && aligned16(w3) && aligned16(x) &&
                    aligned16(ws1) && aligned16(ws3) && aligned16(h) && aligned16(hs),
                MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return do_ffn_up(x_perm, offsets, w1, w3, shared ? x : nullptr, ws1, ws3, sh, h, hs, status, sms,
                     static_cast<cudaStream_t>(stream));
}

moe_status moe_ffn_down(const void* h, const int32_t* offsets, const void* w2, const void* hs, const void* ws2,
                        moe_shape sh, void* y_perm, void* shared_out, void* stream) {
    moe_status v = validate_dense_weights(sh);
    if (v != MOE_OK) return v;
    const bool shared = hs != nullptr && sh.S > 0;
    MOE_REQUIRE(offsets && w2, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (h && y_perm), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(!shared || (ws2 && (sh.T == 0 || shared_out)), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(h) && aligned16(offsets) && aligned16(w2) && aligned16(hs) && aligned16(ws2) &&
                    aligned16(y_perm) && aligned16(shared_out),
                MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return do_ffn_down(h, offsets, w2, shared ? hs : nullptr, ws2, sh, y_perm, shared_out, status, sms,
                       static_cast<cudaStream_t>(stream));
}

moe_status moe_ffn_down_combine(const void* h, const int32_t* offsets, const void* w2, const void* hs,
                                const void* ws2, const int32_t* perm_tok, const float* topk_w, moe_shape sh,
                                float* y_acc, void* stream) {
    moe_status v = validate_dense_weights(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(sh.dtype == MOE_BF16, MOE_ERR_UNSUPPORTED);
    const bool shared = hs != nullptr && sh.S > 0;
    MOE_REQUIRE(offsets && w2, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (h && perm_tok && topk_w && y_acc), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(!shared || ws2, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(h) && aligned16(offsets) && aligned16(w2) && aligned16(hs) && aligned16(ws2) &&
                    aligned16(perm_tok) && aligned16(topk_w) && aligned16(y_acc),
                MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return do_ffn_down_combine(h, offsets, w2, shared ? hs : nullptr, ws2, perm_tok, topk_w, sh, y_acc, status, sms,
                               static_cast<cudaStream_t>(stream));
}

moe_status moe_combine_finish(float* y_acc, moe_shape sh, void* y, void* stream) {
    moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(sh.T == 0 || (y_acc && y), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(y_acc) && aligned16(y), MOE_ERR_ALIGNMENT);
    MOE_REQUIRE(sh.d % 8 == 0, MOE_ERR_UNSUPPORTED);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return moe::launch_combine_finish(y_acc, (long long)sh.T * sh.d, sh.dtype != MOE_F32, y,
                                      static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_combine(const void* y_perm, const float* topk_w, const int32_t* inv_row, const void* shared_out,
                       moe_shape sh, void* y, void* stream) {
    moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(sh.T == 0 || (y_perm && topk_w && inv_row && y), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(y_perm) && aligned16(topk_w) && aligned16(inv_row) && aligned16(shared_out) && aligned16(y),
                MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return moe::launch_combine(y_perm, topk_w, inv_row, shared_out, sh.T, sh.d, sh.k, sh.dtype != MOE_F32, y, status,
                               static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

size_t moe_backward_workspace_size(moe_shape sh, int32_t seq_len) {
    if (validate_dense_weights(sh) != MOE_OK) return 0;
    return moe::backward_scratch_bytes(sh.T, sh.d, sh.E, sh.k, sh.I, sh.S, sh.Is, seq_len > 0 ? seq_len : 0,
                                       sh.dtype == MOE_BF16);
}

moe_status moe_layer_backward(const void* x, const void* w_gate, const void* w1, const void* w3, const void* w2,
                              const void* ws1, const void* ws3, const void* ws2, moe_shape sh, const int32_t* topk_idx,
                              const float* topk_w, const int32_t* counts, const float* affinity, const float* dy,
                              float alpha, int32_t seq_len, float* dx, float* dw_gate, float* dw1, float* dw3,
                              float* dw2, float* dws1, float* dws3, float* dws2, float* balance_loss, void* workspace,
                              size_t ws_bytes, void* stream) {
    moe_status v = validate_dense_weights(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(w_gate && w1 && w3 && w2 && counts && dw_gate && dw1 && dw3 && dw2, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (x && topk_idx && topk_w && affinity && dy && dx), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.S == 0 || (ws1 && ws3 && ws2 && dws1 && dws3 && dws2), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(alpha == alpha && alpha >= 0.0f && alpha < 3.0e38f, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(alpha == 0.0f || (seq_len > 0 && sh.T % seq_len == 0), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(alpha == 0.0f || sh.T / seq_len <= 65535, MOE_ERR_UNSUPPORTED);  // sequences per launch
    MOE_REQUIRE(aligned16(x) && aligned16(w_gate) && aligned16(w1) && aligned16(w3) && aligned16(w2) &&
                    aligned16(ws1) && aligned16(ws3) && aligned16(ws2) && aligned16(topk_idx) && aligned16(topk_w) &&
                    aligned16(counts) && aligned16(affinity) && aligned16(dy) && aligned16(dx) &&
                    aligned16(dw_gate) && aligned16(dw1) && aligned16(dw3) && aligned16(dw2) && aligned16(dws1) &&
                    aligned16(dws3) && aligned16(dws2),
                MOE_ERR_ALIGNMENT);
    const int32_t L = alpha > 0.0f ? seq_len : 0;
    const size_t need = moe::backward_scratch_bytes(sh.T, sh.d, sh.E, sh.k, sh.I, sh.S, sh.Is, L, sh.dtype == MOE_BF16);
    MOE_REQUIRE(workspace && ws_bytes >= need, MOE_ERR_WORKSPACE);
    MOE_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    moe::BackwardArgs a{};
    a.x = x;
    a.w_gate = w_gate;
    a.w1 = w1;
    a.w3 = w3;
    a.w2 = w2;
    a.ws1 = ws1;
    a.ws3 = ws3;
    a.ws2 = ws2;
    a.T = sh.T;
    a.d = sh.d;
    a.E = sh.E;
    a.k = sh.k;
    a.I = sh.I;
    a.S = sh.S;
    a.Is = sh.Is;
    a.bf16 = sh.dtype == MOE_BF16;
    a.idx = topk_idx;
    a.w = topk_w;
    a.counts = counts;
    a.s = affinity;
    a.dy = dy;
    a.alpha = alpha;
    a.seq_len = L;
    a.dx = dx;
    a.dw_gate = dw_gate;
    a.dw1 = dw1;
    a.dw3 = dw3;
    a.dw2 = dw2;
    a.dws1 = dws1;
    a.dws3 = dws3;
    a.dws2 = dws2;
    a.loss = balance_loss;
    a.workspace = workspace;
    a.num_sms = sms;
    return moe::launch_layer_backward(a, status, sms, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_layer_forward(const void* x, const void* w_gate, const float* bias, const void* w1, const void* w3,
                             const void* w2, const void* ws1, const void* ws3, const void* ws2, moe_shape sh, void* y,
                             int32_t* topk_idx, float* topk_w, int32_t* counts, void* workspace, size_t ws_bytes,
                             void* stream) {
    moe_status v = validate_dense_weights(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(w_gate && bias && w1 && w3 && w2 && counts, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.S == 0 || (ws1 && ws3 && ws2), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (x && y && topk_idx && topk_w), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(x) && aligned16(w_gate) && aligned16(bias) && aligned16(w1) && aligned16(w3) &&
                    aligned16(w2) && aligned16(ws1) && aligned16(ws3) && aligned16(ws2) && aligned16(y) &&
                    aligned16(topk_idx) && aligned16(topk_w) && aligned16(counts),
                MOE_ERR_ALIGNMENT);
    const size_t need = moe_workspace_size(sh);
    MOE_REQUIRE(workspace && ws_bytes >= need, MOE_ERR_WORKSPACE);
    MOE_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    const size_t rows = (size_t)sh.T * sh.k;
    const size_t eb = esize(sh);
    char* p = static_cast<char*>(workspace);
    int32_t* offsets = reinterpret_cast<int32_t*>(p);
    p += align256((sh.E + 1) * sizeof(int32_t));
    int32_t* perm = reinterpret_cast<int32_t*>(p);
    p += align256(rows * sizeof(int32_t));
    int32_t* inv = reinterpret_cast<int32_t*>(p);
    p += align256(rows * sizeof(int32_t));
    void* pws = p;
    p += permute_ws(sh);
    void* x_perm = p;  // x_perm, then y_perm
    p += align256(rows * sh.d * eb);
    void* gws = p;
    p += swiglu_ws(sh);
    void* shared_out = sh.S > 0 ? p : nullptr;

    // route; permute (token rows copied into expert order: a row gather
    // inside the GEMM's loads, tile::gather4, measured 2x slower for the
    // routed up projection than this copy plus whole-tile loads)
    void* y_perm = x_perm;  // the down projection overwrites x_perm once the up projection has read it
    if ((v = do_route(x, w_gate, bias, sh, topk_idx, topk_w, counts, nullptr, status, sms, st)) != MOE_OK) return v;
    if (sh.T == 0) return MOE_OK;
    if ((v = do_permute(x, topk_idx, counts, sh, x_perm, offsets, perm, inv, pws, status, st)) != MOE_OK) return v;
    if ((v = do_swiglu(x_perm, offsets, w1, w3, w2, sh.S > 0 ? x : nullptr, ws1, ws3, ws2, sh, y_perm, shared_out,
                       gws, status, sms, st)) != MOE_OK)
        return v;
    return moe::launch_combine(y_perm, topk_w, inv, shared_out, sh.T, sh.d, sh.k, sh.dtype != MOE_F32, y, status,
                               st) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

size_t moe_fp8_scale_bytes(int64_t rows, int32_t K, int32_t layout) {
    if (rows < 0 || K <= 0 || K % 128 != 0 || layout < MOE_SF_TOKENS || layout > MOE_SF_UP) return 0;
    return moe::mx_scale_bytes(rows, K, layout);
}

moe_status moe_quantize_fp8(const void* src, int64_t rows, int32_t kseg, int32_t nseg, int32_t layout, uint8_t* q,
                            void* scales, void* stream) {
    MOE_REQUIRE(rows >= 0 && kseg > 0 && nseg >= 1, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(layout >= MOE_SF_TOKENS && layout <= MOE_SF_UP, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(kseg % 128 == 0, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE((long long)kseg * nseg < (1ll << 31), MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(rows == 0 || (src && q && scales), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(src) && aligned16(q) && aligned16(scales), MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    moe_status v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return moe::launch_quantize_mx(src, rows, kseg, nseg, layout, q, scales, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

size_t moe_fp8_tile_scale_bytes(int64_t rows, int32_t groups, int32_t K) {
    if (rows < 0 || groups < 1 || groups > moe::kMaxGroups || K <= 0 || K % 128 != 0) return 0;
    return tile_image_bytes(rows, groups, K);
}

moe_status moe_fp8_tile_scales(const void* src, int64_t src_rows, int32_t K, const int32_t* row_of, int32_t row_div,
                               const int32_t* offsets, int32_t groups, int64_t rows, void* tiles, void* stream) {
    MOE_REQUIRE(src_rows >= 0 && rows >= 0 && K > 0 && row_div >= 1, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(groups >= 1 && groups <= moe::kMaxGroups && (offsets || groups == 1), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(K % 128 == 0, MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(rows < (1ll << 31) && src_rows < (1ll << 31), MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(rows == 0 || (src && tiles), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(src) && aligned16(row_of) && aligned16(offsets) && aligned16(tiles), MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    moe_status v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return moe::launch_tile_scales(src, src_rows, K, row_of, row_div, offsets, groups, rows, tiles, status,
                                   static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_ffn_up_fp8(const uint8_t* xq_perm, const void* x_tiles, const int32_t* offsets, const uint8_t* xq,
                          const void* xsh_tiles, const moe_fp8_experts* w, moe_shape sh, void* h, void* hs,
                          void* stream) {
    moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(is_fp8(sh), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(offsets && fp8_weights_ok(w, sh), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (xq_perm && x_tiles && h), MOE_ERR_INVALID_ARG);
    const bool shared = xq != nullptr && sh.S > 0;
    MOE_REQUIRE(!shared || sh.T == 0 || (xsh_tiles && hs), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(xq_perm) && aligned16(x_tiles) && aligned16(xsh_tiles) && aligned16(offsets) &&
                    aligned16(xq) && aligned16(h) && aligned16(hs) && fp8_weights_aligned(w),
                MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return do_ffn_up_fp8(xq_perm, x_tiles, offsets, shared ? xq : nullptr, xsh_tiles, w, sh, h, hs, status, sms,
                         static_cast<cudaStream_t>(stream));
}

moe_status moe_ffn_up_fp8_quant(const uint8_t* xq_perm, const void* x_tiles, const int32_t* offsets,
                                const uint8_t* xq, const void* xsh_tiles, const moe_fp8_experts* w, moe_shape sh,
                                uint8_t* hq, void* h_tiles, uint8_t* hsq, void* hs_tiles, void* stream) {
    moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(is_fp8(sh), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(offsets && fp8_weights_ok(w, sh), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (xq_perm && x_tiles && hq && h_tiles), MOE_ERR_INVALID_ARG);
    const bool shared = xq != nullptr && sh.S > 0;
    MOE_REQUIRE(!shared || sh.T == 0 || (xsh_tiles && hsq && hs_tiles), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(xq_perm) && aligned16(x_tiles) && aligned16(xsh_tiles) && aligned16(offsets) &&
                    aligned16(xq) && aligned16(hq) && aligned16(h_tiles) && aligned16(hsq) && aligned16(hs_tiles) &&
                    fp8_weights_aligned(w),
                MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return do_ffn_up_fp8(xq_perm, x_tiles, offsets, shared ? xq : nullptr, xsh_tiles, w, sh, nullptr, nullptr,
                         status, sms, static_cast<cudaStream_t>(stream), hq, h_tiles, shared ? hsq : nullptr,
                         shared ? hs_tiles : nullptr);
}

moe_status moe_ffn_down_fp8(const uint8_t* hq, const void* h_tiles, const int32_t* offsets, const uint8_t* hsq,
                            const void* hs_tiles, const moe_fp8_experts* w, moe_shape sh, void* y_perm,
                            void* shared_out, void* stream) {
    moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(is_fp8(sh), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(offsets && fp8_weights_ok(w, sh), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (hq && h_tiles && y_perm), MOE_ERR_INVALID_ARG);
    const bool shared = hsq != nullptr && sh.S > 0;
    MOE_REQUIRE(!shared || sh.T == 0 || (hs_tiles && shared_out), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(hq) && aligned16(h_tiles) && aligned16(offsets) && aligned16(hsq) && aligned16(hs_tiles) &&
                    aligned16(y_perm) && aligned16(shared_out) && fp8_weights_aligned(w),
                MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return do_ffn_down_fp8(hq, h_tiles, offsets, shared ? hsq : nullptr, hs_tiles, w, sh, y_perm, shared_out, status,
                           sms, static_cast<cudaStream_t>(stream));
}

moe_status moe_layer_forward_fp8(const void* x, const void* w_gate, const float* bias, const moe_fp8_experts* w,
                                 moe_shape sh, void* y, int32_t* topk_idx, float* topk_w, int32_t* counts,
                                 void* workspace, size_t ws_bytes, void* stream) {
    moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(is_fp8(sh), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(w_gate && bias && counts && fp8_weights_ok(w, sh), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(sh.T == 0 || (x && y && topk_idx && topk_w), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(x) && aligned16(w_gate) && aligned16(bias) && aligned16(y) && aligned16(topk_idx) &&
                    aligned16(topk_w) && aligned16(counts) && fp8_weights_aligned(w),
                MOE_ERR_ALIGNMENT);
    MOE_REQUIRE(workspace && ws_bytes >= fp8_work(sh, nullptr, nullptr), MOE_ERR_WORKSPACE);
    MOE_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Fp8Work k8;
    fp8_work(sh, static_cast<char*>(workspace), &k8);
    const bool shared = sh.S > 0;
    if ((v = do_route(x, w_gate, bias, sh, topk_idx, topk_w, counts, nullptr, status, sms, st)) != MOE_OK) return v;
    if (sh.T == 0) return MOE_OK;
    if (moe::launch_quantize_mx(x, sh.T, sh.d, 1, moe::kMxTokens, k8.xq, k8.xs, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if ((v = do_permute(k8.xq, topk_idx, counts, sh, k8.xq_perm, k8.offsets, k8.perm, k8.inv, k8.pws, status, st)) !=
        MOE_OK)
        return v;
    // the token images of the tiles (routed rows through the permutation, the shared experts' rows as they
    // are), then gate/up with h (and hs) quantized by tiles in its epilogue
    const long long rows = (long long)sh.T * sh.k;
    if (moe::launch_tile_scales(k8.xs, sh.T, sh.d, k8.perm, sh.k, k8.offsets, sh.E, rows, k8.x_tiles, status, st) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    if (shared && moe::launch_tile_scales(k8.xs, sh.T, sh.d, nullptr, 1, nullptr, 1, sh.T, k8.xsh_tiles, status, st) !=
                      cudaSuccess)
        return MOE_ERR_CUDA;
    if ((v = do_ffn_up_fp8(k8.xq_perm, k8.x_tiles, k8.offsets, shared ? k8.xq : nullptr, k8.xsh_tiles, w, sh, nullptr,
                           nullptr, status, sms, st, k8.hq, k8.h_tiles, shared ? k8.hsq : nullptr,
                           shared ? k8.hs_tiles : nullptr)) != MOE_OK)
        return v;
    if ((v = do_ffn_down_fp8(k8.hq, k8.h_tiles, k8.offsets, shared ? k8.hsq : nullptr, k8.hs_tiles, w, sh, k8.y_perm,
                             k8.shared_out, status, sms, st)) != MOE_OK)
        return v;
    return moe::launch_combine(k8.y_perm, topk_w, k8.inv, shared ? k8.shared_out : nullptr, sh.T, sh.d, sh.k, true, y,
                               status, st) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

size_t moe_ep_plan_size(int32_t world, moe_shape sh) {
    if (validate_shape(sh) != MOE_OK || world < 1 || world > moe::kMaxRanks || sh.E % world != 0) return 0;
    return align256(moe::ep_plan_ints(world, sh.E) * sizeof(int32_t));
}

moe_status moe_ep_plan(const int32_t* counts_all, int32_t world, int32_t rank, moe_shape sh, int64_t recv_capacity,
                       int32_t* plan, int32_t* recv_offsets, void* stream) {
    moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(world >= 1 && world <= moe::kMaxRanks && sh.E % world == 0 && rank >= 0 && rank < world,
                MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(counts_all && plan, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(recv_capacity > 0 && recv_capacity <= 0x7fffffffLL, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(counts_all) && aligned16(plan) && aligned16(recv_offsets), MOE_ERR_ALIGNMENT);
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (moe::launch_ep_plan(counts_all, world, sh.E, (long long)recv_capacity, plan, status, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (recv_offsets) {
        const int Epr = sh.E / world;
        const size_t at = (size_t)sh.E * world + (size_t)world * (sh.E + 1) + (size_t)rank * (Epr + 1);
        MOE_CUDA(cudaMemcpyAsync(recv_offsets, plan + at, sizeof(int32_t) * (Epr + 1), cudaMemcpyDeviceToDevice, st));
    }
    return MOE_OK;
}

namespace {
moe_status ep_peers(void* const* bufs, int32_t world, moe::EpPeers* out) {
    MOE_REQUIRE(bufs, MOE_ERR_INVALID_ARG);
    for (int i = 0; i < moe::kMaxRanks; ++i) out->p[i] = nullptr;
    for (int i = 0; i < world; ++i) {
        MOE_REQUIRE(bufs[i], MOE_ERR_INVALID_ARG);
        MOE_REQUIRE(aligned16(bufs[i]), MOE_ERR_ALIGNMENT);
        out->p[i] = bufs[i];
    }
    return MOE_OK;
}
}  // namespace

moe_status moe_ep_dispatch(const void* x, const int32_t* perm_tok, const int32_t* plan, int32_t world, int32_t rank,
                           moe_shape sh, void* const* recv_bufs, void* stream) {
    moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(!is_fp8(sh), MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(world >= 1 && world <= moe::kMaxRanks && sh.E % world == 0 && rank >= 0 && rank < world,
                MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(plan && (sh.T == 0 || (x && perm_tok)), MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(x) && aligned16(perm_tok) && aligned16(plan), MOE_ERR_ALIGNMENT);
    moe::EpPeers peers;
    if ((v = ep_peers(recv_bufs, world, &peers)) != MOE_OK) return v;
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    if (sh.T == 0) return MOE_OK;
    return moe::launch_ep_dispatch(x, perm_tok, plan, world, sh.E, sh.k, rank, sh.T, (size_t)sh.d * esize(sh), peers,
                                   sms, status, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_ep_return(const void* y_recv, const int32_t* plan, int32_t world, int32_t rank, moe_shape sh,
                         void* const* back_bufs, void* stream) {
    moe_status v = validate_shape(sh);
    if (v != MOE_OK) return v;
    MOE_REQUIRE(!is_fp8(sh), MOE_ERR_UNSUPPORTED);
    MOE_REQUIRE(world >= 1 && world <= moe::kMaxRanks && sh.E % world == 0 && rank >= 0 && rank < world,
                MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(plan && y_recv, MOE_ERR_INVALID_ARG);
    MOE_REQUIRE(aligned16(y_recv) && aligned16(plan), MOE_ERR_ALIGNMENT);
    moe::EpPeers peers;
    if ((v = ep_peers(back_bufs, world, &peers)) != MOE_OK) return v;
    int dev, sms;
    int* status;
    v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return moe::launch_ep_return(y_recv, plan, world, sh.E, sh.k, rank, sh.T, (size_t)sh.d * esize(sh), peers, sms,
                                 status, static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_selftest_bounded_wait(uint32_t limit_us, void* stream) {
    MOE_REQUIRE(limit_us > 0 && limit_us <= 5000000u, MOE_ERR_INVALID_ARG);
    int dev, sms;
    int* status;
    moe_status v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    return moe::launch_bounded_wait_selftest((uint64_t)limit_us * 1000ull, status,
                                             static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}

moe_status moe_get_last_error(void* stream) {
    int dev, sms;
    int* status;
    moe_status v = device_setup(&dev, &status, &sms);
    if (v != MOE_OK) return v;
    MOE_CUDA(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)));
    int h = 0;
    MOE_CUDA(cudaMemcpy(&h, status, sizeof(int), cudaMemcpyDeviceToHost));
    const int zero = 0;
    MOE_CUDA(cudaMemcpy(status, &zero, sizeof(int), cudaMemcpyHostToDevice));
    return static_cast<moe_status>(h);
}

}  // extern "C"
