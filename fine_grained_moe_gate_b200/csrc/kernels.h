// Internal launchers of the MoE kernels (host side).  Not part of the ABI;
// the entry points in capi.cu validate arguments before calling these.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

constexpr int kMaxExperts = 256;

// Adds n to the library's kernel-launch counter (moe_kernel_launch_count).
void note_launches(int n);
constexpr int kMaxGroups = kMaxExperts;

// One grouped GEMM C = A . B^T (optionally with the SwiGLU pair B0/B1).
// Group g: rows [offsets[g], offsets[g+1]) of A and C, all inside [0, M)
// (or [0, M) itself when offsets is null and G == 1); B block g starts b_gstride elements after
// block g-1.  Element (n, kk) of a B block sits at
//   (kk / kseg) * seg_stride + n * ldb + (kk % kseg)
// which covers both a plain [N][K] matrix (kseg = K) and S stacked
// [N][Is] matrices contracted over their concatenated K (kseg = Is).
struct GemmArgs {
    const void* A;
    int lda;
    const void* B0;
    const void* B1;
    long long b_gstride;
    int ldb;
    int kseg;
    long long seg_stride;
    void* C;
    int ldc;
    int N, K;
    const int32_t* offsets;
    int G;
    int M;
    const int32_t* gather;  // optional: A row of group row r is gather[r] / gather_div
    int gather_div;
};

// quant.cu: per-tile E4M3 quantization (scale layouts described there)
enum MxLayout { kMxTokens = 0, kMxWeights = 1, kMxGate = 2, kMxUp = 3 };
size_t mx_scale_bytes(long long rows, int K, int layout);
cudaError_t launch_quantize_mx(const void* src, long long rows, int kseg, int nseg, int layout, uint8_t* q,
                               void* scales, cudaStream_t st);
// Token images of the grouped GEMMs' tiles: groups [offsets[g], offsets[g+1])
// (offsets null: one group of `rows` rows); tile images in group order, row
// j of a tile taking the token-layout words of src row row_of[r] / row_div
// (row_of null: r itself) of src [K/128][src_rows].  max_tiles bounds the
// images written (mx_tile_images).
long long mx_tile_images(long long rows, int groups);
cudaError_t launch_tile_scales(const void* src, long long src_rows, int K, const int32_t* row_of, int row_div,
                               const int32_t* offsets, int groups, long long rows, void* out, int* status,
                               cudaStream_t st);

// combine.cu: y = dtype(acc) for n elements (n % 8 == 0), then acc = 0
cudaError_t launch_combine_finish(float* acc, long long n, bool bf16, void* y, cudaStream_t st);

// router.cu
cudaError_t launch_router_simt(const void* x, const void* wg, const float* bias, int T, int d, int E, int k,
                               bool bf16, int32_t* idx, float* w, int32_t* counts, float* aff, int* status,
                               cudaStream_t st);
size_t router_simt_smem(int E);
cudaError_t launch_bias_update(const int32_t* counts, int T, int E, int k, float step, const float* target,
                               float* bias, float* load_out, cudaStream_t st);

// router_tc.cu (bf16, tensor cores)
cudaError_t launch_router_tc(const void* x, const void* wg, const float* bias, int T, int d, int E, int k,
                             int32_t* idx, float* w, int32_t* counts, float* aff, int* status, int num_sms,
                             cudaStream_t st);

// permute.cu
size_t permute_scratch_bytes(int T, int E);
cudaError_t launch_permute(const void* x, const int32_t* idx, const int32_t* counts, int T, int d, int E, int k,
                           size_t elem_bytes, void* x_perm, int32_t* offsets, int32_t* perm_tok, int32_t* inv_row,
                           int32_t* scratch, int* status, cudaStream_t st);

// backward.cu: the layer backward (fp32 SIMT contractions).  Pointers as in
// moe_layer_backward; x and the weights bf16 when bf16, else fp32.
struct BackwardArgs {
    const void *x, *w_gate, *w1, *w3, *w2, *ws1, *ws3, *ws2;
    int T, d, E, k, I, S, Is;
    bool bf16;
    const int32_t* idx;
    const float* w;
    const int32_t* counts;
    const float* s;
    const float* dy;
    float alpha;
    int seq_len;
    float *dx, *dw_gate, *dw1, *dw3, *dw2, *dws1, *dws3, *dws2, *loss;
    void* workspace;
    int num_sms;
};
size_t backward_scratch_bytes(int T, int d, int E, int k, int I, int S, int Is, int seq_len, bool bf16);
bool backward_on_tensor_cores(bool bf16, int d, int I, int S, int Is);
cudaError_t launch_layer_backward(const BackwardArgs& a, int* status, int num_sms, cudaStream_t st);

// gemm_bwd_tc.cu: the backward's grouped GEMMs on the tensor cores (bf16 in,
// fp32 out).  Groups: rows [start[g], start[g] + rows[g]) of the per-row
// operands (a padded layout: each group's segment zero-padded to a multiple
// of 64 rows), or one group of M_rows rows from 0 when start is null.
struct BwdRowsArgs {
    const void* W;          // K-major: [W_rows][K]; MN-major: [W_rows][M_total] (rows run along K)
    const void* W1;         // MN-major only, may be null: read after the first K0 rows of W's group
    long long W_rows;
    int K0;
    long long a_grow;       // weight rows per group (K-major: along M; MN-major: along K)
    const void* X;          // [op_rows][K] per-row operand
    long long op_rows;
    int K;
    int M_total;            // output features
    const int32_t* start;
    const int32_t* rows;
    int G;
    int M_rows;
    float* out;             // [op_rows][ldo] fp32
    int ldo;
    bool accumulate;
};
cudaError_t launch_bwd_rows_mnmajor(const BwdRowsArgs& a, int* status, int num_sms, cudaStream_t st);
// out[g][m][n] = sum over group g's rows r (padded to 64) of A[r][a_col0 + m] * B[r][b_col0 + n]
struct BwdWgradArgs {
    const void* A;
    int lda;
    long long a_col0;
    const void* B;
    int ldb;
    long long b_col0;
    long long op_rows;
    int M_total, N_total;   // multiples of 128
    const int32_t* start;
    const int32_t* rows;
    int G;
    int M_rows;
    float* out;             // [G][M_total][N_total] fp32
};
cudaError_t launch_bwd_wgrad(const BwdWgradArgs& a, int* status, int num_sms, cudaStream_t st);

// gemm_simt.cu
cudaError_t launch_simt_gemm(const GemmArgs& p, bool bf16, bool swiglu, int num_sms, cudaStream_t st);

// gemm_tc.cu (bf16, tensor cores)
// Up projection with fused SwiGLU: h[r][n] = silu(A W1^T) * (A W3^T).
//   A: [rows][d] (x_perm, or x for the shared group), W1/W3 row blocks of I
//   rows per group, h: [rows][I].
struct TcUpArgs {
    const void* A;          // [A_rows][d] bf16
    long long A_rows;
    const int32_t* gather;  // optional: group row r reads A row gather[r] / gather_div (A = x, unpermuted)
    int gather_div;
    long long gather_rows;  // rows the groups index when gathering (T * k)
    const void* W1;         // [G * I][d] bf16 (groups stacked)
    const void* W3;
    long long W_rows;       // G * I
    void* H;                // [A_rows][I] bf16
    int d, I;
    const int32_t* offsets; // group rows; null: one group of M rows
    int G, M;
    // E4M3 operands (A, W1, W3 one byte per element) with per-tile scales
    // (quant.cu layouts): w13s the joint W1/W3 scale units ([W_rows / 64][d /
    // 128] x 512 bytes); xs the token images of the groups' tiles ([xs_tiles][d
    // / 128] x 1024 bytes, image i for the i-th token tile over the groups in
    // order).
    bool f8 = false;
    const uint8_t* w13s = nullptr;
    const uint32_t* xs = nullptr;
    long long xs_tiles = 0;
    // E4M3, optional: write h as E4M3 codes hq [A_rows][I] with its tile
    // scales as the down projection's token images hq_img ([tiles][I / 128] x
    // 1024 bytes, the same tiles) instead of bf16 H.
    uint8_t* hq = nullptr;
    uint32_t* hq_img = nullptr;
    // bf16 only, optional: also write the fp32 pre-activations a = W1 . x
    // (pre_a) and g = W3 . x (pre_g), [A_rows][I] each, beside h (the
    // backward's recompute).
    float* pre_a = nullptr;
    float* pre_g = nullptr;
};
// Down projection: Y[r][:] = H[r] . W2_g^T, W2_g = [d][K] (K = I), or for
// the shared group S stacked [d][Is] blocks contracted over K = S * Is.
struct TcDownArgs {
    const void* H;          // [H_rows][K] bf16
    long long H_rows;
    const void* W2;         // [G][d][kseg] bf16 (G = groups, or S for shared)
    int nseg;               // K / kseg segments (1 routed, S shared)
    int kseg;
    void* Y;                // [H_rows][d] bf16
    int d, K;
    const int32_t* offsets;
    int G, M;
    // E4M3 operands (H, W2 one byte per element) with per-tile scales: w2s
    // the 128-row atoms of W2 as [G * d] rows of K = nseg * kseg columns
    // ([G * d / 128][K / 128] x 512 bytes); hs the token images of H's tiles
    // ([hs_tiles][K / 128] x 1024 bytes).
    bool f8 = false;
    const uint8_t* w2s = nullptr;
    const uint32_t* hs = nullptr;
    long long hs_tiles = 0;
    // Weighted combine fused into the epilogue (acc non-null): Y is not
    // written; row r is scaled and added into acc [T][d] fp32 -- routed:
    // token row_tok[r] / row_k, weight row_w[row_tok[r]]; shared (row_tok
    // null): token r, weight 1.
    float* acc = nullptr;
    const int32_t* row_tok = nullptr;
    const float* row_w = nullptr;
    int row_k = 1;
};
// ep.cu: expert-parallel dispatch / return over peer memory.  Plan layout
// (int32): base [E][W], src_off [W][E+1], recv_off [W][E/W+1].
constexpr int kMaxRanks = 64;
struct EpPeers {
    void* p[kMaxRanks];  // per rank: a device pointer valid in this process (peer memory)
};
size_t ep_plan_ints(int W, int E);
cudaError_t launch_ep_plan(const int32_t* counts_all, int W, int E, long long recv_capacity, int32_t* plan,
                           int* status, cudaStream_t st);
// Every rank holds T tokens: receive buffers W*T*k rows, return buffers T*k.
cudaError_t launch_ep_dispatch(const void* x, const int32_t* perm_tok, const int32_t* plan, int W, int E, int k,
                               int rank, int T, size_t row_bytes, const EpPeers& recv, int num_sms, int* status,
                               cudaStream_t st);
cudaError_t launch_ep_return(const void* y, const int32_t* plan, int W, int E, int k, int rank, int T,
                             size_t row_bytes, const EpPeers& back, int num_sms, int* status, cudaStream_t st);


// One launch for the routed set (offsets) and/or the shared set (M rows);
// either pointer may be null.
cudaError_t launch_tc_up(const TcUpArgs* routed, const TcUpArgs* shared, int* status, int num_sms, cudaStream_t st);
cudaError_t launch_tc_down(const TcDownArgs* routed, const TcDownArgs* shared, int* status, int num_sms,
                           cudaStream_t st);

// selftest.cu
cudaError_t launch_bounded_wait_selftest(uint64_t limit_ns, int* status, cudaStream_t st);

// combine.cu
cudaError_t launch_combine(const void* y_perm, const float* w, const int32_t* inv_row, const void* shared, int T,
                           int d, int k, bool bf16, void* y, int* status, cudaStream_t st);

}  // namespace moe
