/*
 * moe_gate.h -- C ABI of the B200 (sm_100a) fine-grained MoE layer: the
 * forward (bf16 / fp32, and E4M3 experts), expert-parallel dispatch and
 * return, and the layer backward with the sequence-wise balance loss.
 *
 * The layer is the DeepSeek-V3 MoE feed-forward as the following web pages
 * state it (cited by page title and section):
 *   [P1] "DeepSeek V3 From Scratch": "The idea" (256 routed + 1 shared
 *        expert, top-8; bias acts on selection only, weights from the
 *        unbiased affinity; FP8 with fine-grained quantization tiles),
 *        "Worked example", "In code" (route() and update_bias()).
 *   [P2] "Scaling Efficiency: A Deep Dive into the DeepSeek-V3
 *        Architecture": DeepSeekMoE module sketch (shared experts on every
 *        token, routed experts combined with their gate weights).
 *   [P3] kbwen.com DeepSeek tag page: "A bias term for each expert"
 *        (per-step load over the whole batch, fixed +-0.001 bias step).
 *   [P4] "DeepSeek V3 Architecture Deep Dive: Multi-Head Latent Attention
 *        (MLA), DeepSeekMoE & FP8 Mixed Precision": "Throughput on NVIDIA
 *        H100/H800" (tokens routed to the same expert batched together),
 *        "FP8 Formats" (E4M3).
 *   [P5] crackai.dev "DeepSeek-V3": "How It Works" (all-to-all dispatch /
 *        combine kernels for expert parallelism; FP8 with per-tile scaling).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library allocates no device memory on any call.  Scratch space is
 *     passed in as `workspace` (size from the matching *_workspace_size).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  Arguments are validated on the host before
 *     anything is enqueued; on an error nothing is launched.
 *   - Layouts are row-major and contiguous.  Weights use nn.Linear's
 *     [out][in] layout: W_gate [E][d]; W1, W3 [E][I][d]; W2 [E][d][I];
 *     shared Ws1, Ws3 [S][Is][d]; Ws2 [S][d][Is].  x and y are [T][d].
 *   - dtype MOE_F32: x, weights, y, intermediates fp32.  MOE_BF16: x,
 *     weights, y, intermediates bf16; every contraction accumulates in
 *     fp32; affinities, router weights and the bias are always fp32.
 *   - Every tensor pointer must be 16-byte aligned (MOE_ERR_ALIGNMENT).
 *   - Anomalies found on the device (an expert index out of range, counts
 *     that disagree with the routing table, a pipeline wait that timed
 *     out) are recorded in a per-device status word and returned by
 *     moe_get_last_error().  Kernels never trap.
 *   - Not thread-safe across host threads for the same device status word
 *     (moe_get_last_error reads and clears it).
 */
#ifndef MOE_GATE_H
#define MOE_GATE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* bad size, null required pointer, k > E ... */
    MOE_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels cover  */
    MOE_ERR_ALIGNMENT = 3,     /* a pointer is not 16-byte aligned          */
    MOE_ERR_WORKSPACE = 4,     /* workspace missing or smaller than needed  */
    MOE_ERR_CUDA = 5,          /* a CUDA runtime call failed                */
    MOE_ERR_DEVICE_CHECK = 6,  /* a device-side consistency check failed    */
    MOE_ERR_TIMEOUT = 7        /* a device-side wait gave up (bounded spin) */
} moe_status;

/* MOE_FP8_E4M3: x, W_gate, y and the bf16 intermediates as MOE_BF16; the
 * expert GEMM operands (expert weights, token rows, h) in E4M3 with a
 * power-of-two scale per tile of 32 elements -- see the FP8 section below. */
typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_FP8_E4M3 = 2 } moe_dtype;

/* Problem sizes.  T tokens of width d; E routed experts, k chosen per
 * token; routed SwiGLU intermediate I; S shared experts of intermediate Is
 * (S may be 0). */
typedef struct {
    int32_t T, d, E, k, I, S, Is;
    int32_t dtype; /* moe_dtype */
} moe_shape;

/* Limits (validated): 1 <= k <= min(E, 16); E <= 256; d % 8 == 0.
 * MOE_BF16 additionally needs d % 64 == 0, I % 128 == 0 and Is % 128 == 0
 * (tensor-core tiles), MOE_FP8_E4M3 d % 128 == 0 as well (and I, Is % 128), else
 * MOE_ERR_UNSUPPORTED.  With MOE_FP8_E4M3, moe_route, moe_load_and_bias_update
 * and moe_combine behave as with MOE_BF16 and moe_permute moves E4M3 rows (one
 * byte per element); the bf16-weight calls (moe_grouped_swiglu, moe_ffn_*,
 * moe_expert_*, moe_layer_forward) return MOE_ERR_UNSUPPORTED. */

/* ---------------------------------------------------------------------------
 * moe_route -- gate affinities, bias-shifted top-k, unbiased weights and the
 * load histogram  [P1 "In code", route(); P1 "The idea"; P3 "A bias term for
 * each expert"].
 *   s[t][i]   = sigmoid( x[t] . W_gate[i] )            fp32 (fp32 accumulate)
 *   v[t][i]   = s[t][i] + bias[i]                        fp32
 *   topk_idx[t][0..k)  the k largest v, descending; equal v -> lower index
 *   topk_w[t][j]       = s[t][idx_j] / sum_{j'} s[t][idx_j'] (sum in slot
 *                        order, fp32, IEEE division)
 *   counts[i] = #{(t, j) : topk_idx[t][j] == i}   (overwritten, not added)
 * x [T][d] dtype; W_gate [E][d] dtype; bias [E] fp32 (read only);
 * topk_idx [T][k] int32; topk_w [T][k] fp32; counts [E] int32;
 * affinity_out: NULL, or [T][E] fp32 receiving s.
 * -------------------------------------------------------------------------*/
MOE_API moe_status moe_route(const void* x, const void* w_gate, const float* bias, moe_shape sh,
                     int32_t* topk_idx, float* topk_w, int32_t* counts, float* affinity_out,
                     void* stream);

/* ---------------------------------------------------------------------------
 * moe_load_and_bias_update -- auxiliary-loss-free balancing step, applied
 * once at the end of a training step  [P1 "In code", update_bias();
 * P3 "A bias term for each expert"].
 *   load[i] = counts[i] / T                      fp32, T = sh.T, the tokens
 *                                                the counts were taken over
 *   bias[i] = bias[i] + step * sign(target[i] - load[i])  (sign(0) = 0)
 * target: NULL means the uniform load k/E for every expert.  bias [E] fp32
 * is updated in place; load_out: NULL or [E] fp32.  step 0 leaves the bias
 * unchanged (the pages' final 0.0 phase).
 * -------------------------------------------------------------------------*/
MOE_API moe_status moe_load_and_bias_update(const int32_t* counts, moe_shape sh, float step, const float* target,
                                    float* bias, float* load_out, void* stream);

/* ---------------------------------------------------------------------------
 * moe_permute -- expert-contiguous token order  [P4 "Throughput on NVIDIA
 * H100/H800": tokens routed to the same expert are batched together].
 * Rows are ordered by (expert ascending, token ascending):
 *   offsets[e]       first row of expert e; offsets[E] = T*k   int32 [E+1]
 *   perm_tok[row]    = t*k + j, the assignment held by that row int32 [T*k]
 *   inv_row[t*k + j] = row                                     int32 [T*k]
 *   x_perm[row]      = x[t]                                    [T*k][d] dtype
 *                      (x_perm may be NULL: only the index outputs)
 * counts: the histogram from moe_route; it is cross-checked on the device
 * (MOE_ERR_DEVICE_CHECK via moe_get_last_error on a mismatch).
 * Out-of-range expert indices are reported the same way and skipped.
 * workspace: >= moe_permute_workspace_size(sh) bytes, 256-byte aligned.
 * -------------------------------------------------------------------------*/
MOE_API moe_status moe_permute(const void* x, const int32_t* topk_idx, const int32_t* counts, moe_shape sh, void* x_perm,
                       int32_t* offsets, int32_t* perm_tok, int32_t* inv_row, void* workspace, size_t ws_bytes,
                       void* stream);
MOE_API size_t moe_permute_workspace_size(moe_shape sh);

/* ---------------------------------------------------------------------------
 * moe_permute_noalloc -- moe_permute without a workspace argument.  The pages
 * have no counterpart: this is an interface for callers that cannot give the
 * library scratch memory (a host framework that owns all device memory and
 * offers its plugins no allocator, or a deployment that reserves a fixed
 * device-memory budget up front and forbids allocation at run time).
 * Same arguments, results and errors as moe_permute, minus workspace.  The
 * scratch lives in a fixed 256 KiB array inside the library's device image,
 * which every GPU that loads the library keeps until the process exits; it
 * holds ceil(T / 128) * E int32 counters, so problems needing more than
 * 65536 (e.g. T > 32768 with E = 256) are rejected with MOE_ERR_UNSUPPORTED
 * before anything is launched.  Nothing is allocated: no cudaMalloc, no
 * cudaFree.  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it; make that
 * first call before any stream capture.  All calls share the one array and
 * it keeps the last call's contents (this permutation overwrites every
 * counter it reads, so nothing needs clearing); calls that overlap on the
 * GPU -- on different streams, or from different host threads -- race on it.
 * -------------------------------------------------------------------------*/
MOE_API moe_status moe_permute_noalloc(const void* x, const int32_t* topk_idx, const int32_t* counts, moe_shape sh,
                                       void* x_perm, int32_t* offsets, int32_t* perm_tok, int32_t* inv_row,
                                       void* stream);

/* ---------------------------------------------------------------------------
 * moe_grouped_swiglu -- the routed experts as one grouped SwiGLU GEMM pair,
 * and optionally the always-on shared experts  [P2 DeepSeekMoE sketch:
 * per-expert MLPs on the tokens routed to them; shared experts on every
 * token; the MLP is SwiGLU without biases].
 *   for expert e, rows r in [offsets[e], offsets[e+1]):
 *     h        = silu(x_perm[r] . W1[e]^T) * (x_perm[r] . W3[e]^T)
 *                (stored once in dtype)
 *     y_perm[r] = h . W2[e]^T                          [T*k][d] dtype
 *   if x != NULL and S > 0, for every token t:
 *     shared_out[t] = sum_s SwiGLU_s(x[t])             [T][d] dtype
 * workspace: >= moe_grouped_swiglu_workspace_size(sh) bytes.
 * -------------------------------------------------------------------------*/
MOE_API moe_status moe_grouped_swiglu(const void* x_perm, const int32_t* offsets, const void* w1, const void* w3,
                              const void* w2, const void* x, const void* ws1, const void* ws3, const void* ws2,
                              moe_shape sh, void* y_perm, void* shared_out, void* workspace, size_t ws_bytes,
                              void* stream);
MOE_API size_t moe_grouped_swiglu_workspace_size(moe_shape sh);

/* ---------------------------------------------------------------------------
 * moe_expert_up / moe_expert_down -- the two grouped GEMMs moe_grouped_swiglu
 * is made of, callable one at a time (to keep h, or to time each launch).
 * `set` picks the expert set:
 *   MOE_ROUTED: a = x_perm [T*k][d], offsets [E+1] (group e owns rows
 *               [offsets[e], offsets[e+1])), W1/W3 [E][I][d], W2 [E][d][I],
 *               h [T*k][I], y = y_perm [T*k][d];
 *   MOE_SHARED: a = x [T][d] (offsets ignored, may be NULL), W1/W3 = Ws1/Ws3
 *               [S][Is][d], W2 = Ws2 [S][d][Is], h [T][S*Is] (shared expert s
 *               in columns [s*Is, (s+1)*Is)), y = shared_out [T][d] = the
 *               sum over the S shared experts.
 * gather_idx (MOE_ROUTED only, may be NULL): when given, `a` is the
 *   unpermuted x [T][d] and row r reads x[gather_idx[r] / k] -- pass
 *   moe_permute's perm_tok to skip the x_perm copy (saves T*k*d elements
 *   of memory; on B200 the row gather in the GEMM's loads is slower than
 *   the copy, so moe_layer_forward copies).
 *   up:   h[r] = silu(a[r] . W1_g^T) * (a[r] . W3_g^T)   stored once in dtype
 *   down: y[r] = h[r] . W2_g^T                            fp32 accumulate
 * Same sources as moe_grouped_swiglu.  Invalid for MOE_SHARED when S == 0.
 * -------------------------------------------------------------------------*/
typedef enum { MOE_ROUTED = 0, MOE_SHARED = 1 } moe_expert_set;

MOE_API moe_status moe_expert_up(const void* a, const int32_t* gather_idx, const int32_t* offsets, const void* w1,
                                 const void* w3, moe_shape sh, int32_t set, void* h, void* stream);
MOE_API moe_status moe_expert_down(const void* h, const int32_t* offsets, const void* w2, moe_shape sh, int32_t set,
                                   void* y, void* stream);

/* ---------------------------------------------------------------------------
 * moe_ffn_up / moe_ffn_down -- the routed AND the shared experts' projection
 * in one launch each: the shared set is one more group of the same
 * persistent grouped GEMM (bf16), so its tiles fill the SMs the routed
 * groups leave idle.  moe_grouped_swiglu is moe_ffn_up then moe_ffn_down.
 *   moe_ffn_up:   h  = moe_expert_up(x_perm; MOE_ROUTED)   [T*k][I]
 *                 hs = moe_expert_up(x;      MOE_SHARED)   [T][S*Is]
 *   moe_ffn_down: y_perm     = moe_expert_down(h;  MOE_ROUTED)  [T*k][d]
 *                 shared_out = moe_expert_down(hs; MOE_SHARED)  [T][d]
 * x == NULL (up), hs == NULL (down) or S == 0 leaves the shared set out
 * (hs / shared_out and the shared weights are then ignored).  Results are
 * bit-identical to the separate calls.  h must not alias x_perm or x; y_perm
 * may alias x_perm (moe_ffn_down does not read it).
 * -------------------------------------------------------------------------*/
MOE_API moe_status moe_ffn_up(const void* x_perm, const int32_t* offsets, const void* w1, const void* w3,
                              const void* x, const void* ws1, const void* ws3, moe_shape sh, void* h, void* hs,
                              void* stream);
MOE_API moe_status moe_ffn_down(const void* h, const int32_t* offsets, const void* w2, const void* hs,
                                const void* ws2, moe_shape sh, void* y_perm, void* shared_out, void* stream);

/* ---------------------------------------------------------------------------
 * moe_combine -- weighted combine back into token order  [P2 DeepSeekMoE
 * sketch: routed_out[mask] += w * expert(x[mask]); shared_out + routed_out].
 *   y[t] = shared_out[t] + sum_{j=0..k-1} topk_w[t][j] * y_perm[inv_row[t*k+j]]
 * accumulated in fp32 in that order, rounded once to dtype.
 * shared_out may be NULL (no shared term).
 * -------------------------------------------------------------------------*/
MOE_API moe_status moe_combine(const void* y_perm, const float* topk_w, const int32_t* inv_row, const void* shared_out,
                       moe_shape sh, void* y, void* stream);

/* ---------------------------------------------------------------------------
 * moe_ffn_down_combine / moe_combine_finish -- moe_ffn_down and moe_combine
 * in one launch: the weighted combine fused into the down projection's
 * epilogue  [P2 DeepSeekMoE sketch: each routed expert's output scaled by
 * its gate weight and added to the token; shared output added].
 *   moe_ffn_down_combine: for every routed row r (assignment a =
 *       perm_tok[r], token a / k): y_acc[a / k] += topk_w[a] * (h[r] . W2_e^T),
 *       and with hs (S > 0) y_acc[t] += hs[t] . Ws2^T; fp32 additions straight
 *       from the fp32 accumulators (no bf16 rounding of expert outputs).
 *       y_acc [T][d] fp32 must hold zeros (or a partial sum to add to).  The
 *       additions of one element come from different tiles in no fixed
 *       order: y_acc is reproducible only up to fp32 rounding order.
 *   moe_combine_finish: y = dtype(y_acc) (one rounding), then y_acc = 0.
 * MOE_BF16 only (tensor-core path); perm_tok / topk_w from moe_permute /
 * moe_route.  Same weights and arguments as moe_ffn_down otherwise.
 * -------------------------------------------------------------------------*/
MOE_API moe_status moe_ffn_down_combine(const void* h, const int32_t* offsets, const void* w2, const void* hs,
                                        const void* ws2, const int32_t* perm_tok, const float* topk_w, moe_shape sh,
                                        float* y_acc, void* stream);
MOE_API moe_status moe_combine_finish(float* y_acc, moe_shape sh, void* y, void* stream);

/* ---------------------------------------------------------------------------
 * moe_layer_forward -- the whole layer: route, permute, grouped SwiGLU for
 * routed and shared experts, combine.  Same semantics as the five calls in
 * sequence.  The bias is read, not updated (call moe_load_and_bias_update
 * with the returned counts at the end of a training step).
 * Outputs: y [T][d] dtype; topk_idx [T][k]; topk_w [T][k]; counts [E].
 * workspace: >= moe_workspace_size(sh) bytes.  No host synchronisation.
 * -------------------------------------------------------------------------*/
MOE_API moe_status moe_layer_forward(const void* x, const void* w_gate, const float* bias, const void* w1, const void* w3,
                             const void* w2, const void* ws1, const void* ws3, const void* ws2, moe_shape sh, void* y,
                             int32_t* topk_idx, float* topk_w, int32_t* counts, void* workspace, size_t ws_bytes,
                             void* stream);
MOE_API size_t moe_workspace_size(moe_shape sh);  /* moe_layer_forward, or moe_layer_forward_fp8 for MOE_FP8_E4M3 */

/* ---------------------------------------------------------------------------
 * moe_layer_backward -- gradients of the layer forward for the selection the
 * forward made  [P1 "In code", route(): the weights renormalised over the
 * chosen unbiased scores; P2 DeepSeekMoE sketch: shared + weighted routed
 * SwiGLU experts; P3 "A bias term for each expert": the bias enters only the
 * choice, so it and the choice carry no gradient, and a small complementary
 * sequence-wise balance loss is kept].
 * The balance loss is not defined on the pages; the DeepSeek-V3 report's
 * form is used: for each sequence of seq_len consecutive tokens,
 *   f_i = E / (k L) * #{t : i in topk_idx[t]},  P_i = 1/L sum_t s_ti / sum_j s_tj
 *   L_seq = alpha * sum_i f_i P_i,   balance_loss = mean over the T / L sequences.
 * Computes, for the objective <dy, y> + balance_loss:
 *   dx [T][d], dw_gate [E][d], dw1 / dw3 [E][I][d], dw2 [E][d][I],
 *   dws1 / dws3 [S][Is][d], dws2 [S][d][Is]   -- all fp32, overwritten;
 *   balance_loss: NULL or one fp32 (0 when alpha == 0).
 * Inputs: x, w_gate, w1, w3, w2, ws1, ws3, ws2 as in moe_layer_forward
 * (dtype MOE_F32 or MOE_BF16); topk_idx, topk_w and counts as moe_route
 * returned them; affinity [T][E] fp32, moe_route's affinity_out; dy [T][d]
 * fp32.  alpha >= 0; with alpha > 0, seq_len > 0 must divide T (at most
 * 65535 sequences per call, else MOE_ERR_UNSUPPORTED).  h is
 * recomputed and rounded like the forward's (bf16 layers); the output
 * rounding of y is treated as identity.  fp32 accumulation throughout.
 * dws1 / dws3 / dws2 and ws1 / ws3 / ws2 may be NULL when S == 0.
 * workspace: >= moe_backward_workspace_size(sh, seq_len) bytes, 256-byte
 * aligned.  MOE_FP8_E4M3: MOE_ERR_UNSUPPORTED.  No host synchronisation.
 * -------------------------------------------------------------------------*/
MOE_API moe_status moe_layer_backward(const void* x, const void* w_gate, const void* w1, const void* w3,
                                      const void* w2, const void* ws1, const void* ws3, const void* ws2, moe_shape sh,
                                      const int32_t* topk_idx, const float* topk_w, const int32_t* counts,
                                      const float* affinity, const float* dy, float alpha, int32_t seq_len, float* dx,
                                      float* dw_gate, float* dw1, float* dw3, float* dw2, float* dws1, float* dws3,
                                      float* dws2, float* balance_loss, void* workspace, size_t ws_bytes,
                                      void* stream);
MOE_API size_t moe_backward_workspace_size(moe_shape sh, int32_t seq_len);

/* ---------------------------------------------------------------------------
 * FP8 experts with per-tile scales  [P1 "The idea": FP8 mixed precision with
 * fine-grained quantization tiles; P5 "How It Works": per-tile scaling;
 * P4 "FP8 Formats": E4M3 for weights and activations].  The pages fix
 * neither the tile nor the scale arithmetic; read as:
 *   - a tile is 32 consecutive elements of a row along the contraction
 *     dimension (weights: an output row's input features; token rows and h:
 *     their features);
 *   - its scale is 2^e, e the smallest integer with amax <= 448 * 2^e (amax
 *     the tile's largest magnitude; 0 for an all-zero tile; e >= -127), kept
 *     as the byte e + 127;
 *   - codes are E4M3(v * 2^-e), nearest, ties to even (nothing saturates);
 *   - a dot product is sum over tiles of 2^(e_a + e_b) * sum_i a_i b_i in
 *     fp32 (the tensor cores' block-scaled E4M3 MMA).
 * E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa bits, no infinities, largest
 * finite 448.  Row lengths (K) must be multiples of 128.
 *
 * Scale layouts (moe_fp8_scale_bytes gives the size of each):
 *   MOE_SF_TOKENS  token rows and h: uint32 [K/128][rows]; word (s, r) holds
 *                  the four tile bytes of row r's columns [128 s, 128 s + 128)
 *                  (byte j = tile 4 s + j).
 *   MOE_SF_WEIGHTS W2 and Ws2: 512-byte atoms, one per 128 rows and 128
 *                  columns, [rows/128][K/128]; byte (m % 32) * 16 + (m / 32) *
 *                  4 + j of atom (r / 128, s) is tile 4 s + j of row r, m =
 *                  r % 128.
 *   MOE_SF_GATE,   W1 and W3 (Ws1 and Ws3) share ONE buffer of 512-byte
 *   MOE_SF_UP      units, one per 64 rows and 128 columns, [rows/64][K/128];
 *                  byte (m % 32) * 16 + (m / 32) * 4 + j of unit (r / 64, s)
 *                  is tile 4 s + j of row r of W1 (MOE_SF_GATE, m = r % 64)
 *                  or of W3 (MOE_SF_UP, m = 64 + r % 64): quantize W1 with
 *                  MOE_SF_GATE and W3 with MOE_SF_UP into the same buffer.
 * These are the orders in which the GEMMs copy the scales of 128 operand rows
 * into tensor memory; treat them as opaque otherwise.
 *
 * Token tile images (moe_fp8_tile_scales): the grouped GEMMs run each group
 * of n rows as ceil(n / 256) token tiles of near-equal size (tile t has q +
 * (t < r) rows, q = n / tiles, r = n % tiles) and read the token scales of a
 * tile as one image of 256 uint32 words per 128 columns: [tiles][K/128][256],
 * the tiles of all groups in order; the word of the tile's row j sits at
 * (j / 128) * 128 + (j % 32) * 4 + (j / 32) % 4, zeros past its rows.
 * -------------------------------------------------------------------------*/
typedef enum { MOE_SF_TOKENS = 0, MOE_SF_WEIGHTS = 1, MOE_SF_GATE = 2, MOE_SF_UP = 3 } moe_sf_layout;

/* Bytes of the tile scales of a matrix of `rows` rows and K columns in the
 * given layout (0 if K % 128 != 0 or the layout is unknown; MOE_SF_GATE and
 * MOE_SF_UP give the size of the joint buffer). */
MOE_API size_t moe_fp8_scale_bytes(int64_t rows, int32_t K, int32_t layout);

/* moe_quantize_fp8 -- per-tile E4M3 quantization of a bf16 matrix with
 * `rows` rows stored as nseg column blocks of kseg columns ([nseg][rows][kseg];
 * nseg = 1 is plain row major; a row and its tiles span all blocks, K =
 * nseg * kseg).  q has src's layout, one byte per element; scales in
 * `layout`.  Needs kseg % 128 == 0; src, q and scales 16-byte aligned.
 * Used once per weight tensor (W1 / W3 [E][I][d] as rows = E*I with
 * MOE_SF_GATE / MOE_SF_UP into one buffer; W2 [E][d][I] as rows = E*d, kseg =
 * I, MOE_SF_WEIGHTS; the shared Ws1 / Ws3 [S][Is][d] as rows = S*Is likewise;
 * Ws2 [S][d][Is] as rows = d, kseg = Is, nseg = S) and per step for the token
 * rows and h (MOE_SF_TOKENS). */
MOE_API moe_status moe_quantize_fp8(const void* src, int64_t rows, int32_t kseg, int32_t nseg, int32_t layout,
                                    uint8_t* q, void* scales, void* stream);

/* Bytes of the token tile images of `rows` operand rows in `groups` groups
 * (1 <= groups <= 256) with K columns: room for rows / 256 + groups tiles. */
MOE_API size_t moe_fp8_tile_scale_bytes(int64_t rows, int32_t groups, int32_t K);

/* moe_fp8_tile_scales -- the token tile images of a grouped GEMM's token
 * operand of `rows` rows: groups [offsets[g], offsets[g+1]) (offsets NULL:
 * one group of all rows, groups = 1); operand row r takes the MOE_SF_TOKENS
 * words of row row_of[r] / row_div of src [K/128][src_rows] (row_of NULL:
 * row r).  Routed gate/up: src = the tokens' scales [d/128][T], row_of =
 * perm_tok, row_div = k, offsets from moe_permute, groups = E, rows = T*k;
 * shared experts: offsets NULL, rows = T; down from moe_quantize_fp8's h
 * scales: row_of NULL.  tiles: moe_fp8_tile_scale_bytes(rows, groups, K)
 * bytes, all of it written.  Pointers 16-byte aligned.  A row outside
 * [0, rows) or a source row outside src reports MOE_ERR_DEVICE_CHECK (its
 * word is left 0). */
MOE_API moe_status moe_fp8_tile_scales(const void* src, int64_t src_rows, int32_t K, const int32_t* row_of,
                                       int32_t row_div, const int32_t* offsets, int32_t groups, int64_t rows,
                                       void* tiles, void* stream);

/* E4M3 expert weights and their tile scales, all device pointers, 16-byte
 * aligned. */
typedef struct {
    const uint8_t* w1;  const uint8_t* w3;  const void* w13_scale;    /* [E][I][d] each, rows E*I, K = d;
                                                                        MOE_SF_GATE / MOE_SF_UP, one buffer */
    const uint8_t* w2;  const void* w2_scale;                         /* [E][d][I] rows E*d, K = I; MOE_SF_WEIGHTS */
    const uint8_t* ws1; const uint8_t* ws3; const void* ws13_scale;   /* [S][Is][d], rows S*Is, K = d (NULL if S == 0) */
    const uint8_t* ws2; const void* ws2_scale;                        /* [S][d][Is] rows d, K = S*Is (blocks joined) */
} moe_fp8_experts;

/* moe_ffn_up_fp8 / moe_ffn_up_fp8_quant / moe_ffn_down_fp8 -- moe_ffn_up /
 * moe_ffn_down on E4M3 operands (sh.dtype == MOE_FP8_E4M3), routed and shared
 * experts in one launch each.  Token scales come as tile images
 * (moe_fp8_tile_scales) of the same offsets:
 *   up:    xq_perm [T*k][d] E4M3 token rows in expert order (moe_permute of
 *          xq) with x_tiles; xq [T][d] the unpermuted quantized tokens with
 *          xsh_tiles (shared experts; xq NULL leaves them out).  h =
 *          bf16(silu(a) * g) with a, g the tile-scaled sums [T*k][I]; hs
 *          likewise [T][S*Is].
 *   quant: the same launch with h and hs leaving it quantized for the down
 *          projection: the epilogue rounds h to bf16 as moe_ffn_up_fp8 writes
 *          it, then quantizes each 1x32 tile as moe_quantize_fp8 does, so hq
 *          [T*k][I] / hsq [T][S*Is] equal the codes of that h, and h_tiles /
 *          hs_tiles its scales as tile images (equal to moe_fp8_tile_scales of
 *          moe_quantize_fp8's scales at every tile row; rows past a tile up to
 *          a multiple of 16 hold scale byte 127, the rest is not written),
 *          without the bf16 h round trip through HBM.
 *   down:  hq [T*k][I] with h_tiles, hsq [T][S*Is] with hs_tiles (NULL leaves
 *          the shared set out); y_perm [T*k][d] and shared_out [T][d] bf16.
 * Image buffers: moe_fp8_tile_scale_bytes(T*k, E, K) (routed) and (T, 1, K)
 * (shared).  Pointers 16-byte aligned. */
MOE_API moe_status moe_ffn_up_fp8(const uint8_t* xq_perm, const void* x_tiles, const int32_t* offsets,
                                  const uint8_t* xq, const void* xsh_tiles, const moe_fp8_experts* w, moe_shape sh,
                                  void* h, void* hs, void* stream);
MOE_API moe_status moe_ffn_up_fp8_quant(const uint8_t* xq_perm, const void* x_tiles, const int32_t* offsets,
                                        const uint8_t* xq, const void* xsh_tiles, const moe_fp8_experts* w,
                                        moe_shape sh, uint8_t* hq, void* h_tiles, uint8_t* hsq, void* hs_tiles,
                                        void* stream);
MOE_API moe_status moe_ffn_down_fp8(const uint8_t* hq, const void* h_tiles, const int32_t* offsets,
                                    const uint8_t* hsq, const void* hs_tiles, const moe_fp8_experts* w,
                                    moe_shape sh, void* y_perm, void* shared_out, void* stream);

/* moe_layer_forward_fp8 -- the layer with FP8 experts: route (bf16 x),
 * quantize x by tiles, permute the E4M3 rows, the token tile images,
 * gate/up with h and hs quantized by tiles in its epilogue
 * (moe_ffn_up_fp8_quant), down, combine
 * into y [T][d] bf16.  sh.dtype == MOE_FP8_E4M3;
 * workspace >= moe_workspace_size(sh). */
MOE_API moe_status moe_layer_forward_fp8(const void* x, const void* w_gate, const float* bias,
                                         const moe_fp8_experts* w, moe_shape sh, void* y, int32_t* topk_idx,
                                         float* topk_w, int32_t* counts, void* workspace, size_t ws_bytes,
                                         void* stream);

/* ---------------------------------------------------------------------------
 * Expert parallelism (no counterpart in the pages' code; their "custom
 * all-to-all kernels for MoE dispatch/combine", crackai.dev "DeepSeek-V3",
 * "How It Works").  W ranks, one per GPU; rank o owns experts
 * [o*E/W, (o+1)*E/W) (E % W == 0, W <= 64) and keeps its own T tokens.  Per
 * step, on every rank:
 *   1. moe_route and moe_permute (x_perm may be NULL) on the local tokens;
 *   2. gather all ranks' counts into counts_all [W][E] (any collective);
 *   3. moe_ep_plan: the receive layout, identical on every rank;
 *   4. moe_ep_dispatch: this rank's permuted rows go straight into the
 *      owners' receive buffers (peer stores); then a barrier across ranks;
 *   5. the grouped GEMMs (moe_ffn_up / moe_ffn_down, shape with E/W experts)
 *      on the receive buffer with recv_offsets; the shared experts on the
 *      local tokens (moe_expert_up / moe_expert_down, MOE_SHARED);
 *   6. moe_ep_return: each output row goes straight back into its source
 *      rank's return buffer, at the row's place in that rank's own
 *      permutation; then a barrier;
 *   7. moe_combine on the return buffer with the local inv_row.
 * A receive buffer holds its experts in order, each expert's rows by source
 * rank, each source's rows by token: the rows, and so the results, of the
 * single-GPU layer over the ranks' concatenated batch (same routing).
 * recv_capacity: rows every rank's receive buffer holds (the same on all
 * ranks).  W*T*k can never overflow; with the load balanced by the bias a
 * small multiple of T*k is enough.  If the step's counts would send more
 * rows to some owner than that, the plan records it and reports
 * MOE_ERR_DEVICE_CHECK, and moe_ep_dispatch / moe_ep_return with that plan
 * store nothing (no row is dropped silently).  Return buffers hold T*k rows.
 * recv_bufs / back_bufs: host arrays of W device pointers valid in the
 * calling process (peer memory, e.g. IPC or symmetric memory; on one GPU
 * plain allocations).  bf16 and fp32 rows; MOE_FP8_E4M3 is unsupported.
 * -------------------------------------------------------------------------*/
MOE_API size_t moe_ep_plan_size(int32_t world, moe_shape sh);  /* bytes; 0 if invalid */
MOE_API moe_status moe_ep_plan(const int32_t* counts_all, int32_t world, int32_t rank, moe_shape sh,
                               int64_t recv_capacity, int32_t* plan, int32_t* recv_offsets,
                               void* stream);  /* recv_offsets [E/W+1]: this rank's */
MOE_API moe_status moe_ep_dispatch(const void* x, const int32_t* perm_tok, const int32_t* plan, int32_t world,
                                   int32_t rank, moe_shape sh, void* const* recv_bufs, void* stream);
MOE_API moe_status moe_ep_return(const void* y_recv, const int32_t* plan, int32_t world, int32_t rank,
                                 moe_shape sh, void* const* back_bufs, void* stream);

/* Synchronises `stream`, then returns and clears the current device's
 * status word (MOE_OK if no kernel reported an anomaly). */
MOE_API moe_status moe_get_last_error(void* stream);

/* Failure-detection self-test (no counterpart in the pages): launches one
 * kernel that waits, with the same bounded mbarrier wait the pipelined
 * kernels use, on a barrier nothing arrives on.  After limit_us
 * microseconds (1 .. 5e6) the wait gives up and records MOE_ERR_TIMEOUT in
 * the device status word, which moe_get_last_error then returns; the
 * context stays usable.  Returns MOE_OK when the kernel was launched. */
MOE_API moe_status moe_selftest_bounded_wait(uint32_t limit_us, void* stream);

/* Number of CUDA kernels this library has launched in this process (all
 * devices, all streams); a tracing aid, e.g. to count the kernels of one
 * step.  Host-side counter, no synchronisation. */
MOE_API uint64_t moe_kernel_launch_count(void);

/* Static description of a status code. */
MOE_API const char* moe_status_string(moe_status s);

/* ABI version of this header (major * 100 + minor). */
MOE_API int moe_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_GATE_H */
