/*
 * Reference oracle for the fine-grained MoE layer forward.  TEST
 * INFRASTRUCTURE ONLY: the tests, the package's smoke check and the bench's
 * CPU-baseline leg may call it; the product path never does.
 *
 * Plain, slow, obviously correct C.  Dot products accumulate in double over the
 * exact input values (bf16 inputs are widened losslessly).  The router's fp32
 * quantities (affinity, biased score, weights, load, bias) are rounded to fp32
 * at the points the method defines them, so that integer decisions (top-k,
 * counts, signs) are taken in fp32, the precision of the GPU path.
 *
 * It shares no code, header or constant with the CUDA library.
 *
 * Sources (web pages on DeepSeek-V3, cited by title and section):
 *   [P1] "DeepSeek V3 From Scratch": "The idea", "Worked example", "In code"
 *        (the route() and update_bias() sketches).
 *   [P2] "Scaling Efficiency: A Deep Dive into the DeepSeek-V3 Architecture":
 *        the DeepSeekMoE module sketch (shared + routed experts, weighted
 *        combine loop).
 *   [P3] kbwen.com DeepSeek tag page: "A bias term for each expert".
 *
 * Parity pins: every function below is pinned by the CPU tests against
 * brute force, closed forms, invariants the pages state, or library
 * routines on special cases -- except the general layer output for
 * arbitrary shapes, which the pages pin only through its formula and the
 * special cases (E = k = 1, W2 = 0, k = E).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_BF16 1

/* ---- element access ---------------------------------------------------- */

static double bf16_bits_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a float to bf16, round-to-nearest-even (NaN kept quiet). */
static uint16_t float_to_bf16_bits(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

static double load_elem(const void* base, int dtype, size_t i) {
    if (dtype == ORC_BF16) return bf16_bits_to_double(((const uint16_t*)base)[i]);
    return (double)((const float*)base)[i];
}

static void store_elem(void* base, int dtype, size_t i, double v) {
    float f = (float)v;
    if (dtype == ORC_BF16)
        ((uint16_t*)base)[i] = float_to_bf16_bits(f);
    else
        ((float*)base)[i] = f;
}

/* Value after the storage rounding of dtype (used for the documented bf16
 * rounding of the SwiGLU intermediate h). */
static double round_to_dtype(double v, int dtype) {
    float f = (float)v;
    if (dtype == ORC_BF16) return bf16_bits_to_double(float_to_bf16_bits(f));
    return (double)f;
}

static double dot_rows(const void* a, size_t a_off, const void* b, size_t b_off, int dtype, int n) {
    double acc = 0.0;
    for (int c = 0; c < n; ++c) acc += load_elem(a, dtype, a_off + c) * load_elem(b, dtype, b_off + c);
    return acc;
}

/* ---- router ------------------------------------------------------------ */

/* Gate affinities [P1 "In code", route: sigmoid(x @ gate_w.T)].
 * s[t][i] = fl32( 1 / (1 + exp(-sum_c x[t][c] * W_g[i][c])) ), the sum and the
 * sigmoid in double.  x is [T][d], W_g is [E][d], both row-major in dtype. */
void orc_affinity(const void* x, const void* w_gate, int dtype, int T, int d, int E, float* s_out) {
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < E; ++i) {
            double z = dot_rows(x, (size_t)t * d, w_gate, (size_t)i * d, dtype, d);
            s_out[(size_t)t * E + i] = (float)(1.0 / (1.0 + exp(-z)));
        }
    }
}

/* Bias-shifted top-k and unbiased, renormalised weights
 * [P1 "In code", route; P1 "The idea"; P3 "A bias term for each expert"].
 *
 * v_i = fl32(s_i + b_i).  Selection by rank counting:
 *   rank_i = #{ j : v_j > v_i  or  (v_j == v_i and j < i) }
 * expert i is chosen iff rank_i < k, and it occupies slot rank_i, so slots are
 * ordered by descending v with ties going to the lower expert index.
 * Weights use the UNBIASED s: den = fl32 sum of s over slots 0..k-1 in slot
 * order, w_j = fl32(s_idx_j / den).
 * Returns 0, or -1 if a row does not fill k slots (NaN scores). */
int orc_select(const float* s, const float* bias, int T, int E, int k, int32_t* idx, float* w) {
    int bad = 0;
    #pragma omp parallel for schedule(static) reduction(| : bad)
    for (int t = 0; t < T; ++t) {
        const float* st = s + (size_t)t * E;
        float* v = (float*)malloc(sizeof(float) * (size_t)E);
        for (int i = 0; i < E; ++i) {
            volatile float vi = st[i] + bias[i]; /* one fp32 add, no contraction */
            v[i] = vi;
        }
        int filled = 0;
        for (int i = 0; i < E; ++i) {
            int rank = 0;
            for (int j = 0; j < E; ++j)
                if (v[j] > v[i] || (v[j] == v[i] && j < i)) ++rank;
            if (rank < k && v[i] == v[i]) {
                idx[(size_t)t * k + rank] = i;
                ++filled;
            }
        }
        free(v);
        if (filled != k) { bad = 1; continue; }
        float den = 0.0f;
        for (int j = 0; j < k; ++j) {
            volatile float nd = den + st[idx[(size_t)t * k + j]];
            den = nd;
        }
        for (int j = 0; j < k; ++j) {
            volatile float q = st[idx[(size_t)t * k + j]] / den;
            w[(size_t)t * k + j] = q;
        }
    }
    return bad ? -1 : 0;
}

/* Per-expert load histogram over the whole batch of the step
 * [P1 "In code", update_bias comment "load: fraction of tokens per expert";
 *  P3 "A bias term for each expert"].  c_i = #{(t, j) : idx[t][j] = i}.
 * Returns -1 if an index is out of range. */
int orc_histogram(const int32_t* idx, int T, int k, int E, int32_t* counts) {
    for (int i = 0; i < E; ++i) counts[i] = 0;
    for (size_t a = 0; a < (size_t)T * k; ++a) {
        int e = idx[a];
        if (e < 0 || e >= E) return -1;
        counts[e] += 1;
    }
    return 0;
}

/* Auxiliary-loss-free bias update, applied once at the end of the step
 * [P1 "In code", update_bias: bias + step * sign(target - load);
 *  P3 "A bias term for each expert": fixed amount, down for overloaded,
 *  up for underloaded].
 * load_i = fl32(c_i / T), target_i = target ? target[i] : fl32(k / E),
 * delta_i = sign(fl32(target_i - load_i)) in {-1, 0, +1},
 * b_i = fl32(b_i + delta_i * fl32(step)).  load_out may be NULL. */
void orc_bias_update(const int32_t* counts, int T, int E, int k, float step, const float* target,
                     float* bias, float* load_out) {
    for (int i = 0; i < E; ++i) {
        volatile float load = (float)counts[i] / (float)T;
        volatile float tgt = target ? target[i] : (float)k / (float)E;
        volatile float diff = tgt - load;
        float sgn = diff > 0.0f ? 1.0f : (diff < 0.0f ? -1.0f : 0.0f);
        volatile float nb = bias[i] + sgn * step;
        bias[i] = nb;
        if (load_out) load_out[i] = load;
    }
}

/* ---- permutation ------------------------------------------------------- */

/* Expert-contiguous order ["Tokens routed to the same expert can be batched
 * together", locionic.com DeepSeek V3 Architecture Deep Dive, "Throughput on
 * NVIDIA H100/H800"].  Rows are ordered by (expert ascending, token
 * ascending); offsets[e] = first row of expert e, offsets[E] = T*k;
 * perm_tok[row] = t*k + j (the assignment held by that row);
 * inv_row[t*k + j] = row.  Returns -1 on an out-of-range index. */
int orc_permute(const int32_t* idx, int T, int k, int E, int32_t* offsets, int32_t* perm_tok, int32_t* inv_row) {
    int32_t* counts = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    if (orc_histogram(idx, T, k, E, counts) != 0) { free(counts); return -1; }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            int row = cursor[e]++;
            perm_tok[row] = t * k + j;
            inv_row[(size_t)t * k + j] = row;
        }
    }
    free(cursor);
    free(counts);
    return 0;
}

/* ---- experts and combine ----------------------------------------------- */

/* One SwiGLU expert applied to n token rows, accumulated into a double buffer
 * [P2 DeepSeekMoE sketch: routed_out[mask] += w * expert(x[mask]); the expert
 *  MLP is SwiGLU without biases]:
 *   a = W1 x,  g = W3 x            (W1, W3: [I][d], row-major, dtype)
 *   h = round_dtype( a / (1 + exp(-a)) * g )   (h stored in dtype once)
 *   o = W2 h                       (W2: [d][I], row-major, dtype)
 *   yacc[dest[r]][:] += wts[r] * o
 * x_rows is [n][d] in dtype.  W2 may be addressed with a row stride (ld2)
 * and W1/W3 likewise (ld1) so a shared expert of a stacked tensor can be
 * passed without copying. */
void orc_expert_accumulate(const void* x_rows, int n, const int32_t* dest, const double* wts,
                           const void* w1, const void* w3, const void* w2, int d, int I, int dtype,
                           double* yacc) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < n; ++r) {
        double* h = (double*)malloc(sizeof(double) * (size_t)I);
        for (int c = 0; c < I; ++c) {
            double a = dot_rows(w1, (size_t)c * d, x_rows, (size_t)r * d, dtype, d);
            double g = dot_rows(w3, (size_t)c * d, x_rows, (size_t)r * d, dtype, d);
            double silu = a / (1.0 + exp(-a));
            h[c] = round_to_dtype(silu * g, dtype);
        }
        double* yr = yacc + (size_t)dest[r] * d;
        for (int o = 0; o < d; ++o) {
            double acc = 0.0;
            for (int c = 0; c < I; ++c) acc += load_elem(w2, dtype, (size_t)o * I + c) * h[c];
            /* rows of one call never share a destination (one expert per
             * token), so the update is race-free */
            yr[o] += wts[r] * acc;
        }
        free(h);
    }
}

/* The two halves of one expert's SwiGLU MLP, for checking the grouped GEMMs
 * one projection at a time [P2 DeepSeekMoE sketch: each expert an MLP over
 * the tokens routed to it; SwiGLU without biases].  The arithmetic is that of
 * orc_expert_accumulate, split at h.
 * orc_expert_up:   h[r][c] = round_dtype( silu(a) * g ),
 *                  a = sum_i W1[c][i] x[r][i], g = sum_i W3[c][i] x[r][i] (double)
 *                  x_rows [n][d], W1/W3 [I][d], h [n][I] in dtype.
 * orc_expert_down: o[r][j] = sum_c W2[j][c] h[r][c]  (double, not rounded)
 *                  h_rows [n][K], W2 [d][K] in dtype, o [n][d] double. */
void orc_expert_up(const void* x_rows, int n, const void* w1, const void* w3, int d, int I, int dtype, void* h_out) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int c = 0; c < I; ++c) {
        for (int r = 0; r < n; ++r) {
            double a = dot_rows(w1, (size_t)c * d, x_rows, (size_t)r * d, dtype, d);
            double g = dot_rows(w3, (size_t)c * d, x_rows, (size_t)r * d, dtype, d);
            store_elem(h_out, dtype, (size_t)r * I + c, round_to_dtype(a / (1.0 + exp(-a)) * g, dtype));
        }
    }
}

void orc_expert_down(const void* h_rows, int n, const void* w2, int d, int K, int dtype, double* o_out) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int j = 0; j < d; ++j)
        for (int r = 0; r < n; ++r) o_out[(size_t)r * d + j] = dot_rows(w2, (size_t)j * K, h_rows, (size_t)r * K, dtype, K);
}

/* Round the double accumulator to the output dtype once
 * [P2 DeepSeekMoE sketch: shared_out + routed_out]. */
void orc_finalize(const double* yacc, size_t n, int dtype, void* y_out) {
    for (size_t i = 0; i < n; ++i) store_elem(y_out, dtype, i, yacc[i]);
}

/* Whole layer for small cases, in the order of the pages' forward:
 * shared expert(s) on every token, then for each routed expert e the tokens
 * routed to it, weighted by the unbiased weight of that slot.
 * idx/w are the routing decisions (from orc_select, or injected).
 * Natural layouts: W1, W3 [E][I][d]; W2 [E][d][I]; Ws1, Ws3 [S][Is][d];
 * Ws2 [S][d][Is].  y is [T][d] in dtype. */
void orc_layer_output(const void* x, const int32_t* idx, const float* w, const void* w1, const void* w3,
                      const void* w2, const void* ws1, const void* ws3, const void* ws2, int T, int d, int E,
                      int k, int I, int S, int Is, int dtype, void* y) {
    size_t esz = dtype == ORC_BF16 ? 2 : 4;
    double* yacc = (double*)calloc((size_t)T * d, sizeof(double));
    int32_t* dest = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
    double* wts = (double*)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    char* rows = (char*)malloc(esz * (size_t)(T > 0 ? T : 1) * d);
    /* shared experts: weight 1 on every token */
    for (int s = 0; s < S; ++s) {
        for (int t = 0; t < T; ++t) { dest[t] = t; wts[t] = 1.0; }
        orc_expert_accumulate(x, T, dest, wts, (const char*)ws1 + esz * (size_t)s * Is * d,
                              (const char*)ws3 + esz * (size_t)s * Is * d, (const char*)ws2 + esz * (size_t)s * d * Is,
                              d, Is, dtype, yacc);
    }
    /* routed experts: the tokens whose top-k holds e */
    for (int e = 0; e < E; ++e) {
        int n = 0;
        for (int t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j)
                if (idx[(size_t)t * k + j] == e) {
                    memcpy(rows + esz * (size_t)n * d, (const char*)x + esz * (size_t)t * d, esz * (size_t)d);
                    dest[n] = t;
                    wts[n] = (double)w[(size_t)t * k + j];
                    ++n;
                }
        if (n == 0) continue;
        orc_expert_accumulate(rows, n, dest, wts, (const char*)w1 + esz * (size_t)e * I * d,
                              (const char*)w3 + esz * (size_t)e * I * d, (const char*)w2 + esz * (size_t)e * d * I, d, I,
                              dtype, yacc);
    }
    orc_finalize(yacc, (size_t)T * d, dtype, y);
    free(rows);
    free(wts);
    free(dest);
    free(yacc);
}

/* ---- E4M3 codec ----------------------------------------------------------
 * [P4] "DeepSeek V3 Architecture Deep Dive ...", "FP8 Formats": E4M3 (4
 * exponent, 3 mantissa bits) for weights and activations.  Values, from the
 * format's definition (the "fn" variant with no infinities): exponent bias
 * 7; field e in 1..15 gives (1 + m/8) * 2^(e-7), e = 0 gives subnormals
 * (m/8) * 2^-6; S.1111.111 is NaN; the largest finite magnitude is
 * 1.75 * 2^8 = 448. */

double orc_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7) return NAN;
    double v = e == 0 ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* Nearest E4M3 value, ties to the even mantissa; magnitudes at or above 448
 * give +-448 (saturating conversion).  Exact: every step is a multiplication
 * by a power of two or an integer rounding in double. */
uint8_t orc_e4m3_encode(float x) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;
    int e;
    frexp(a, &e);            /* a = f * 2^e with f in [0.5, 1): the binade is 2^(e-1) */
    int be = e - 1;
    if (be < -6) be = -6;    /* below 2^-6 the grid is the subnormal one, step 2^-9 */
    double step = ldexp(1.0, be - 3);
    double n = a / step;
    double r = floor(n);
    double frac = n - r;
    if (frac > 0.5 || (frac == 0.5 && fmod(r, 2.0) != 0.0)) r += 1.0;
    double v = r * step;
    if (v >= 448.0) return sign | 0x7E;
    if (v == 0.0) return sign;
    int e2;
    frexp(v, &e2);
    int vbe = e2 - 1;
    if (vbe < -6) return sign | (uint8_t)(v / ldexp(1.0, -9));              /* subnormal: m * 2^-9 */
    int m = (int)((v / ldexp(1.0, vbe) - 1.0) * 8.0);
    return sign | (uint8_t)(((vbe + 7) << 3) | m);
}

/* The 256 code values, from orc_e4m3_decode, for the expert sums below. */
static double e4m3_table[256];
static int e4m3_table_ready = 0;
static const double* e4m3_values(void) {
    if (!e4m3_table_ready) {
        #pragma omp critical(e4m3_table)
        {
            if (!e4m3_table_ready) {
                for (int c = 0; c < 256; ++c) e4m3_table[c] = orc_e4m3_decode((uint8_t)c);
                e4m3_table_ready = 1;
            }
        }
    }
    return e4m3_table;
}

void orc_e4m3_encode_array(const float* x, size_t n, uint8_t* q) {
    for (size_t i = 0; i < n; ++i) q[i] = orc_e4m3_encode(x[i]);
}
void orc_e4m3_decode_array(const uint8_t* q, size_t n, double* x) {
    for (size_t i = 0; i < n; ++i) x[i] = orc_e4m3_decode(q[i]);
}

/* Element (r, c) of a matrix with `rows` rows stored as nseg column blocks of
 * kseg columns each ([nseg][rows][kseg], the layout of stacked experts whose
 * blocks are joined along the contraction); nseg = 1 is plain row major. */
static size_t seg_index(long r, int c, long rows, int kseg) {
    return (size_t)(c / kseg) * (size_t)rows * kseg + (size_t)r * kseg + (size_t)(c % kseg);
}

/* ---- FP8 (E4M3) experts with per-tile scaling ----------------------------
 * [P1 "The idea": FP8 mixed precision with fine-grained quantization tiles;
 *  P5 "How It Works": FP8 training with per-tile scaling; P4 "FP8 Formats":
 *  E4M3 for weights and activations.]  The pages fix neither the tile nor
 * the scale arithmetic.  Read here as: a tile is 32 consecutive elements of
 * one row along the contraction dimension (weights: along the input features
 * of each output row; activations: along the features of each token row),
 * and its scale is a power of two, 2^e with e the smallest integer such that
 * the tile's largest magnitude fits the E4M3 range (amax <= 448 * 2^e), so no
 * element saturates.  Codes are E4M3(v * 2^-e).  The scale of a tile is kept
 * as its exponent byte e + 127.  A dot product then sums, tile by tile,
 * 2^(e_a + e_b) * sum_{i in tile} dec(qa_i) dec(qb_i). */

#define ORC_MX_TILE 32

/* Smallest e in [-127, 127] with amax <= 448 * 2^e (0 for an all-zero tile;
 * -127 for tiles whose amax is below 448 * 2^-127). */
int orc_mx_exponent(double amax) {
    if (!(amax > 0.0)) return 0;
    int e = -127;
    while (e < 127 && amax > ldexp(448.0, e)) ++e;
    return e;
}

/* Tile quantization of a matrix with `rows` rows of K = nseg * kseg columns,
 * stored as [nseg][rows][kseg] (nseg = 1: plain row major); kseg % 32 == 0.
 * q has src's layout; ebyte [rows][K / 32] holds e + 127 of tile b of row r
 * at r * (K / 32) + b, tiles numbered along the whole row. */
void orc_quantize_mx(const void* src, int dtype, long rows, int kseg, int nseg, uint8_t* q, uint8_t* ebyte) {
    int K = kseg * nseg, nb = K / ORC_MX_TILE;
    #pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; ++r) {
        for (int b = 0; b < nb; ++b) {
            double amax = 0.0;
            for (int c = b * ORC_MX_TILE; c < (b + 1) * ORC_MX_TILE; ++c) {
                double v = fabs(load_elem(src, dtype, seg_index(r, c, rows, kseg)));
                if (v > amax) amax = v;
            }
            int e = orc_mx_exponent(amax);
            ebyte[(size_t)r * nb + b] = (uint8_t)(e + 127);
            for (int c = b * ORC_MX_TILE; c < (b + 1) * ORC_MX_TILE; ++c) {
                size_t i = seg_index(r, c, rows, kseg);
                q[i] = orc_e4m3_encode((float)(load_elem(src, dtype, i) * ldexp(1.0, -e)));
            }
        }
    }
}

/* sum over the K/32 tiles of 2^(ea + eb) * sum_i dec(qa_i) dec(qb_i), in
 * double; a and b are rows of K codes whose tile exponent bytes are ea, eb. */
static double mx_dot(const uint8_t* qa, const uint8_t* ea, const uint8_t* qb, const uint8_t* eb, int K,
                     size_t (*bidx)(const void*, int), const void* bctx) {
    const double* val = e4m3_values();
    double acc = 0.0;
    for (int b = 0; b < K / ORC_MX_TILE; ++b) {
        double s = 0.0;
        for (int i = b * ORC_MX_TILE; i < (b + 1) * ORC_MX_TILE; ++i)
            s += val[qa[i]] * val[qb[bidx ? bidx(bctx, i) : (size_t)i]];
        acc += ldexp(s, ((int)ea[b] - 127) + ((int)eb[b] - 127));
    }
    return acc;
}

/* Gate/up of one FP8 expert on n token rows quantized by tiles:
 *   a[r][c] = mx_dot(xq[r], W1q[c]),  g[r][c] = mx_dot(xq[r], W3q[c])  (double)
 *   h[r][c] = bf16(silu(a) * g)
 * xq [n][d] with xe [n][d/32]; w1q/w3q [I][d] with w1e/w3e [I][d/32]. */
void orc_expert_up_mx(const uint8_t* xq, const uint8_t* xe, int n, const uint8_t* w1q, const uint8_t* w1e,
                      const uint8_t* w3q, const uint8_t* w3e, int d, int I, uint16_t* h) {
    int nb = d / ORC_MX_TILE;
    #pragma omp parallel for schedule(dynamic, 4)
    for (int c = 0; c < I; ++c) {
        for (int r = 0; r < n; ++r) {
            const uint8_t* xr = xq + (size_t)r * d;
            const uint8_t* xer = xe + (size_t)r * nb;
            double a = mx_dot(xr, xer, w1q + (size_t)c * d, w1e + (size_t)c * nb, d, NULL, NULL);
            double g = mx_dot(xr, xer, w3q + (size_t)c * d, w3e + (size_t)c * nb, d, NULL, NULL);
            h[(size_t)r * I + c] = float_to_bf16_bits((float)(a / (1.0 + exp(-a)) * g));
        }
    }
}

/* Down projection of one FP8 expert on n rows of h quantized by tiles:
 *   o[r][j] = mx_dot(hq[r], W2q(j, .))  (double)
 * hq [n][K] with he [n][K/32]; W2q is [d][K] stored as nseg blocks of kseg
 * columns ([nseg][d][kseg], K = nseg * kseg) with w2e [d][K/32] (tiles
 * numbered along the whole row, as orc_quantize_mx gives them). */
struct mx_seg_ctx { long rows; int kseg; long j; };
static size_t mx_seg_col(const void* ctx, int c) {
    const struct mx_seg_ctx* s = (const struct mx_seg_ctx*)ctx;
    return seg_index(s->j, c, s->rows, s->kseg);
}
void orc_expert_down_mx(const uint8_t* hq, const uint8_t* he, int n, const uint8_t* w2q, const uint8_t* w2e, int d,
                        int kseg, int nseg, double* o) {
    int K = kseg * nseg, nb = K / ORC_MX_TILE;
    #pragma omp parallel for schedule(dynamic, 4)
    for (int j = 0; j < d; ++j) {
        struct mx_seg_ctx ctx = {d, kseg, j};
        for (int r = 0; r < n; ++r)
            o[(size_t)r * d + j] = mx_dot(hq + (size_t)r * K, he + (size_t)r * nb, w2q, w2e + (size_t)j * nb, K,
                                          mx_seg_col, &ctx);
    }
}
