// Backward of the MoE layer forward: gradients of <dy, y> (+ the sequence-wise
// balance loss) with respect to x, the gate weights and the routed and shared
// expert weights, for the selection the forward made.
//
// What is differentiated (page title, section):
//   "DeepSeek V3 From Scratch", "In code" (route): s = sigmoid(x W_g^T); the
//     top-k is chosen on s + b; w_j = s_{idx_j} / sum_j' s_{idx_j'} from the
//     unbiased scores.  The bias and the choice carry no gradient.
//   "Scaling Efficiency: A Deep Dive into the DeepSeek-V3 Architecture",
//     DeepSeekMoE sketch: y_t = sum_s shared_s(x_t) + sum_j w_j expert_{idx_j}(x_t),
//     every expert W2 (silu(W1 x) * (W3 x)).
//   kbwen.com DeepSeek tag page, "A bias term for each expert": a small
//     complementary sequence-wise balance loss is kept; its formula is not
//     on the pages -- the DeepSeek-V3 report's is used: per sequence of L
//     tokens, f_i = E/(kL) #{t : i chosen}, P_i = 1/L sum_t s_ti / sum_j s_tj,
//     loss = alpha sum_i f_i P_i, averaged over the sequences.
//
// Gradients (per routed assignment r = (t, j) of expert e, h recomputed and
// rounded like the forward's):
//   dw_tj = <dy_t, o_r>,  o_r = W2_e h_r;   do_r = w_tj dy_t
//   dW2_e = sum_r do_r h_r^T;   dh_r = W2_e^T do_r
//   da = dh g sigma(a) (1 + a (1 - sigma(a))),   dg = dh a sigma(a)
//   dW1_e = sum_r da_r x_t^T,  dW3_e likewise;  dx_t += W1_e^T da_r + W3_e^T dg_r
//   shared experts the same with weight 1;  router: ds_{t,idx_j} =
//   (dw_tj - sum_j' dw_tj' w_tj') / sum_j' s_{t,idx_j'} (+ the balance term),
//   dz = ds s (1 - s),  dx += dz W_g,  dW_g = dz^T x.
//
// Two paths compute these.  bf16 layers whose widths are multiples of 128 run
// every contraction on the tensor cores (gemm_bwd_tc.cu: bf16 operands, fp32
// accumulation) over a padded row layout (each expert's rows padded to a
// multiple of 64 with zero rows); there a, g and h are recomputed by one
// launch of the forward's gate/up kernel (the forward's own h, with the fp32
// a and g beside it), and the routed dw comes without recomputing o: with
// u_r = W2_e^T dy_t (the dh GEMM run on the unweighted dy),
// dw_tj = <dy_t, W2_e h_r> = <u_r, h_r> and dh_r = w_tj u_r.  Every
// other layer runs two fp32 SIMT kernels over strided operand views (no
// transposed copies): a "rows" GEMM (C[r][n] = sum_k A(r,k) B_g(n,k) for the
// rows r of group g) and a weight-gradient GEMM whose contraction runs over a
// group's rows (C_g[m][n] = sum_r A(r,m) B(r,n)); groups and tiles are
// resolved on the device from the routing offsets.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {
namespace {

constexpr int TB = 128, TK = 16;  // block tile (both output dimensions), contraction slab

// Element (r, c) of group g: base + g*gs + row(r)*rs + c*cs, where row(r) =
// gather[r] / gdiv when a gather index is given, else r.
struct Opnd {
    const void* p;
    int bf16;
    long long rs, cs, gs;
    const int32_t* gather;
    int gdiv;
};

__device__ __forceinline__ long long row_off(const Opnd& o, int r) {
    const long long row = o.gather ? (long long)(o.gather[r] / o.gdiv) : (long long)r;
    return row * o.rs;
}
__device__ __forceinline__ float ld_at(const Opnd& o, long long off) {
    if (o.bf16) return __uint_as_float((uint32_t)static_cast<const uint16_t*>(o.p)[off] << 16);
    return static_cast<const float*>(o.p)[off];
}

// Eight consecutive elements from element offset off (16-byte aligned for
// bf16, 32-byte aligned for fp32: one or two vector loads).
__device__ __forceinline__ void ld8(const Opnd& o, long long off, float (&v)[8]) {
    if (o.bf16) {
        const uint4 u = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(o.p) + off);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else {
        const float4 a = *reinterpret_cast<const float4*>(static_cast<const float*>(o.p) + off);
        const float4 b = *reinterpret_cast<const float4*>(static_cast<const float*>(o.p) + off + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
}
// A k-contiguous operand whose row and group strides keep every run of eight
// elements starting at a multiple of 8 on a 16-byte (bf16) / 32-byte (fp32)
// boundary: the rows GEMM then loads its eight k per thread with ld8.
bool vec8_ok(const void* p, int bf16, long long rs, long long cs, long long gs) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(p);
    return cs == 1 && rs % 8 == 0 && gs % 8 == 0 && (a % (bf16 ? 16u : 32u)) == 0;
}

// Rows r of group g: [offsets[g], offsets[g+1]) or, without offsets, [0, M).
// A corrupt range is skipped and reported.
__device__ __forceinline__ void group_rows(const int32_t* offsets, int g, int M, int* status, int& rs, int& re) {
    if (!offsets) {
        rs = 0;
        re = M;
        return;
    }
    rs = offsets[g];
    re = offsets[g + 1];
    if (rs < 0 || re < rs || re > M) {
        report(status, kStDeviceCheck);
        rs = re = 0;
    }
}

// acc[i][j] += As[kk][ty*8 + i] * Bs[kk][tx*8 + j] over one slab (float4 reads).
__device__ __forceinline__ void slab_fma(const float (*As)[TB + 4], const float (*Bs)[TB + 4], int ty, int tx,
                                         float (&acc)[8][8]) {
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
        const float4 a0 = *reinterpret_cast<const float4*>(&As[kk][ty * 8]);
        const float4 a1 = *reinterpret_cast<const float4*>(&As[kk][ty * 8 + 4]);
        const float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 8]);
        const float4 b1 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 8 + 4]);
        const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
}

struct RowsGemm {
    Opnd A, B;          // A(r, k) (no group), B(n, k) of group g
    float* C;           // C[r * c_rs + n]
    long long c_rs;
    int M, N, K;
    const int32_t* offsets;
    int G;
    int accumulate;
    int a_vec, b_vec;   // operand loads eight k at a time (vec8_ok)
    int* status;
};

// C[r][n] (+)= sum_k A(r, k) B_g(n, k) for every row r of every group g.
// 128 x 128 output tiles, 256 threads with 8 x 8 outputs each, K in slabs of
// 16 through shared memory; the tile's row offsets (the gather resolved) are
// computed once per tile.  Tiles of all groups in one grid-stride list.
__global__ void __launch_bounds__(256, 2) rows_gemm_kernel(RowsGemm p) {
    __shared__ __align__(16) float As[TK][TB + 4];
    __shared__ __align__(16) float Bs[TK][TB + 4];
    __shared__ long long arow[TB], brow[TB];
    __shared__ int prefix[kMaxGroups + 1];
    __shared__ int gstart[kMaxGroups], grows[kMaxGroups];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int n_tiles = (p.N + TB - 1) / TB;
    for (int g = tid; g < p.G; g += blockDim.x) {
        int rs, re;
        group_rows(p.offsets, g, p.M, p.status, rs, re);
        gstart[g] = rs;
        grows[g] = re - rs;
    }
    __syncthreads();
    if (tid == 0) {
        int acc = 0;
        for (int g = 0; g < p.G; ++g) {
            prefix[g] = acc;
            acc += (grows[g] + TB - 1) / TB * n_tiles;
        }
        prefix[p.G] = acc;
    }
    __syncthreads();
    const bool a_kfast = p.A.cs == 1, b_kfast = p.B.cs == 1;
    for (int tile = blockIdx.x; tile < prefix[p.G]; tile += gridDim.x) {
        int lo = 0, hi = p.G - 1;
        while (lo < hi) {  // last group whose first tile is <= tile
            const int mid = (lo + hi + 1) >> 1;
            if (prefix[mid] <= tile) lo = mid; else hi = mid - 1;
        }
        const int g = lo;
        const int mt = (grows[g] + TB - 1) / TB;
        const int q = tile - prefix[g];
        const int m0 = (q % mt) * TB, n0 = (q / mt) * TB;
        const int row0 = gstart[g] + m0;
        const int nrows = min(TB, grows[g] - m0);
        __syncthreads();  // the previous tile's readers of arow / brow are done
        if (tid < TB) {
            arow[tid] = tid < nrows ? row_off(p.A, row0 + tid) : -1;
        } else {
            const int n = tid - TB;
            brow[n] = n0 + n < p.N ? (long long)g * p.B.gs + (long long)(n0 + n) * p.B.rs : -1;
        }
        __syncthreads();
        // each thread loads one row of each operand per slab: 8 consecutive k
        // (k contiguous in memory) or every other k (rows contiguous)
        const int am = a_kfast ? tid >> 1 : tid & (TB - 1), bn = b_kfast ? tid >> 1 : tid & (TB - 1);
        const long long ra = arow[am], rb = brow[bn];
        float acc[8][8] = {};
#pragma unroll 1
        for (int k0 = 0; k0 < p.K; k0 += TK) {
            const int kh = k0 + (tid & 1) * 8;  // first of this thread's eight k (k-contiguous operands)
            if (p.a_vec && ra >= 0 && kh + 8 <= p.K) {
                float v[8];
                ld8(p.A, ra + kh, v);
#pragma unroll
                for (int i = 0; i < 8; ++i) As[(tid & 1) * 8 + i][am] = v[i];
            } else {
#pragma unroll 1
                for (int i = 0; i < 8; ++i) {
                    const int ka = a_kfast ? (tid & 1) * 8 + i : (tid >> 7) + 2 * i;
                    As[ka][am] = (ra >= 0 && k0 + ka < p.K) ? ld_at(p.A, ra + (long long)(k0 + ka) * p.A.cs) : 0.0f;
                }
            }
            if (p.b_vec && rb >= 0 && kh + 8 <= p.K) {
                float v[8];
                ld8(p.B, rb + kh, v);
#pragma unroll
                for (int i = 0; i < 8; ++i) Bs[(tid & 1) * 8 + i][bn] = v[i];
            } else {
#pragma unroll 1
                for (int i = 0; i < 8; ++i) {
                    const int kb = b_kfast ? (tid & 1) * 8 + i : (tid >> 7) + 2 * i;
                    Bs[kb][bn] = (rb >= 0 && k0 + kb < p.K) ? ld_at(p.B, rb + (long long)(k0 + kb) * p.B.cs) : 0.0f;
                }
            }
            __syncthreads();
            slab_fma(As, Bs, ty, tx, acc);
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int m = ty * 8 + i;
            if (m >= nrows) continue;
            float* crow = p.C + (long long)(row0 + m) * p.c_rs;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int n = n0 + tx * 8 + j;
                if (n < p.N) crow[n] = p.accumulate ? crow[n] + acc[i][j] : acc[i][j];
            }
        }
    }
}

struct WgradGemm {
    Opnd A, B;          // A(r, m), B(r, n) over the group's rows r
    float* C;           // C_g[m][n] at C + g * c_gs + m * c_rs + n
    long long c_rs, c_gs;
    int M, N;
    const int32_t* offsets;
    int G;
    int rows;           // rows of the single group without offsets
    int accumulate;
    int* status;
};

// C_g[m][n] (+)= sum over the rows r of group g of A(r, m) B(r, n).  Grid:
// x = 128 x 128 output tiles of one group, y = group; the slab's 16 row
// offsets of each operand are resolved once per slab.  An empty group writes
// zeros.
__global__ void __launch_bounds__(256, 2) wgrad_gemm_kernel(WgradGemm p) {
    __shared__ __align__(16) float As[TK][TB + 4];
    __shared__ __align__(16) float Bs[TK][TB + 4];
    __shared__ long long arow[TK], brow[TK];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int g = blockIdx.y;
    const int m_tiles = (p.M + TB - 1) / TB;
    const int m0 = (blockIdx.x % m_tiles) * TB, n0 = (blockIdx.x / m_tiles) * TB;
    int rs, re;
    group_rows(p.offsets, g, p.rows, p.status, rs, re);
    const bool a_mfast = p.A.cs == 1, b_nfast = p.B.cs == 1;
    float acc[8][8] = {};
    for (int r0 = rs; r0 < re; r0 += TK) {
        if (tid < TK) {
            arow[tid] = r0 + tid < re ? row_off(p.A, r0 + tid) : -1;
        } else if (tid < 2 * TK) {
            brow[tid - TK] = r0 + tid - TK < re ? row_off(p.B, r0 + tid - TK) : -1;
        }
        __syncthreads();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = tid + 256 * i;
            const int m = a_mfast ? e % TB : e / TK, kk = a_mfast ? e / TB : e % TK;
            const long long ra = arow[kk];
            As[kk][m] = (ra >= 0 && m0 + m < p.M) ? ld_at(p.A, ra + (long long)(m0 + m) * p.A.cs) : 0.0f;
            const int n = b_nfast ? e % TB : e / TK, kb = b_nfast ? e / TB : e % TK;
            const long long rb = brow[kb];
            Bs[kb][n] = (rb >= 0 && n0 + n < p.N) ? ld_at(p.B, rb + (long long)(n0 + n) * p.B.cs) : 0.0f;
        }
        __syncthreads();
        slab_fma(As, Bs, ty, tx, acc);
        __syncthreads();
    }
    float* cg = p.C + (long long)g * p.c_gs;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int m = m0 + ty * 8 + i;
        if (m >= p.M) continue;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int n = n0 + tx * 8 + j;
            if (n < p.N) {
                float* c = cg + (long long)m * p.c_rs + n;
                *c = p.accumulate ? *c + acc[i][j] : acc[i][j];
            }
        }
    }
}

__device__ __forceinline__ float sigmoid_acc(float a) { return 1.0f / (1.0f + expf(-a)); }

// h = silu(a) * g, rounded to bf16 when the layer is bf16 (the forward's rounding point).
__global__ void swiglu_fwd_kernel(const float* __restrict__ a, const float* __restrict__ g, float* __restrict__ h,
                                  long long n, int bf16) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const float av = a[i];
        float v = av * sigmoid_acc(av) * g[i];
        if (bf16) v = __bfloat162float(__float2bfloat16_rn(v));
        h[i] = v;
    }
}

// In place: dh_da <- dh g s (1 + a (1 - s)),  g_dg <- dh a s,  s = sigmoid(a).
__global__ void swiglu_bwd_kernel(const float* __restrict__ a, float* __restrict__ g_dg, float* __restrict__ dh_da,
                                  long long n) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
        const float av = a[i], gv = g_dg[i], dh = dh_da[i];
        const float s = sigmoid_acc(av);
        dh_da[i] = dh * gv * s * (1.0f + av * (1.0f - s));
        g_dg[i] = dh * av * s;
    }
}

// Fixed-order block sum (warp shuffles, then warp 0 over the warp partials).
__device__ float block_sum(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[w] = v;
    __syncthreads();
    if (w == 0) {
        v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    const float r = red[0];
    __syncthreads();
    return r;
}

// One block per assignment q = t*k + j, row r = inv[q] of the permuted
// buffers: dw[q] = <dy_t, o_r>, then o_r <- do_r = w[q] dy_t (in place).
__global__ void __launch_bounds__(256) combine_bwd_kernel(const float* __restrict__ dy, const float* __restrict__ w,
                                                          const int32_t* __restrict__ inv, float* o_do,
                                                          float* __restrict__ dw, int d, int k, int rows,
                                                          int* status) {
    __shared__ float red[32];
    const int q = blockIdx.x, t = q / k;
    const int r = inv[q];
    if (r < 0 || r >= rows) {
        if (threadIdx.x == 0) report(status, kStDeviceCheck);
        return;
    }
    const float* dyt = dy + (long long)t * d;
    float* orow = o_do + (long long)r * d;
    float part = 0.0f;
    for (int c = threadIdx.x; c < d; c += blockDim.x) part = fmaf(dyt[c], orow[c], part);
    const float tot = block_sum(part, red);  // every read of the row is done past this point
    if (threadIdx.x == 0) dw[q] = tot;
    const float wq = w[q];
    for (int c = threadIdx.x; c < d; c += blockDim.x) orow[c] = wq * dyt[c];
}

// dx[t] = sum_j dxp[inv[t*k + j]] (overwrite), one block per token.
__global__ void unpermute_sum_kernel(const float* __restrict__ dxp, const int32_t* __restrict__ inv, float* dx, int d,
                                     int k, int rows, int* status) {
    const int t = blockIdx.x;
    for (int c = threadIdx.x; c < d; c += blockDim.x) {
        float v = 0.0f;
        for (int j = 0; j < k; ++j) {
            const int r = inv[(long long)t * k + j];
            if (r < 0 || r >= rows) {
                report(status, kStDeviceCheck);
                continue;
            }
            v += dxp[(long long)r * d + c];
        }
        dx[(long long)t * d + c] = v;
    }
}

// Per-sequence choice counts: cnt[b][i] = #{(t in sequence b, j) : idx[t][j] = i}.
__global__ void seq_counts_kernel(const int32_t* __restrict__ idx, int T, int k, int E, int L, int32_t* cnt,
                                  int* status) {
    for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < (long long)T * k;
         q += (long long)gridDim.x * blockDim.x) {
        const int e = idx[q];
        if (e < 0 || e >= E) {
            report(status, kStDeviceCheck);
            continue;
        }
        atomicAdd(&cnt[(q / k) / L * E + e], 1);
    }
}

// One warp per token: ds over all experts (the renormalised gate's part on
// the chosen ones, plus the balance term), dz = ds s (1 - s); tot[t] = sum_i s_ti.
__global__ void router_bwd_kernel(const float* __restrict__ s, const int32_t* __restrict__ idx,
                                  const float* __restrict__ dw, const int32_t* __restrict__ cnt, float alpha, int L,
                                  int nb, int T, int E, int k, float* __restrict__ dz, float* __restrict__ tot,
                                  int* status) {
    const int warps = blockDim.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * warps + (threadIdx.x >> 5);
    if (t >= T) return;
    const float* st = s + (long long)t * E;
    const int32_t* it = idx + (long long)t * k;
    const float* dwt = dw + (long long)t * k;
    bool bad = false;
    for (int j = 0; j < k; ++j) bad |= it[j] < 0 || it[j] >= E;
    if (bad) {  // corrupt selection: report, no gradient for this token
        if (lane == 0) report(status, kStDeviceCheck);
        for (int i = lane; i < E; i += 32) dz[(long long)t * E + i] = 0.0f;
        if (lane == 0 && tot) tot[t] = 1.0f;
        return;
    }
    float ssel = 0.0f;
    for (int j = 0; j < k; ++j) ssel += st[it[j]];
    float dot = 0.0f;  // sum_j dw_j w_j with w_j = s_{idx_j} / ssel
    for (int j = 0; j < k; ++j) dot += dwt[j] * (st[it[j]] / ssel);
    float sum_s = 0.0f, sum_fs = 0.0f;
    const float fscale = (float)E / ((float)k * (float)L);
    const int32_t* cb = cnt ? cnt + (long long)(t / L) * E : nullptr;
    if (alpha > 0.0f) {
        for (int i = lane; i < E; i += 32) {
            sum_s += st[i];
            sum_fs += fscale * (float)cb[i] * st[i];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            sum_s += __shfl_xor_sync(0xffffffffu, sum_s, o);
            sum_fs += __shfl_xor_sync(0xffffffffu, sum_fs, o);
        }
        if (lane == 0) tot[t] = sum_s;
    }
    for (int i = lane; i < E; i += 32) {
        float ds = 0.0f;
        for (int j = 0; j < k; ++j)
            if (it[j] == i) ds += (dwt[j] - dot) / ssel;
        if (alpha > 0.0f) ds += alpha / ((float)nb * (float)L) * (fscale * (float)cb[i] - sum_fs / sum_s) / sum_s;
        const float sv = st[i];
        dz[(long long)t * E + i] = ds * sv * (1.0f - sv);
    }
}

constexpr int kLossChunk = 32;  // tokens per partial sum of the balance loss

// Block (c, b): chunk[b][c][i] = sum over tokens t of chunk c of sequence b of s_ti / tot_t.  The block's
// threads form G = blockDim.x / E groups (E <= blockDim.x); group g sums the tokens t0 + g, t0 + g + G, ...
// of the chunk, and the G partial sums are added in group order (deterministic for a given block size).
__global__ void balance_chunk_kernel(const float* __restrict__ s, const float* __restrict__ tot, int L, int E,
                                     int C, float* __restrict__ chunk) {
    extern __shared__ float gpart[];  // [G][E]
    const int b = blockIdx.y, c = blockIdx.x;
    const int t0 = b * L + c * kLossChunk, t1 = min((b + 1) * L, t0 + kLossChunk);
    const int G = blockDim.x / E;
    const int g = threadIdx.x / E, i = threadIdx.x - g * E;
    if (g < G) {
        float P = 0.0f;
        for (int t = t0 + g; t < t1; t += G) P += s[(long long)t * E + i] / tot[t];
        gpart[g * E + i] = P;
    }
    __syncthreads();
    if (threadIdx.x < E) {
        float P = 0.0f;
        for (int q = 0; q < G; ++q) P += gpart[q * E + threadIdx.x];
        chunk[((long long)b * C + c) * E + threadIdx.x] = P;
    }
}

// One block per sequence b: part[b] = alpha * sum_i f_bi P_bi, the chunks summed in order: G = blockDim.x / E
// groups each add a contiguous run of chunks, then the runs are added in order.
__global__ void balance_part_kernel(const float* __restrict__ chunk, const int32_t* __restrict__ cnt, float alpha,
                                    int L, int E, int k, int C, float* __restrict__ part) {
    extern __shared__ float gpart[];  // [G][E]
    __shared__ float red[32];
    const int b = blockIdx.x;
    const float fscale = (float)E / ((float)k * (float)L);
    const int G = blockDim.x / E;
    const int g = threadIdx.x / E, i = threadIdx.x - g * E;
    if (g < G) {
        const int c0 = g * C / G, c1 = (g + 1) * C / G;
        float P = 0.0f;
        for (int c = c0; c < c1; ++c) P += chunk[((long long)b * C + c) * E + i];
        gpart[g * E + i] = P;
    }
    __syncthreads();
    float v = 0.0f;
    if (threadIdx.x < E) {
        float P = 0.0f;
        for (int q = 0; q < G; ++q) P += gpart[q * E + threadIdx.x];
        v = fscale * (float)cnt[(long long)b * E + threadIdx.x] * (P / (float)L);
    }
    v = block_sum(v, red);
    if (threadIdx.x == 0) part[b] = alpha * v;
}

__global__ void balance_sum_kernel(const float* __restrict__ part, int nb, float* loss) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    float v = 0.0f;
    for (int b = 0; b < nb; ++b) v += part[b];
    *loss = v / (float)nb;
}

// ------------------------------------------------------------------ tensor-core path (bf16 layers)
//
// The routed rows live in a padded layout for the tensor-core GEMMs: expert
// e's rows start at pstart[e] = sum_{e' < e} ceil64(counts[e']), so the
// weight-gradient GEMMs can run their contraction over whole 64-row stages
// of zeros past each expert's rows.  prow[r] maps a permuted row to its
// padded row.

constexpr int kPad = 64;

// One block: pstart[e] (exclusive scan of the rounded-up counts), pstart[E] = total.
__global__ void pad_plan_kernel(const int32_t* __restrict__ counts, int E, int32_t* __restrict__ pstart, int* status) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int acc = 0;
    for (int e = 0; e < E; ++e) {
        pstart[e] = acc;
        int c = counts[e];
        if (c < 0) {
            report(status, kStDeviceCheck);
            c = 0;
        }
        acc += (c + kPad - 1) / kPad * kPad;
    }
    pstart[E] = acc;
}

// Zero the padding rows of group g (rows [pstart[g] + count, pstart[g + 1]))
// in every padded operand the weight-gradient contractions run over: the
// real rows are all written by their producers, so only these need clearing.
// One block per group; each matrix's rows are whole 16-byte vectors.
struct PadZero {
    uint4* p[4];
    int vec[4];  // 16-byte vectors per row
};
__global__ void pad_zero_kernel(const int32_t* __restrict__ counts, const int32_t* __restrict__ pstart, int E,
                                PadZero z) {
    const int g = blockIdx.x;
    if (g >= E) return;
    const int c = counts[g] < 0 ? 0 : counts[g];
    const long long r0 = (long long)pstart[g] + c, r1 = pstart[g + 1];
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const long long n = (r1 - r0) * z.vec[m];
        uint4* base = z.p[m] + r0 * z.vec[m];
        for (long long i = threadIdx.x; i < n; i += blockDim.x) base[i] = zero;
    }
}

// last index i in [0, n) with a[i] <= v (a non-decreasing, a[0] <= v)
__device__ __forceinline__ int last_le(const int32_t* a, int n, int v) {
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (a[mid] <= v) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// One warp per permuted row r: prow[r] = its padded row; x_pad[prow[r]] = x[perm[r] / k] (bf16, 16-byte copies).
__global__ void gather_pad_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm,
                                  const int32_t* __restrict__ offsets, const int32_t* __restrict__ pstart, int E,
                                  int k, int R, int T, int vec, int32_t* __restrict__ prow, uint4* __restrict__ xp,
                                  int* status) {
    const int lane = threadIdx.x & 31;
    for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < R; r += gridDim.x * (blockDim.x >> 5)) {
        const int e = last_le(offsets, E, r);
        const int pr = pstart[e] + (r - offsets[e]);
        const int t = perm[r] / k;
        if (t < 0 || t >= T) {
            if (lane == 0) report(status, kStDeviceCheck);
            continue;
        }
        if (lane == 0) prow[r] = pr;
        for (int v = lane; v < vec; v += 32) xp[(size_t)pr * vec + v] = x[(size_t)t * vec + v];
    }
}

__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&b);
}

// One warp per assignment q = t*k + j (row r = inv[q], padded row pr):
// dy_pad[pr] = bf16(dy_t), do_pad[pr] = bf16(w[q] dy_t).  d % 4 == 0:
// 16-byte loads, 8-byte stores.
__global__ void __launch_bounds__(256) spread_dy_pad_kernel(const float* __restrict__ dy, const float* __restrict__ w,
                                                            const int32_t* __restrict__ inv,
                                                            const int32_t* __restrict__ prow,
                                                            uint16_t* __restrict__ dyp, uint16_t* __restrict__ dop,
                                                            int d, int k, int rows, int nq, int* status) {
    const int lane = threadIdx.x & 31;
    const int q = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (q >= nq) return;  // warp-uniform
    const int t = q / k;
    const int r = inv[q];
    if (r < 0 || r >= rows) {
        if (lane == 0) report(status, kStDeviceCheck);
        return;
    }
    const long long pr = prow[r];
    const float4* dyt = reinterpret_cast<const float4*>(dy + (long long)t * d);
    uint2* dst_y = reinterpret_cast<uint2*>(dyp + pr * d);
    uint2* dst_o = reinterpret_cast<uint2*>(dop + pr * d);
    const float wq = w[q];
    const int d4 = d / 4;
#pragma unroll 4
    for (int c = lane; c < d4; c += 32) {
        const float4 y = dyt[c];
        dst_y[c] = make_uint2(bf16x2(y.x, y.y), bf16x2(y.z, y.w));
        dst_o[c] = make_uint2(bf16x2(wq * y.x, wq * y.y), bf16x2(wq * y.z, wq * y.w));
    }
}

// Routed rows, one warp per row r (padded row pr = prow[r], assignment
// q = perm[r]), from u = dy_t W2_e (fp32, the unweighted upstream gradient
// of h): dh = w[q] u, the SwiGLU derivative as below into dadg, and the
// combine weight's gradient dw[q] = <dy_t, o> = <u, h> with h recomputed
// exactly as the forward rounds it (bf16(silu(a) g)).  n % 4 == 0.
__global__ void __launch_bounds__(256) swiglu_bwd_dw_pad_kernel(const float* __restrict__ a,
                                                                const float* __restrict__ g,
                                                                const float* __restrict__ u,
                                                                const int32_t* __restrict__ prow,
                                                                const int32_t* __restrict__ perm,
                                                                const float* __restrict__ w, int R, int n,
                                                                uint16_t* __restrict__ dadg, float* __restrict__ dw) {
    const int lane = threadIdx.x & 31;
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= R) return;  // warp-uniform
    const long long pr = prow[r];
    const int q = perm[r];
    const float wq = w[q];
    const int n4 = n / 4;
    const float4* ar = reinterpret_cast<const float4*>(a + pr * n);
    const float4* gr = reinterpret_cast<const float4*>(g + pr * n);
    const float4* ur = reinterpret_cast<const float4*>(u + pr * n);
    uint2* row = reinterpret_cast<uint2*>(dadg + pr * 2 * n);
    float dot = 0.0f;
    for (int c = lane; c < n4; c += 32) {
        const float4 av = ar[c], gv = gr[c], uv = ur[c];
        const float al[4] = {av.x, av.y, av.z, av.w}, gl[4] = {gv.x, gv.y, gv.z, gv.w},
                    ul[4] = {uv.x, uv.y, uv.z, uv.w};
        float da[4], dg[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const float s = sigmoid_acc(al[v]);
            const float h = __bfloat162float(__float2bfloat16_rn(al[v] * s * gl[v]));
            dot = fmaf(ul[v], h, dot);
            const float dh = wq * ul[v];
            da[v] = dh * gl[v] * s * (1.0f + al[v] * (1.0f - s));
            dg[v] = dh * al[v] * s;
        }
        row[c] = make_uint2(bf16x2(da[0], da[1]), bf16x2(da[2], da[3]));
        row[n4 + c] = make_uint2(bf16x2(dg[0], dg[1]), bf16x2(dg[2], dg[3]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    if (lane == 0) dw[q] = dot;
}

// SwiGLU derivative on the real rows: with s = sigmoid(a),
//   da = dh g s (1 + a (1 - s)),  dg = dh a s,
// stored bf16 side by side: dadg[pr][c] = da, dadg[pr][n + c] = dg.  Four
// columns per thread (n % 4 == 0): 16-byte loads, 8-byte stores.
__global__ void swiglu_bwd_pad_kernel(const float* __restrict__ a, const float* __restrict__ g,
                                      const float* __restrict__ dh, const int32_t* __restrict__ prow, int R, int n,
                                      uint16_t* __restrict__ dadg) {
    const int n4 = n / 4;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < (long long)R * n4;
         i += (long long)gridDim.x * blockDim.x) {
        const int r = (int)(i / n4), c = (int)(i - (long long)r * n4);
        const long long pr = prow ? prow[r] : r;
        const float4 av = reinterpret_cast<const float4*>(a + pr * n)[c];
        const float4 gv = reinterpret_cast<const float4*>(g + pr * n)[c];
        const float4 dv = reinterpret_cast<const float4*>(dh + pr * n)[c];
        const float al[4] = {av.x, av.y, av.z, av.w}, gl[4] = {gv.x, gv.y, gv.z, gv.w},
                    dl[4] = {dv.x, dv.y, dv.z, dv.w};
        float da[4], dg[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float s = sigmoid_acc(al[u]);
            da[u] = dl[u] * gl[u] * s * (1.0f + al[u] * (1.0f - s));
            dg[u] = dl[u] * al[u] * s;
        }
        uint2* row = reinterpret_cast<uint2*>(dadg + pr * 2 * n);
        row[c] = make_uint2(bf16x2(da[0], da[1]), bf16x2(da[2], da[3]));
        row[n4 + c] = make_uint2(bf16x2(dg[0], dg[1]), bf16x2(dg[2], dg[3]));
    }
}

// y = bf16(x), n elements (fp32 dy of the shared experts, whose weight is 1).
__global__ void to_bf16_kernel(const float* __restrict__ x, long long n, __nv_bfloat16* __restrict__ y) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
        y[i] = __float2bfloat16_rn(x[i]);
}

// dx[t] = sum_j dxp[prow[inv[t*k + j]]] (overwrite, j in order), one warp
// per token; d % 4 == 0: 16-byte loads and stores.
__global__ void __launch_bounds__(256) unpermute_sum_pad_kernel(const float* __restrict__ dxp,
                                                                const int32_t* __restrict__ inv,
                                                                const int32_t* __restrict__ prow, float* dx, int d,
                                                                int k, int rows, int T, int* status) {
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;  // warp-uniform
    // padded row of assignment j in lane j (k <= 32); -1: a corrupt inverse entry, skipped
    long long my_row = -1;
    if (lane < k) {
        const int r = inv[(long long)t * k + lane];
        if (r < 0 || r >= rows)
            report(status, kStDeviceCheck);
        else
            my_row = prow[r];
    }
    const int d4 = d / 4;
    float4* out = reinterpret_cast<float4*>(dx + (long long)t * d);
    for (int c = lane; c < d4; c += 32) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const long long pr = __shfl_sync(0xffffffffu, my_row, j);
            if (pr < 0) continue;
            const float4 x = reinterpret_cast<const float4*>(dxp + pr * d)[c];
            v.x += x.x;
            v.y += x.y;
            v.z += x.z;
            v.w += x.w;
        }
        out[c] = v;
    }
}

// ------------------------------------------------------------------ launch helpers

Opnd view(const void* p, bool bf16, long long rs, long long cs, long long gs = 0, const int32_t* gather = nullptr,
          int gdiv = 1) {
    return Opnd{p, bf16 ? 1 : 0, rs, cs, gs, gather, gdiv};
}

cudaError_t rows_gemm(const Opnd& A, const Opnd& B, float* C, long long c_rs, int M, int N, int K,
                      const int32_t* offsets, int G, bool accumulate, int* status, int num_sms, cudaStream_t st) {
    if (M <= 0 || N <= 0) return cudaSuccess;
    RowsGemm p{A, B, C, c_rs, M, N, K, offsets, G, accumulate ? 1 : 0,
               vec8_ok(A.p, A.bf16, A.rs, A.cs, A.gs) ? 1 : 0, vec8_ok(B.p, B.bf16, B.rs, B.cs, B.gs) ? 1 : 0,
               status};
    // an upper bound of the tile count: every group adds at most one partial m-tile
    const long long tiles = ((long long)(M + TB - 1) / TB + G) * ((N + TB - 1) / TB);
    const int grid = (int)(tiles < (long long)num_sms * 2 ? tiles : (long long)num_sms * 2);
    rows_gemm_kernel<<<grid, 256, 0, st>>>(p);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t wgrad_gemm(const Opnd& A, const Opnd& B, float* C, long long c_rs, long long c_gs, int M, int N,
                       const int32_t* offsets, int G, int rows, bool accumulate, int* status, cudaStream_t st) {
    if (M <= 0 || N <= 0 || G <= 0) return cudaSuccess;
    WgradGemm p{A, B, C, c_rs, c_gs, M, N, offsets, G, rows, accumulate ? 1 : 0, status};
    const dim3 grid((unsigned)(((M + TB - 1) / TB) * ((N + TB - 1) / TB)), (unsigned)G);
    wgrad_gemm_kernel<<<grid, 256, 0, st>>>(p);
    note_launches(1);
    return cudaGetLastError();
}

int ew_grid(long long n) {
    const long long b = (n + 255) / 256;
    return (int)(b < 4096 ? (b > 0 ? b : 1) : 4096);
}

}  // namespace

// Whether the expert contractions run on the tensor cores: bf16 layers whose
// widths fit the 128-column tiles of the MN-major operands.
bool backward_on_tensor_cores(bool bf16, int d, int I, int S, int Is) {
    return bf16 && d % 128 == 0 && I % 128 == 0 && (S == 0 || Is % 128 == 0);
}

namespace {
struct BwdCarve {
    char* p;
    size_t used = 0;
    template <typename T>
    T* take(size_t bytes) {
        const size_t al = (bytes + 255) & ~size_t(255);
        T* q = reinterpret_cast<T*>(p ? p + used : nullptr);
        used += al;
        return q;
    }
};

// Buffers of the backward, carved from the workspace in this order (the
// sizes depend on the path: fp32 SIMT, or the tensor cores' padded bf16 layout).
struct BwdBufs {
    int32_t *offsets, *perm, *inv, *pscratch, *cnt;
    float *dw, *dz, *tot, *part, *chunk;
    // SIMT path
    float *abuf, *gbuf, *hbuf, *dhbuf, *obuf, *as, *gs, *hs, *dhs;
    // tensor-core path: routed rows in the padded layout (Rp rows), shared rows T
    int32_t *pstart, *prow;
    uint16_t *x_pad, *h_pad, *do_pad, *dadg, *hs16, *dys16, *dadgs, *dz16;
    float *a_pad, *g_pad, *o_pad, *dh_pad, *as32, *gs32, *dhs32;
};

size_t carve(BwdBufs* o, char* base, int T, int d, int E, int k, int I, int S, int Is, int seq_len, bool tc) {
    BwdCarve c{base};
    const size_t R = (size_t)T * k;
    const size_t nb = seq_len > 0 ? (size_t)T / seq_len : 0;
    const size_t C = seq_len > 0 ? ((size_t)seq_len + kLossChunk - 1) / kLossChunk : 0;
    const size_t SI = (size_t)S * Is;
    BwdBufs b{};
    b.offsets = c.take<int32_t>((E + 1) * 4);
    b.perm = c.take<int32_t>(R * 4);
    b.inv = c.take<int32_t>(R * 4);
    b.pscratch = c.take<int32_t>(permute_scratch_bytes(T, E));
    b.dw = c.take<float>(R * 4);
    b.dz = c.take<float>((size_t)T * E * 4);
    b.tot = c.take<float>((size_t)T * 4);
    b.cnt = c.take<int32_t>(nb * E * 4);
    b.part = c.take<float>(nb * 4);
    b.chunk = c.take<float>(nb * C * E * 4);
    if (!tc) {
        b.abuf = c.take<float>(R * I * 4);
        b.gbuf = c.take<float>(R * I * 4);
        b.hbuf = c.take<float>(R * I * 4);
        b.dhbuf = c.take<float>(R * I * 4);
        b.obuf = c.take<float>(R * d * 4);
        b.as = c.take<float>((size_t)T * SI * 4);
        b.gs = c.take<float>((size_t)T * SI * 4);
        b.hs = c.take<float>((size_t)T * SI * 4);
        b.dhs = c.take<float>((size_t)T * SI * 4);
    } else {
        const size_t Rp = R + (size_t)kPad * E;  // padded rows: at most kPad - 1 more per expert
        b.pstart = c.take<int32_t>((E + 1) * 4);
        b.prow = c.take<int32_t>(R * 4);
        b.x_pad = c.take<uint16_t>(Rp * d * 2);
        b.h_pad = c.take<uint16_t>(Rp * I * 2);
        b.do_pad = c.take<uint16_t>(Rp * d * 2);
        b.dadg = c.take<uint16_t>(Rp * 2 * I * 2);
        b.a_pad = c.take<float>(Rp * I * 4);
        b.g_pad = c.take<float>(Rp * I * 4);
        b.dh_pad = c.take<float>(Rp * I * 4);
        b.o_pad = c.take<float>(Rp * d * 4);
        b.as32 = c.take<float>((size_t)T * SI * 4);
        b.gs32 = c.take<float>((size_t)T * SI * 4);
        b.dhs32 = c.take<float>((size_t)T * SI * 4);
        b.hs16 = c.take<uint16_t>((size_t)T * SI * 2);
        b.dys16 = c.take<uint16_t>((size_t)T * d * 2);
        b.dadgs = c.take<uint16_t>((size_t)T * 2 * SI * 2);
        b.dz16 = c.take<uint16_t>((size_t)T * E * 2);
    }
    if (o) *o = b;
    return c.used;
}
}  // namespace

size_t backward_scratch_bytes(int T, int d, int E, int k, int I, int S, int Is, int seq_len, bool bf16) {
    return carve(nullptr, nullptr, T, d, E, k, I, S, Is, seq_len, backward_on_tensor_cores(bf16, d, I, S, Is));
}

namespace {

// The expert part of the backward on the tensor cores (bf16 layer): writes
// dw (per assignment), dx (routed + shared), dW1/dW3/dW2 and the shared
// gradients.  bf16 operands (x, h, do = w dy, da, dg, the shared dy), fp32
// accumulation and fp32 results.
cudaError_t experts_backward_tc(const BackwardArgs& a, const BwdBufs& b, int* status, int num_sms, cudaStream_t st) {
    const int T = a.T, d = a.d, E = a.E, k = a.k, I = a.I, S = a.S, Is = a.Is;
    const int R = T * k;
    const long long Rp = (long long)R + (long long)kPad * E;
    const int SI = S * Is;
    cudaError_t err;
#define TC_TRY(x)                                  \
    do {                                           \
        if ((err = (x)) != cudaSuccess) return err; \
    } while (0)
    // padded layout of the routed rows, and the zero padding of the GEMM operands
    pad_plan_kernel<<<1, 32, 0, st>>>(a.counts, E, b.pstart, status);
    note_launches(1);
    {
        PadZero z{{reinterpret_cast<uint4*>(b.x_pad), reinterpret_cast<uint4*>(b.h_pad),
                    reinterpret_cast<uint4*>(b.do_pad), reinterpret_cast<uint4*>(b.dadg)},
                   {d / 8, I / 8, d / 8, 2 * I / 8}};
        pad_zero_kernel<<<E, 256, 0, st>>>(a.counts, b.pstart, E, z);
        note_launches(1);
    }
    if (R > 0) {
        gather_pad_kernel<<<num_sms * 4, 256, 0, st>>>(static_cast<const uint4*>(a.x), b.perm, b.offsets, b.pstart,
                                                       E, k, R, T, d / 8, b.prow, reinterpret_cast<uint4*>(b.x_pad),
                                                       status);
        note_launches(1);
    }
    auto rows_args = [&](const void* W, long long W_rows, long long a_grow, const void* X, long long op_rows, int K,
                         int M_total, float* out, bool routed) {
        BwdRowsArgs r{};
        r.W = W;
        r.W1 = nullptr;
        r.W_rows = W_rows;
        r.K0 = 0;
        r.a_grow = a_grow;
        r.X = X;
        r.op_rows = op_rows;
        r.K = K;
        r.M_total = M_total;
        r.start = routed ? b.pstart : nullptr;
        r.rows = routed ? a.counts : nullptr;
        r.G = routed ? E : 1;
        r.M_rows = routed ? 0 : T;
        r.out = out;
        r.ldo = M_total;
        r.accumulate = false;
        return r;
    };
    auto wgrad_args = [&](const void* A, int lda, long long a_col0, const void* B, int ldb, long long b_col0,
                          long long op_rows, int M_total, int N_total, float* out, bool routed) {
        BwdWgradArgs w{};
        w.A = A;
        w.lda = lda;
        w.a_col0 = a_col0;
        w.B = B;
        w.ldb = ldb;
        w.b_col0 = b_col0;
        w.op_rows = op_rows;
        w.M_total = M_total;
        w.N_total = N_total;
        w.start = routed ? b.pstart : nullptr;
        w.rows = routed ? a.counts : nullptr;
        w.G = routed ? E : 1;
        w.M_rows = routed ? 0 : T;
        w.out = out;
        return w;
    };

    // ---- recompute, routed and shared experts in one launch of the forward's gate/up GEMM: a = x W1^T and
    // g = x W3^T (fp32) beside h = bf16(silu(a) g), the very h the forward computed.  The routed groups are the
    // padded segments (pstart), whose zero padding rows give a = g = h = 0; the shared set is one group of T rows.
    {
        TcUpArgs ur{};
        ur.A = b.x_pad;
        ur.A_rows = Rp;
        ur.gather_div = 1;
        ur.W1 = a.w1;
        ur.W3 = a.w3;
        ur.W_rows = (long long)E * I;
        ur.H = b.h_pad;
        ur.d = d;
        ur.I = I;
        ur.offsets = b.pstart;
        ur.G = E;
        ur.pre_a = b.a_pad;
        ur.pre_g = b.g_pad;
        TcUpArgs us{};
        us.A = a.x;
        us.A_rows = T;
        us.gather_div = 1;
        us.W1 = a.ws1;
        us.W3 = a.ws3;
        us.W_rows = (long long)S * Is;
        us.H = b.hs16;
        us.d = d;
        us.I = S * Is;
        us.G = 1;
        us.M = T;
        us.pre_a = b.as32;
        us.pre_g = b.gs32;
        TC_TRY(launch_tc_up(R > 0 ? &ur : nullptr, S > 0 && T > 0 ? &us : nullptr, status, num_sms, st));
    }

    // ---- routed experts
    // dy_t and do = w dy_t (bf16) on every assignment's padded row; dy_pad lives in the o_pad buffer,
    // which dx_perm overwrites only after its last use.  Its padding rows are never cleared: a B row of
    // the rows GEMM only reaches the output row of the same index, and padding rows are not stored.
    uint16_t* dy_pad = reinterpret_cast<uint16_t*>(b.o_pad);
    if (R > 0) {
        spread_dy_pad_kernel<<<(R + 7) / 8, 256, 0, st>>>(a.dy, a.w, b.inv, b.prow, dy_pad, b.do_pad, d, k, R, R,
                                                          status);
        note_launches(1);
    }
    // dW2_e = do^T h
    TC_TRY(launch_bwd_wgrad(wgrad_args(b.do_pad, d, 0, b.h_pad, I, 0, Rp, d, I, a.dw2, true), status, num_sms, st));
    // u = dy W2_e (W2 read along its output dimension); dh = w u.  The combine weight's gradient
    // <dy_t, o> = <dy_t, W2_e h> = <u, h> comes with it, so o is never recomputed.
    {
        BwdRowsArgs r = rows_args(a.w2, (long long)E * d, d, dy_pad, Rp, d, I, b.dh_pad, true);
        TC_TRY(launch_bwd_rows_mnmajor(r, status, num_sms, st));
    }
    if (R > 0) {
        swiglu_bwd_dw_pad_kernel<<<(R + 7) / 8, 256, 0, st>>>(b.a_pad, b.g_pad, b.dh_pad, b.prow, b.perm, a.w, R, I,
                                                              b.dadg, b.dw);
        note_launches(1);
    }
    // dW1_e = da^T x, dW3_e = dg^T x
    TC_TRY(launch_bwd_wgrad(wgrad_args(b.dadg, 2 * I, 0, b.x_pad, d, 0, Rp, I, d, a.dw1, true), status, num_sms, st));
    TC_TRY(launch_bwd_wgrad(wgrad_args(b.dadg, 2 * I, I, b.x_pad, d, 0, Rp, I, d, a.dw3, true), status, num_sms, st));
    // dx_perm = da W1_e + dg W3_e (the o buffer), then summed back per token
    {
        BwdRowsArgs r = rows_args(a.w1, (long long)E * I, I, b.dadg, Rp, 2 * I, d, b.o_pad, true);
        r.W1 = a.w3;
        r.K0 = I;
        TC_TRY(launch_bwd_rows_mnmajor(r, status, num_sms, st));
    }
    if (T > 0) {
        unpermute_sum_pad_kernel<<<(T + 7) / 8, 256, 0, st>>>(b.o_pad, b.inv, b.prow, a.dx, d, k, R, T, status);
        note_launches(1);
    }

    // ---- shared experts: one group of T rows (rows past T read as zeros), S blocks stacked along the features
    if (S > 0 && T > 0) {
        // (as, gs and hs came with the recompute launch above)
        to_bf16_kernel<<<ew_grid((long long)T * d), 256, 0, st>>>(a.dy, (long long)T * d,
                                                                  reinterpret_cast<__nv_bfloat16*>(b.dys16));
        note_launches(1);
        const size_t eb = 2;
        for (int s = 0; s < S; ++s) {
            const char* w2s = static_cast<const char*>(a.ws2) + eb * (size_t)s * d * Is;
            // dWs2_s = dy^T hs_s
            TC_TRY(launch_bwd_wgrad(wgrad_args(b.dys16, d, 0, b.hs16, SI, (long long)s * Is, T, d, Is,
                                               a.dws2 + (size_t)s * d * Is, false),
                                    status, num_sms, st));
            // dhs_s = dy Ws2_s
            BwdRowsArgs r = rows_args(w2s, d, 0, b.dys16, T, d, Is, b.dhs32 + (size_t)s * Is, false);
            r.ldo = SI;
            TC_TRY(launch_bwd_rows_mnmajor(r, status, num_sms, st));
        }
        swiglu_bwd_pad_kernel<<<ew_grid((long long)T * SI / 4), 256, 0, st>>>(b.as32, b.gs32, b.dhs32, nullptr, T,
                                                                              SI, b.dadgs);
        note_launches(1);
        TC_TRY(launch_bwd_wgrad(wgrad_args(b.dadgs, 2 * SI, 0, a.x, d, 0, T, SI, d, a.dws1, false), status, num_sms,
                                st));
        TC_TRY(launch_bwd_wgrad(wgrad_args(b.dadgs, 2 * SI, SI, a.x, d, 0, T, SI, d, a.dws3, false), status, num_sms,
                                st));
        BwdRowsArgs r = rows_args(a.ws1, SI, 0, b.dadgs, T, 2 * SI, d, a.dx, false);
        r.W1 = a.ws3;
        r.K0 = SI;
        r.accumulate = true;
        TC_TRY(launch_bwd_rows_mnmajor(r, status, num_sms, st));
    }
#undef TC_TRY
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_layer_backward(const BackwardArgs& a, int* status, int num_sms, cudaStream_t st) {
    const int T = a.T, d = a.d, E = a.E, k = a.k, I = a.I, S = a.S, Is = a.Is;
    const bool bf = a.bf16;
    const int R = T * k;
    const int nb = a.alpha > 0.0f ? T / a.seq_len : 0;
    const bool tc = backward_on_tensor_cores(bf, d, I, S, Is);
    BwdBufs bb;
    carve(&bb, static_cast<char*>(a.workspace), T, d, E, k, I, S, Is, a.alpha > 0.0f ? a.seq_len : 0, tc);
    int32_t* offsets = bb.offsets;
    int32_t* perm = bb.perm;
    int32_t* inv = bb.inv;
    int32_t* pscratch = bb.pscratch;
    float* dw = bb.dw;
    float* dz = bb.dz;
    float* tot = bb.tot;
    int32_t* cnt = bb.cnt;
    float* part = bb.part;
    float* chunk = bb.chunk;
    const int C = nb > 0 ? (a.seq_len + kLossChunk - 1) / kLossChunk : 0;
    float* abuf = bb.abuf;
    float* gbuf = bb.gbuf;
    float* hbuf = bb.hbuf;
    float* dhbuf = bb.dhbuf;
    float* obuf = bb.obuf;
    const int SI = S * Is;
    float* as = bb.as;
    float* gs = bb.gs;
    float* hs = bb.hs;
    float* dhs = bb.dhs;

    cudaError_t err;
#define BWD_TRY(x)                          \
    do {                                    \
        if ((err = (x)) != cudaSuccess) return err; \
    } while (0)

    // routing layout of the forward: offsets, perm_tok, inv_row (no row copy)
    BWD_TRY(launch_permute(nullptr, a.idx, a.counts, T, d, E, k, bf ? 2 : 4, nullptr, offsets, perm, inv, pscratch,
                           status, st));

    if (tc) {
        BWD_TRY(experts_backward_tc(a, bb, status, num_sms, st));
    } else {
        // ---- routed experts
        const Opnd xg = view(a.x, bf, d, 1, 0, perm, k);  // x row of permuted row r
        BWD_TRY(rows_gemm(xg, view(a.w1, bf, d, 1, (long long)I * d), abuf, I, R, I, d, offsets, E, false, status,
                          a.num_sms, st));
        BWD_TRY(rows_gemm(xg, view(a.w3, bf, d, 1, (long long)I * d), gbuf, I, R, I, d, offsets, E, false, status,
                          a.num_sms, st));
        swiglu_fwd_kernel<<<ew_grid((long long)R * I), 256, 0, st>>>(abuf, gbuf, hbuf, (long long)R * I, bf ? 1 : 0);
        note_launches(1);
        // o = h W2_e^T
        BWD_TRY(rows_gemm(view(hbuf, false, I, 1), view(a.w2, bf, I, 1, (long long)d * I), obuf, d, R, d, I, offsets, E,
                          false, status, a.num_sms, st));
        if (R > 0) {
            combine_bwd_kernel<<<R, 256, 0, st>>>(a.dy, a.w, inv, obuf, dw, d, k, R, status);
            note_launches(1);
        }
        // dW2_e[c][i] = sum_r do[r][c] h[r][i]
        BWD_TRY(wgrad_gemm(view(obuf, false, d, 1), view(hbuf, false, I, 1), a.dw2, I, (long long)d * I, d, I, offsets, E,
                           R, false, status, st));
        // dh[r][i] = sum_c do[r][c] W2_e[c][i]
        BWD_TRY(rows_gemm(view(obuf, false, d, 1), view(a.w2, bf, 1, I, (long long)d * I), dhbuf, I, R, I, d, offsets, E,
                          false, status, a.num_sms, st));
        swiglu_bwd_kernel<<<ew_grid((long long)R * I), 256, 0, st>>>(abuf, gbuf, dhbuf, (long long)R * I);
        note_launches(1);
        // dW1_e = da^T x, dW3_e = dg^T x
        BWD_TRY(wgrad_gemm(view(dhbuf, false, I, 1), xg, a.dw1, d, (long long)I * d, I, d, offsets, E, R, false, status,
                           st));
        BWD_TRY(wgrad_gemm(view(gbuf, false, I, 1), xg, a.dw3, d, (long long)I * d, I, d, offsets, E, R, false, status,
                           st));
        // dx_perm = da W1_e + dg W3_e  (into the do buffer, no longer needed)
        BWD_TRY(rows_gemm(view(dhbuf, false, I, 1), view(a.w1, bf, 1, d, (long long)I * d), obuf, d, R, d, I, offsets, E,
                          false, status, a.num_sms, st));
        BWD_TRY(rows_gemm(view(gbuf, false, I, 1), view(a.w3, bf, 1, d, (long long)I * d), obuf, d, R, d, I, offsets, E,
                          true, status, a.num_sms, st));
        if (T > 0) {
            unpermute_sum_kernel<<<T, 256, 0, st>>>(obuf, inv, a.dx, d, k, R, status);
            note_launches(1);
        }

        // ---- shared experts: one group of T rows, the S blocks stacked along the features
        if (S > 0) {
            const Opnd x = view(a.x, bf, d, 1);
            BWD_TRY(rows_gemm(x, view(a.ws1, bf, d, 1), as, SI, T, SI, d, nullptr, 1, false, status, a.num_sms, st));
            BWD_TRY(rows_gemm(x, view(a.ws3, bf, d, 1), gs, SI, T, SI, d, nullptr, 1, false, status, a.num_sms, st));
            swiglu_fwd_kernel<<<ew_grid((long long)T * SI), 256, 0, st>>>(as, gs, hs, (long long)T * SI, bf ? 1 : 0);
            note_launches(1);
            const Opnd dyv = view(a.dy, false, d, 1);
            const size_t eb = bf ? 2 : 4;
            for (int s = 0; s < S; ++s) {
                const char* w2s = static_cast<const char*>(a.ws2) + eb * (size_t)s * d * Is;
                // dWs2_s[c][i] = sum_t dy[t][c] hs[t][s*Is + i]
                BWD_TRY(wgrad_gemm(dyv, view(hs + (size_t)s * Is, false, SI, 1), a.dws2 + (size_t)s * d * Is, Is, 0, d,
                                   Is, nullptr, 1, T, false, status, st));
                // dhs[t][s*Is + i] = sum_c dy[t][c] Ws2_s[c][i]
                BWD_TRY(rows_gemm(dyv, view(w2s, bf, 1, Is), dhs + (size_t)s * Is, SI, T, Is, d, nullptr, 1, false, status,
                                  a.num_sms, st));
            }
            swiglu_bwd_kernel<<<ew_grid((long long)T * SI), 256, 0, st>>>(as, gs, dhs, (long long)T * SI);
            note_launches(1);
            BWD_TRY(wgrad_gemm(view(dhs, false, SI, 1), x, a.dws1, d, 0, SI, d, nullptr, 1, T, false, status, st));
            BWD_TRY(wgrad_gemm(view(gs, false, SI, 1), x, a.dws3, d, 0, SI, d, nullptr, 1, T, false, status, st));
            BWD_TRY(rows_gemm(view(dhs, false, SI, 1), view(a.ws1, bf, 1, d), a.dx, d, T, d, SI, nullptr, 1, true, status,
                              a.num_sms, st));
            BWD_TRY(rows_gemm(view(gs, false, SI, 1), view(a.ws3, bf, 1, d), a.dx, d, T, d, SI, nullptr, 1, true, status,
                              a.num_sms, st));
        }
    }

    // ---- router and balance loss
    if (T > 0) {
        if (nb > 0) {
            BWD_TRY(cudaMemsetAsync(cnt, 0, (size_t)nb * E * 4, st));
            seq_counts_kernel<<<ew_grid((long long)R), 256, 0, st>>>(a.idx, T, k, E, a.seq_len, cnt, status);
            note_launches(1);
        }
        router_bwd_kernel<<<(T + 7) / 8, 256, 0, st>>>(a.s, a.idx, dw, nb > 0 ? cnt : nullptr, a.alpha, a.seq_len,
                                                        nb, T, E, k, dz, tot, status);
        note_launches(1);
        if (nb > 0 && a.loss) {
            const size_t gsm = (size_t)(256 / E) * E * sizeof(float);  // E <= 256
            balance_chunk_kernel<<<dim3((unsigned)C, (unsigned)nb), 256, gsm, st>>>(a.s, tot, a.seq_len, E, C, chunk);
            balance_part_kernel<<<nb, 256, gsm, st>>>(chunk, cnt, a.alpha, a.seq_len, E, k, C, part);
            balance_sum_kernel<<<1, 32, 0, st>>>(part, nb, a.loss);
            note_launches(3);
        }
        // dx += dz W_g;  dW_g = dz^T x.  On the tensor-core path with dz in bf16: dW_g whenever E % 8 == 0
        // (16-byte rows of dz), dx when E % 64 == 0 (whole 64-column stages of the contraction).
        if (tc && E % 8 == 0) {
            to_bf16_kernel<<<ew_grid((long long)T * E), 256, 0, st>>>(dz, (long long)T * E,
                                                                      reinterpret_cast<__nv_bfloat16*>(bb.dz16));
            note_launches(1);
        }
        if (tc && E % 64 == 0) {
            BwdRowsArgs r{};
            r.W = a.w_gate;
            r.W1 = nullptr;
            r.W_rows = E;
            r.K0 = 0;
            r.a_grow = 0;
            r.X = bb.dz16;
            r.op_rows = T;
            r.K = E;
            r.M_total = d;
            r.start = nullptr;
            r.rows = nullptr;
            r.G = 1;
            r.M_rows = T;
            r.out = a.dx;
            r.ldo = d;
            r.accumulate = true;
            BWD_TRY(launch_bwd_rows_mnmajor(r, status, num_sms, st));
        } else {
            BWD_TRY(rows_gemm(view(dz, false, E, 1), view(a.w_gate, bf, 1, d), a.dx, d, T, d, E, nullptr, 1, true,
                              status, a.num_sms, st));
        }
    }
    if (tc && E % 8 == 0 && T > 0) {
        BwdWgradArgs w{};
        w.A = bb.dz16;
        w.lda = E;
        w.a_col0 = 0;
        w.B = a.x;
        w.ldb = d;
        w.b_col0 = 0;
        w.op_rows = T;
        w.M_total = E;
        w.N_total = d;
        w.start = nullptr;
        w.rows = nullptr;
        w.G = 1;
        w.M_rows = T;
        w.out = a.dw_gate;
        BWD_TRY(launch_bwd_wgrad(w, status, num_sms, st));
    } else {
        BWD_TRY(wgrad_gemm(view(dz, false, E, 1), view(a.x, bf, d, 1), a.dw_gate, d, 0, E, d, nullptr, 1, T, false,
                           status, st));
    }
    if (a.loss && nb == 0) BWD_TRY(cudaMemsetAsync(a.loss, 0, sizeof(float), st));
#undef BWD_TRY
    return cudaSuccess;
}

}  // namespace moe
