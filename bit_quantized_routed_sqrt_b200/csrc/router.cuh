// router.cuh -- router logits, certified top-k with normalised sqrt(softplus) weights,
// and the token->expert permutation.
//
// Selection must equal an fp64 evaluation whose logit is the sequential sum
// sum_i x_i * Wr_i (i ascending, then + bias) ranked by (logit desc, index asc).
// The fast logits here carry a rigorous error bound |fast - exact| <= c * A + tiny, where
// A >= sum_i |x_i Wr_i|; the fp64 sequential sum is itself within 4.6e-13 * A of the exact
// value.  When the selected set and its order are decided by more than both bounds the
// result is certain; otherwise the candidates whose intervals overlap are recomputed
// with the same sequential fp64 sum and ranked again.
#pragma once
#include "common.cuh"

namespace ds4 {

constexpr int MAX_TOPK = 16;
constexpr int MAX_EXPERTS = 256;

// Coefficients c of the fast-logit error bound (per unit of A):
//  pairs summed in fp32 (one rounding per two exact products), then fp64:  u32 + O(1e-12)
//  chunks of 8 products summed in fp32, then fp64:                         gamma_7 + O(1e-12)
constexpr float BOUND_PAIR = 6.0e-8f;
constexpr float BOUND_CHUNK8 = 4.2e-7f;

struct RouteOut {
    int *topk_idx;   // [T][k]
    float *topk_w;   // [T][k]
    int *offsets;    // [E+1]
    int *sorted_token, *sorted_slot, *inv_pos;  // [T*k]
    int *active;     // [E] experts with pairs, ascending
    int *n_active;   // [1]
    unsigned long long *fallbacks;
    int *status;
};

__device__ __forceinline__ double margin_of(double lg, float a, float coef, int H) {
    // a is an fp32 accumulation of non-negative terms: inflate by its own relative error.
    return (double)coef * (double)a * (1.0 + H * 1.2e-7) + 1e-15 * fabs(lg) + 1e-38;
}

// The oracle-order logit: sequential fp64 sum of the exact products, then + bias.
__device__ double exact_logit(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ w, int H,
                              const float *bias_e) {
    double acc = 0.0;
    for (int i = 0; i < H; i += 8) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(x + i));
        const uint4 wv = __ldg(reinterpret_cast<const uint4 *>(w + i));
        const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w}, ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            acc = __dadd_rn(acc, __dmul_rn((double)bf16lo(xs[q]), (double)bf16lo(ws[q])));
            acc = __dadd_rn(acc, __dmul_rn((double)bf16hi(xs[q]), (double)bf16hi(ws[q])));
        }
    }
    if (bias_e) acc = __dadd_rn(acc, (double)*bias_e);
    return acc;
}

__device__ __forceinline__ bool better(double va, int ia, double vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

// Warp-wide selection of the k best (value desc, index asc) among lane-held values.
// vals[i] is expert lane + 32 i (NPL per lane); sel bit i marks taken values.
template <int NPL>
__device__ __forceinline__ void warp_select(const double (&vals)[NPL], int E, int k, unsigned &sel, int *sel_e,
                                            double *sel_v) {
    const int lane = threadIdx.x & 31;
    for (int j = 0; j < k; ++j) {
        double bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !(sel >> i & 1u) && better(vals[i], e, bv, bi)) { bv = vals[i]; bi = e; }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
            const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
            if (better(ov, oi, bv, bi)) { bv = ov; bi = oi; }
        }
        if (bi < 0 || bi >= E) bi = 0;   // only reachable with non-finite logits
        if ((bi & 31) == lane) sel |= 1u << (bi >> 5);
        sel_e[j] = bi;
        sel_v[j] = bv;
    }
}

// Certified top-k of one token, executed by one full warp.
//  lg/la: the token's E fast logits (fp64) and bound bases A (fp32), in memory written by
//  this or an earlier kernel (read through L2).  Writes idx/w for the token (lane j < k).
template <int NPL>
__device__ void warp_topk_certified(const double *lg, const float *la, int E, int k, float coef, int H,
                                    const __nv_bfloat16 *xrow, const __nv_bfloat16 *wr, const float *bias,
                                    int *out_idx, float *out_w, unsigned long long *fallbacks) {
    const int lane = threadIdx.x & 31;
    double v[NPL], m[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            v[i] = __ldcg(lg + e);
            m[i] = margin_of(v[i], __ldcg(la + e), coef, H);
        } else {
            v[i] = -INFINITY;
            m[i] = 0.0;
        }
    }
    unsigned sel = 0;
    int se[MAX_TOPK];
    double sv[MAX_TOPK];
    warp_select<NPL>(v, E, k, sel, se, sv);

    // certification
    // margins of the selected experts, fetched from the owning lanes
    double sm[MAX_TOPK];
    for (int j = 0; j < k; ++j) {
        double mine = 0.0;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (lane + 32 * i == se[j]) mine = m[i];
        sm[j] = __shfl_sync(0xffffffffu, mine, se[j] & 31);
    }
    double msel = INFINITY;
    bool ordered = true;
    for (int j = 0; j < k; ++j) {
        msel = fmin(msel, sv[j] - sm[j]);
        if (j + 1 < k && !(sv[j] - sm[j] > sv[j + 1] + sm[j + 1])) ordered = false;
    }
    double omax = -INFINITY;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        if (lane + 32 * i < E && !(sel >> i & 1u)) omax = fmax(omax, v[i] + m[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) omax = fmax(omax, __shfl_xor_sync(0xffffffffu, omax, o));
    const bool certified = ordered && omax < msel;

    if (!certified) {
        // candidates: every expert whose interval reaches the lowest selected lower bound;
        // each is recomputed in the sequential fp64 order, the rest drop out.
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            if (e < E && v[i] + m[i] >= msel)
                v[i] = exact_logit(xrow, wr + (size_t)e * H, H, bias ? bias + e : nullptr);
            else
                v[i] = -INFINITY;
        }
        sel = 0;
        warp_select<NPL>(v, E, k, sel, se, sv);
        if (lane == 0 && fallbacks) atomicAdd(fallbacks, 1ull);
    }

    float s[MAX_TOPK];
    float ssum = 0.0f;
    for (int j = 0; j < k; ++j) {
        s[j] = router_score((float)sv[j]);
        ssum += s[j];
    }
    for (int j = 0; j < k; ++j)
        if (lane == j) {
            out_idx[j] = se[j];
            out_w[j] = ssum > 0.0f ? s[j] / ssum : 1.0f / k;
        }
}

// ---------------------------------------------------------------------------------------
// Decode router rows: one warp computes RW router rows for all T tokens (pairs of exact
// products rounded once in fp32, then accumulated in fp64), with A = sum |x_i Wr_i|.
template <int RW, int TT>
__device__ void router_rows_warp(const __nv_bfloat16 *__restrict__ x, int T, int H, const __nv_bfloat16 *__restrict__ wr,
                                 const float *bias, int e0, int E, double *logits, float *labs) {
    const int lane = threadIdx.x & 31;
    for (int t0 = 0; t0 < T; t0 += TT) {
        const int nt = min(TT, T - t0);
        double acc[RW][TT];
        float ab[RW][TT];
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int t = 0; t < TT; ++t) { acc[r][t] = 0.0; ab[r][t] = 0.0f; }
        for (int k0 = lane * 8; k0 < H; k0 += 256) {
            uint4 wv[RW];
#pragma unroll
            for (int r = 0; r < RW; ++r)
                wv[r] = (e0 + r < E) ? ld_stream_v4(wr + (size_t)(e0 + r) * H + k0) : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                if (t < nt) {
                    const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)(t0 + t) * H + k0));
                    const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                    for (int r = 0; r < RW; ++r) {
                        const uint32_t ws[4] = {wv[r].x, wv[r].y, wv[r].z, wv[r].w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float x0 = bf16lo(xs[q]), x1 = bf16hi(xs[q]);
                            const float w0 = bf16lo(ws[q]), w1 = bf16hi(ws[q]);
                            const float p = __fmaf_rn(x1, w1, __fmul_rn(x0, w0));
                            acc[r][t] += (double)p;
                            ab[r][t] = __fmaf_rn(fabsf(x0), fabsf(w0), __fmaf_rn(fabsf(x1), fabsf(w1), ab[r][t]));
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int r = 0; r < RW; ++r)
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                const double s = warp_sum(acc[r][t]);
                const float a = warp_sum(ab[r][t]);
                if (lane == 0 && t < nt && e0 + r < E) {
                    const int e = e0 + r;
                    logits[(size_t)(t0 + t) * E + e] = bias ? __dadd_rn(s, (double)bias[e]) : s;
                    labs[(size_t)(t0 + t) * E + e] = a;
                }
            }
    }
}

// ---------------------------------------------------------------------------------------
// Permutation of one block of up to 64 tokens, executed by a whole CTA.
//   idx: [nt][k] selected experts of tokens t0 .. t0+nt-1 (smem or global)
//   cnt/mask: smem [E] scratch, zeroed by the caller and synchronised.
__device__ void block_count_masks(const int *idx, int nt, int k, int *cnt, unsigned long long *mask) {
    for (int p = threadIdx.x; p < nt * k; p += blockDim.x) {
        const int e = idx[p];
        atomicAdd(cnt + e, 1);
        atomicOr(mask + e, 1ull << (p / k));
    }
}

// Exclusive scan of cnt[0..E) into off[0..E] and the ascending list of experts with pairs;
// executed by warp 0 of the CTA.  E <= 256.
__device__ void warp_scan_active(const int *cnt, int E, int *off, int *active, int *n_active) {
    const int lane = threadIdx.x & 31;
    int base = 0, nact = 0;
    for (int c = 0; c < E; c += 32) {
        const int e = c + lane;
        const int v = e < E ? cnt[e] : 0;
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += n;
        }
        if (e < E) off[e] = base + incl - v;
        const unsigned bal = __ballot_sync(0xffffffffu, v > 0);
        if (v > 0) active[nact + __popc(bal & ((1u << lane) - 1))] = e;
        nact += __popc(bal);
        base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
        off[E] = base;
        *n_active = nact;
    }
}

// Prefill router: CTA tile of RT tokens x RE experts, SIMT fp32 chunks of 8 products
// accumulated in fp64, bound base A = ||x_t||_2 * ||Wr_e||_2 (Cauchy-Schwarz).
constexpr int PR_T = 32, PR_E = 64, PR_K = 32;
__global__ void __launch_bounds__(256) router_gemm_kernel(const __nv_bfloat16 *__restrict__ x, int T, int H,
                                                          const __nv_bfloat16 *__restrict__ wr, int E,
                                                          const float *__restrict__ bias,
                                                          const float *__restrict__ wr_norm, double *logits,
                                                          float *labs) {
    __shared__ float xs[PR_T][PR_K + 1];
    __shared__ float ws[PR_E][PR_K + 1];
    __shared__ double xn2[PR_T];
    const int t0 = blockIdx.x * PR_T, e0 = blockIdx.y * PR_E;
    const int tid = threadIdx.x;
    const int tr = tid / 16, er = tid % 16;   // thread computes tokens tr*2 +{0,1}, experts er*4 + {0..3}
    double acc[2][4];
    float c32[2][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) { acc[i][j] = 0.0; c32[i][j] = 0.0f; }
    if (tid < PR_T) xn2[tid] = 0.0;
    for (int k0 = 0; k0 < H; k0 += PR_K) {
        __syncthreads();
        // load X tile: 32 tokens x 32 k (bf16) -> fp32
        for (int i = tid; i < PR_T * PR_K / 2; i += 256) {
            const int tt = i / (PR_K / 2), kk = (i % (PR_K / 2)) * 2;
            uint32_t v = 0;
            if (t0 + tt < T) v = __ldg(reinterpret_cast<const uint32_t *>(x + (size_t)(t0 + tt) * H + k0 + kk));
            xs[tt][kk] = bf16lo(v);
            xs[tt][kk + 1] = bf16hi(v);
        }
        for (int i = tid; i < PR_E * PR_K / 2; i += 256) {
            const int ee = i / (PR_K / 2), kk = (i % (PR_K / 2)) * 2;
            uint32_t v = 0;
            if (e0 + ee < E) v = __ldg(reinterpret_cast<const uint32_t *>(wr + (size_t)(e0 + ee) * H + k0 + kk));
            ws[ee][kk] = bf16lo(v);
            ws[ee][kk + 1] = bf16hi(v);
        }
        __syncthreads();
        if (tid < PR_T) {
            double s = 0.0;
            for (int kk = 0; kk < PR_K; ++kk) s += (double)xs[tid][kk] * (double)xs[tid][kk];
            xn2[tid] += s;
        }
#pragma unroll
        for (int kc = 0; kc < PR_K; kc += 8) {
#pragma unroll
            for (int kk = kc; kk < kc + 8; ++kk) {
                float a[2], b[4];
#pragma unroll
                for (int i = 0; i < 2; ++i) a[i] = xs[tr * 2 + i][kk];
#pragma unroll
                for (int j = 0; j < 4; ++j) b[j] = ws[er * 4 + j][kk];
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) c32[i][j] = __fmaf_rn(a[i], b[j], c32[i][j]);
            }
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) { acc[i][j] += (double)c32[i][j]; c32[i][j] = 0.0f; }
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int t = t0 + tr * 2 + i;
        if (t >= T) continue;
        const float xn = (float)sqrt(xn2[tr * 2 + i]) * (1.0f + 1e-6f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + er * 4 + j;
            if (e >= E) continue;
            const double s = acc[i][j];
            logits[(size_t)t * E + e] = bias ? __dadd_rn(s, (double)bias[e]) : s;
            labs[(size_t)t * E + e] = xn * wr_norm[e];
        }
    }
}

// Prefill top-k + per-64-token-block counts and masks: one CTA (8 warps) per 64 tokens.
template <int NPL>
__global__ void __launch_bounds__(256) topk_block_kernel(const double *logits, const float *labs, int T, int E,
                                                         int k, int H, float coef,
                                                         const __nv_bfloat16 *__restrict__ x,
                                                         const __nv_bfloat16 *__restrict__ wr,
                                                         const float *__restrict__ bias, RouteOut ro,
                                                         int *blk_cnt, unsigned long long *blk_mask) {
    __shared__ int cnt[MAX_EXPERTS];
    __shared__ unsigned long long mask[MAX_EXPERTS];
    __shared__ int sidx[64 * MAX_TOPK];
    const int t0 = blockIdx.x * 64;
    const int nt = min(64, T - t0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < E; e += blockDim.x) { cnt[e] = 0; mask[e] = 0ull; }
    for (int tt = warp; tt < nt; tt += 8) {
        const int t = t0 + tt;
        warp_topk_certified<NPL>(logits + (size_t)t * E, labs + (size_t)t * E, E, k, coef, H, x + (size_t)t * H, wr,
                                 bias, ro.topk_idx + (size_t)t * k, ro.topk_w + (size_t)t * k, ro.fallbacks);
        __syncwarp();
        if (lane < k) sidx[tt * k + lane] = ro.topk_idx[(size_t)t * k + lane];
    }
    __syncthreads();
    block_count_masks(sidx, nt, k, cnt, mask);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        blk_cnt[(size_t)blockIdx.x * E + e] = cnt[e];
        blk_mask[(size_t)blockIdx.x * E + e] = mask[e];
    }
}

// Prefill permutation scatter: one CTA per 64-token block; each CTA recomputes the
// expert offsets and its own per-expert base from the block counts (E * n_blocks reads).
__global__ void __launch_bounds__(256) permute_scatter_kernel(const int *blk_cnt, const unsigned long long *blk_mask,
                                                              int n_blocks, int T, int E, int k, RouteOut ro) {
    __shared__ int tot[MAX_EXPERTS], pre[MAX_EXPERTS], off[MAX_EXPERTS + 1];
    __shared__ int act[MAX_EXPERTS];
    __shared__ int nact;
    const int b = blockIdx.x;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int s = 0, p = 0;
        for (int bb = 0; bb < n_blocks; ++bb) {
            const int c = __ldcg(blk_cnt + (size_t)bb * E + e);
            if (bb < b) p += c;
            s += c;
        }
        tot[e] = s;
        pre[e] = p;
    }
    __syncthreads();
    if (threadIdx.x < 32) warp_scan_active(tot, E, off, act, &nact);
    __syncthreads();
    if (b == 0) {
        for (int e = threadIdx.x; e <= E; e += blockDim.x) ro.offsets[e] = off[e];
        for (int e = threadIdx.x; e < E; e += blockDim.x) ro.active[e] = e < nact ? act[e] : -1;
        if (threadIdx.x == 0) *ro.n_active = nact;
    }
    const int t0 = b * 64, nt = min(64, T - t0);
    for (int p = threadIdx.x; p < nt * k; p += blockDim.x) {
        const int tt = p / k, j = p % k, t = t0 + tt;
        const int e = __ldcg(ro.topk_idx + (size_t)t * k + j);
        const unsigned long long m = __ldcg(blk_mask + (size_t)b * E + e);
        const int pos = off[e] + pre[e] + __popcll(m & ((1ull << tt) - 1ull));
        ro.sorted_token[pos] = t;
        ro.sorted_slot[pos] = j;
        ro.inv_pos[(size_t)t * k + j] = pos;
    }
}

}  // namespace ds4
