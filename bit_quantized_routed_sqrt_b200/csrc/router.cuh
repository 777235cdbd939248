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
#include "mbar.cuh"

namespace ds4 {

constexpr int MAX_TOPK = 16;
constexpr int MAX_EXPERTS = 256;

// Coefficients c of the fast-logit error bound (per unit of A):
//  pairs summed in fp32 (one rounding per two exact products), then fp64:  u32 + O(1e-12)
//  chunks of 8 products summed in fp32, then fp64:                         gamma_7 + O(1e-12)
constexpr float BOUND_PAIR = 6.0e-8f;

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

// The oracle-order logit: sequential fp64 sum of the exact products, then + bias.  The
// operands of 32 inputs are loaded ahead of their additions (H is a multiple of 256).
__device__ double exact_logit(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ w, int H,
                              const float *bias_e) {
    double acc = 0.0;
    for (int i = 0; i < H; i += 32) {
        uint4 xv[4], wv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            xv[j] = __ldg(reinterpret_cast<const uint4 *>(x + i + 8 * j));
            wv[j] = __ldg(reinterpret_cast<const uint4 *>(w + i + 8 * j));
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t xs[4] = {xv[j].x, xv[j].y, xv[j].z, xv[j].w}, ws[4] = {wv[j].x, wv[j].y, wv[j].z, wv[j].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                acc = __dadd_rn(acc, __dmul_rn((double)bf16lo(xs[q]), (double)bf16lo(ws[q])));
                acc = __dadd_rn(acc, __dmul_rn((double)bf16hi(xs[q]), (double)bf16hi(ws[q])));
            }
        }
    }
    if (bias_e) acc = __dadd_rn(acc, (double)*bias_e);
    return acc;
}

// A logit to within a bound of the oracle's value, computed by the whole warp: each lane
// sums its 8-input slices of the exact products in fp64 (two alternating accumulators),
// then the lanes are summed by a butterfly.  Every product of two bf16 values is exact in
// fp64.  With A = sum_i |x_i w_i| and u = 2^-53, this sum is within gamma_(H/64 + 6) A of
// the exact one (H/64 additions per accumulator, one to join the two, five in the
// butterfly), the oracle's sequential sum within gamma_(H-1) A, and both add the bias with
// one more rounding, so the two values differ by at most the margin returned:
// (1.04 H + 64) * 1.12e-16 * A + 2.3e-16 * |logit| (+ 1e-300).
__device__ double precise_logit_warp(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ w,
                                     int H, const float *bias_e, double &margin) {
    const int lane = threadIdx.x & 31;
    double s0 = 0.0, s1 = 0.0, a = 0.0;
    for (int i = lane * 8; i < H; i += 256) {
        const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(x + i));
        const uint4 wv = __ldg(reinterpret_cast<const uint4 *>(w + i));
        const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w}, ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const double p0 = __dmul_rn((double)bf16lo(xs[q]), (double)bf16lo(ws[q]));
            const double p1 = __dmul_rn((double)bf16hi(xs[q]), (double)bf16hi(ws[q]));
            s0 = __dadd_rn(s0, p0);
            s1 = __dadd_rn(s1, p1);
            a = __dadd_rn(a, fabs(p0) + fabs(p1));
        }
    }
    double s = warp_sum(__dadd_rn(s0, s1));
    a = warp_sum(a) * (1.0 + 1e-12);
    if (bias_e) s = __dadd_rn(s, (double)*bias_e);
    margin = (1.04 * (double)H + 64.0) * 1.12e-16 * a + 2.3e-16 * fabs(s) + 1e-300;
    return s;
}

__device__ __forceinline__ bool better(double va, int ia, double vb, int ib) {
    return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ double shfl_d(double v, int src) { return __shfl_sync(0xffffffffu, v, src); }
__device__ __forceinline__ double warp_min_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmin(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ double warp_max_d(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// Order-preserving map of a double to an unsigned 64-bit key (larger value -> larger key).
__device__ __forceinline__ unsigned long long dkey(double v) {
    const unsigned long long u = (unsigned long long)__double_as_longlong(v);
    return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
__device__ __forceinline__ double dkey_value(unsigned long long k) {
    const unsigned long long u = (k >> 63) ? (k & 0x7fffffffffffffffull) : ~k;
    return __longlong_as_double((long long)u);
}
// Warp-wide max / min of a 64-bit key (two 32-bit reductions).
__device__ __forceinline__ unsigned long long warp_max_key(unsigned long long k) {
    const unsigned hi = __reduce_max_sync(0xffffffffu, (unsigned)(k >> 32));
    const unsigned lo = __reduce_max_sync(0xffffffffu, (unsigned)(k >> 32) == hi ? (unsigned)k : 0u);
    return ((unsigned long long)hi << 32) | lo;
}
__device__ __forceinline__ unsigned long long warp_min_key(unsigned long long k) {
    const unsigned hi = __reduce_min_sync(0xffffffffu, (unsigned)(k >> 32));
    const unsigned lo = __reduce_min_sync(0xffffffffu, (unsigned)(k >> 32) == hi ? (unsigned)k : 0xffffffffu);
    return ((unsigned long long)hi << 32) | lo;
}

// Warp-wide selection of the k best (value desc, index asc) among lane-held values;
// vals[i] / mrg[i] belong to expert lane + 32 i.  Each lane first orders its own values
// (a sorting network on registers); every round then takes the best lane head with three
// warp reductions (key high word, key low word among the tied, lowest index among equal
// keys).  Lane j < k receives slot j: its expert, value and margin.  sel marks the taken
// values of this lane (by original position).
template <int NPL>
__device__ __forceinline__ void warp_select(const double (&vals)[NPL], const double (&mrg)[NPL], int E, int k,
                                            unsigned &sel, int &my_e, double &my_v, double &my_m) {
    const int lane = threadIdx.x & 31;
    unsigned long long key[NPL];
    int pos[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        key[i] = (lane + 32 * i < E) ? dkey(vals[i]) : 0ull;
        pos[i] = i;
    }
    // odd-even transposition sort, descending by key; equal keys keep ascending position
#pragma unroll
    for (int r = 0; r < NPL; ++r)
#pragma unroll
        for (int i = r & 1; i + 1 < NPL; i += 2)
            if (key[i + 1] > key[i]) {
                const unsigned long long tk = key[i]; key[i] = key[i + 1]; key[i + 1] = tk;
                const int tp = pos[i]; pos[i] = pos[i + 1]; pos[i + 1] = tp;
            }
    int head = 0;
    for (int j = 0; j < k; ++j) {
        unsigned long long hk = 0ull;
        int hp = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (i == head) { hk = key[i]; hp = pos[i]; }
        const int he = (head < NPL) ? lane + 32 * hp : 0x7fffffff;
        if (head >= NPL) hk = 0ull;
        const unsigned long long best = warp_max_key(hk);
        const unsigned win_e = __reduce_min_sync(0xffffffffu, (hk == best && head < NPL) ? (unsigned)he : 0xffffffffu);
        int be = (int)win_e;
        if (be < 0 || be >= E) be = 0;   // only reachable with non-finite logits
        double bm = 0.0;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (lane + 32 * i == be) bm = mrg[i];
        bm = __shfl_sync(0xffffffffu, bm, be & 31);
        if ((be & 31) == lane) {
            sel |= 1u << (be >> 5);
            ++head;
        }
        if (lane == j) { my_e = be; my_v = dkey_value(best); my_m = bm; }
    }
}

// Certified top-k of one token, executed by one full warp.
//  lg/la: the token's E fast logits (fp64) and bound bases A (fp32), in memory written by
//  this or an earlier kernel (read through L2).  Writes idx/w for the token (lane j < k).
template <int NPL>
__device__ void warp_topk_certified(const double *lg, const float *la, int E, int k, float coef, int H,
                                    const __nv_bfloat16 *xrow, const __nv_bfloat16 *wr, const float *bias,
                                    int *out_idx, float *out_w, unsigned long long *fallbacks,
                                    int *out_idx_smem = nullptr, unsigned long long *stamps = nullptr) {
    const int lane = threadIdx.x & 31;
    auto mark = [&](int i) {
        if (stamps && lane == 0) {
            unsigned long long t;
            asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
            stamps[i] = t;
        }
    };
    mark(0);
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
    mark(1);
    unsigned sel = 0;
    int my_e = 0;
    double my_v = -INFINITY, my_m = 0.0;
    warp_select<NPL>(v, m, E, k, sel, my_e, my_v, my_m);
    mark(2);

    // certification: the selected set and its order are decided by more than the bounds
    const bool in_k = lane < k;
    const double lower = in_k ? my_v - my_m : INFINITY;
    double msel = dkey_value(warp_min_key(dkey(lower)));
    const double next_upper = __shfl_down_sync(0xffffffffu, my_v + my_m, 1);
    const bool pair_ok = !(lane + 1 < k) || (lower > next_upper);
    bool ordered = __all_sync(0xffffffffu, pair_ok);
    double omax = -INFINITY;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        if (lane + 32 * i < E && !(sel >> i & 1u)) omax = fmax(omax, v[i] + m[i]);
    omax = dkey_value(warp_max_key(dkey(omax)));
    mark(3);
    const bool fell_back = !(ordered && omax < msel);

    // Not certified: every expert whose interval reaches the lowest selected lower bound is
    // a candidate (the rest are beaten by k experts and drop out).  Level 1 recomputes the
    // candidates with the whole warp to within a tiny bound of the oracle's own values and
    // certifies again; level 2, for what is still unresolved (near-exact ties), takes the
    // oracle's sequential sums themselves, which warp_select then orders exactly (value
    // descending, index ascending).
    for (int level = 1; level <= 2 && !(ordered && omax < msel); ++level) {
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            const bool cand = e < E && v[i] + m[i] >= msel;
            if (level == 1) {
                unsigned bal = __ballot_sync(0xffffffffu, cand);
                double nv = -INFINITY, nm = 0.0;
                while (bal) {
                    const int src = __ffs(bal) - 1;
                    bal &= bal - 1;
                    const int ce = src + 32 * i;
                    double cm;
                    const double cv = precise_logit_warp(xrow, wr + (size_t)ce * H, H, bias ? bias + ce : nullptr, cm);
                    if (lane == src) { nv = cv; nm = cm; }
                }
                v[i] = cand ? nv : -INFINITY;
                m[i] = cand ? nm : 0.0;
            } else {
                v[i] = cand ? exact_logit(xrow, wr + (size_t)e * H, H, bias ? bias + e : nullptr) : -INFINITY;
                m[i] = 0.0;
            }
        }
        sel = 0;
        warp_select<NPL>(v, m, E, k, sel, my_e, my_v, my_m);
        if (level == 2) break;
        // certify the level-1 selection
        const double lower1 = in_k ? my_v - my_m : INFINITY;
        msel = dkey_value(warp_min_key(dkey(lower1)));
        const double next_upper1 = __shfl_down_sync(0xffffffffu, my_v + my_m, 1);
        ordered = __all_sync(0xffffffffu, !(lane + 1 < k) || (lower1 > next_upper1));
        omax = -INFINITY;
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (lane + 32 * i < E && !(sel >> i & 1u)) omax = fmax(omax, v[i] + m[i]);
        omax = dkey_value(warp_max_key(dkey(omax)));
    }
    if (fell_back && lane == 0 && fallbacks) atomicAdd(fallbacks, 1ull);

    mark(4);
    const float s = in_k ? router_score((float)my_v) : 0.0f;
    const float ssum = warp_sum(s);
    if (in_k) {
        out_idx[lane] = my_e;
        out_w[lane] = ssum > 0.0f ? s / ssum : 1.0f / k;
        if (out_idx_smem) out_idx_smem[lane] = my_e;
    }
    mark(5);
}

// Warp-wide selection of the k best (value desc, index asc) of the values in shared memory
// sv[0..E) (entry e belongs to lane e % 32); lane j < k receives slot j's expert, value
// and bound (sm).  sel marks this lane's taken entries (bit i: expert lane + 32 i).
template <int NPL>
__device__ __forceinline__ void smem_select(const double *sv, const double *sm, int E, int k, unsigned &sel, int &my_e,
                                            double &my_v, double &my_m) {
    const int lane = threadIdx.x & 31;
    sel = 0;
    for (int j = 0; j < k; ++j) {
        unsigned long long bk = 0ull;
        int bi = -1;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !(sel >> i & 1u)) {
                const unsigned long long key = dkey(sv[e]);
                if (bi < 0 || key > bk) { bk = key; bi = i; }
            }
        }
        const unsigned long long best = warp_max_key(bi >= 0 ? bk : 0ull);
        const unsigned win = __reduce_min_sync(0xffffffffu, (bi >= 0 && bk == best) ? (unsigned)(lane + 32 * bi) : 0xffffffffu);
        const int be = win < (unsigned)E ? (int)win : 0;   // only reachable with non-finite logits
        if ((be & 31) == lane) sel |= 1u << (be >> 5);
        if (lane == j) { my_e = be; my_v = sv[be]; my_m = sm[be]; }
    }
}

// The exact selection of a token that the fast pass could not certify, with the logits and
// bounds in shared memory (sv, sm), written by this warp: every expert whose interval
// reaches the lowest selected lower bound (msel) is a candidate; level 1 recomputes the
// candidates with the whole warp to within a tiny bound of the oracle's own values and
// certifies again; level 2 takes the oracle's sequential sums for what is still open, which
// the selection then orders exactly.  Keeps no per-expert values in registers.
template <int NPL>
__device__ void smem_topk_exact(double *sv, double *sm, int E, int k, double msel, int H,
                                const __nv_bfloat16 *xrow, const __nv_bfloat16 *wr, const float *bias, unsigned &sel,
                                int &my_e, double &my_v, double &my_m) {
    const int lane = threadIdx.x & 31;
    const bool in_k = lane < k;
    for (int level = 1; level <= 2; ++level) {
        unsigned cand = 0;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            if (e < E && sv[e] + sm[e] >= msel) cand |= 1u << i;
        }
        __syncwarp();
        // a rolled loop: the logit evaluations inside are large code, and this path is rare
#pragma unroll 1
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            if (level == 1) {
                unsigned bal = __ballot_sync(0xffffffffu, (cand >> i) & 1u);
                while (bal) {
                    const int src = __ffs(bal) - 1;
                    bal &= bal - 1;
                    const int ce = src + 32 * i;
                    double cm;
                    const double cv = precise_logit_warp(xrow, wr + (size_t)ce * H, H, bias ? bias + ce : nullptr, cm);
                    if (lane == src) { sv[ce] = cv; sm[ce] = cm; }
                }
            } else if ((cand >> i) & 1u) {
                sv[e] = exact_logit(xrow, wr + (size_t)e * H, H, bias ? bias + e : nullptr);
                sm[e] = 0.0;
            }
            if (e < E && !((cand >> i) & 1u)) { sv[e] = -INFINITY; sm[e] = 0.0; }
        }
        __syncwarp();
        smem_select<NPL>(sv, sm, E, k, sel, my_e, my_v, my_m);
        if (level == 2) break;
        const double lower = in_k ? my_v - my_m : INFINITY;
        msel = dkey_value(warp_min_key(dkey(lower)));
        const double next_upper = __shfl_down_sync(0xffffffffu, my_v + my_m, 1);
        const bool ordered = __all_sync(0xffffffffu, !(lane + 1 < k) || (lower > next_upper));
        double omax = -INFINITY;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !(sel >> i & 1u)) omax = fmax(omax, sv[e] + sm[e]);
        }
        omax = dkey_value(warp_max_key(dkey(omax)));
        if (ordered && omax < msel) break;
        __syncwarp();
    }
}

// Faster level 0 for short latency: the selection runs on 32-bit keys -- the logit rounded
// to fp32 in an order-preserving encoding, its lowest 8 bits replaced by 255 - e (so equal
// keys rank the lower expert first, and every key is distinct) -- with one warp-wide max per
// slot.  That order may differ from the exact one only between logits closer than the
// rounding, and the certification that follows (the same as warp_topk_certified's, on the
// fp64 logits and bounds) rejects any such order; a token that is not certified goes
// through the exact selection (smem_topk_exact).  E <= 256.
// The fp64 logits and their bounds wait in shared memory (sv, sm: E entries each, this
// warp's own) while the selection keeps only the keys in registers.
template <int NPL>
__device__ void warp_topk_fast(const double *lg, const float *la, int E, int k, float coef, int H,
                               const __nv_bfloat16 *xrow, const __nv_bfloat16 *wr, const float *bias, int *out_idx,
                               float *out_w, unsigned long long *fallbacks, double *sv, double *sm,
                               unsigned long long *stamps = nullptr) {
    const int lane = threadIdx.x & 31;
    auto mark = [&](int i) {
        if (stamps && lane == 0) {
            unsigned long long t;
            asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
            stamps[i] = t;
        }
    };
    mark(0);
    const uint32_t svs = smem_u32(sv), sms = smem_u32(sm);   // shared-memory addresses of the scratch
    uint32_t key[NPL];
    {
        double v[NPL];
        float a[NPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            v[i] = e < E ? __ldcg(lg + e) : 0.0;
            a[i] = e < E ? __ldcg(la + e) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            if (e < E) {
                sts_f64(svs + 8u * (uint32_t)e, v[i]);
                sts_f64(sms + 8u * (uint32_t)e, margin_of(v[i], a[i], coef, H));
                const uint32_t u = __float_as_uint((float)v[i]);
                const uint32_t ok = (u >> 31) ? ~u : (u | 0x80000000u);
                key[i] = (ok & 0xFFFFFF00u) | (uint32_t)(255 - e);
            } else {
                key[i] = 0u;
            }
        }
    }
    mark(1);
    // k rounds, each taking the warp's best remaining key (keys are distinct).  A small
    // loop rather than a sorting network: this code runs once per launch on one warp, and
    // its cost is mostly fetching its instructions.
    int my_e = 0;
    unsigned sel = 0;   // bit i: expert lane + 32 i is selected
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
        uint32_t mk = key[0];
#pragma unroll
        for (int i = 1; i < NPL; ++i) mk = max(mk, key[i]);
        const uint32_t best = __reduce_max_sync(0xffffffffu, mk);
        const int be = 255 - (int)(best & 0xFFu);
#pragma unroll
        for (int i = 0; i < NPL; ++i)
            if (key[i] == best) key[i] = 0u;
        if (lane == j) my_e = be;
        if ((be & 31) == lane) sel |= 1u << (be >> 5);
    }
    mark(2);
    // certification on the fp64 logits and bounds of the selection
    __syncwarp();
    const bool in_k = lane < k;
    const double my_v = in_k ? lds_f64(svs + 8u * (uint32_t)my_e) : -INFINITY;
    const double my_m = in_k ? lds_f64(sms + 8u * (uint32_t)my_e) : 0.0;
    const double lower = in_k ? my_v - my_m : INFINITY;
    const double msel = dkey_value(warp_min_key(dkey(lower)));
    const double next_upper = __shfl_down_sync(0xffffffffu, my_v + my_m, 1);
    const bool ordered = __all_sync(0xffffffffu, !(lane + 1 < k) || (lower > next_upper));
    double omax = -INFINITY;
#pragma unroll 1
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !(sel >> i & 1u)) omax = fmax(omax, lds_f64(svs + 8u * (uint32_t)e) + lds_f64(sms + 8u * (uint32_t)e));
    }
    omax = dkey_value(warp_max_key(dkey(omax)));
    mark(3);
    double fv = my_v;
    if (!(ordered && omax < msel)) {
        unsigned sel2;
        int e2 = 0;
        double v2 = -INFINITY, m2 = 0.0;
        __syncwarp();
        smem_topk_exact<NPL>(sv, sm, E, k, msel, H, xrow, wr, bias, sel2, e2, v2, m2);
        my_e = e2;
        fv = v2;
        if (lane == 0 && fallbacks) atomicAdd(fallbacks, 1ull);
    }
    mark(4);
    const float s = in_k ? router_score((float)fv) : 0.0f;
    const float ssum = warp_sum(s);
    if (in_k) {
        out_idx[lane] = my_e;
        out_w[lane] = ssum > 0.0f ? s / ssum : 1.0f / k;
    }
    mark(5);
}

// ---------------------------------------------------------------------------------------
// Decode router row: one warp computes router row e for all T tokens (pairs of exact
// products rounded once in fp32, then accumulated in fp64), with A = sum |x_i Wr_i|.
// The row is fetched 4096 inputs at a time (sixteen 16-byte loads in flight per lane).
template <int TT, bool XS = false>
__device__ void router_row_warp(const __nv_bfloat16 *__restrict__ x, int T, int H, const __nv_bfloat16 *__restrict__ wr,
                                const float *bias, int e, int E, double *logits, float *labs) {
    const int lane = threadIdx.x & 31;
    const __nv_bfloat16 *row = wr + (size_t)e * H;
    for (int t0 = 0; t0 < T; t0 += TT) {
        const int nt = min(TT, T - t0);
        double acc[TT];
        float ab[TT];
#pragma unroll
        for (int t = 0; t < TT; ++t) { acc[t] = 0.0; ab[t] = 0.0f; }
        for (int kb = 0; kb < H; kb += 4096) {
            uint4 wv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int k = kb + i * 256 + lane * 8;
                wv[i] = k < H ? ld_stream_v4(row + k) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                if (t < nt) {
                    const __nv_bfloat16 *xr = x + (size_t)(t0 + t) * H;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int k = kb + i * 256 + lane * 8;
                        if (k < H) {
                            const uint4 xv = XS ? *reinterpret_cast<const uint4 *>(xr + k)
                                                : __ldg(reinterpret_cast<const uint4 *>(xr + k));
                            const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
                            const uint32_t ws[4] = {wv[i].x, wv[i].y, wv[i].z, wv[i].w};
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                const float x0 = bf16lo(xs[q]), x1 = bf16hi(xs[q]);
                                const float w0 = bf16lo(ws[q]), w1 = bf16hi(ws[q]);
                                const float p = __fmaf_rn(x1, w1, __fmul_rn(x0, w0));
                                acc[t] += (double)p;
                                ab[t] = __fmaf_rn(fabsf(x0), fabsf(w0), __fmaf_rn(fabsf(x1), fabsf(w1), ab[t]));
                            }
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            const double sum = warp_sum(acc[t]);
            const float a = warp_sum(ab[t]);
            if (lane == 0 && t < nt) {
                logits[(size_t)(t0 + t) * E + e] = bias ? __dadd_rn(sum, (double)bias[e]) : sum;
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

// Prefill router: CTA tile of 64 tokens x 32 experts, 128 threads, each thread 4 tokens x
// 4 experts in registers.  Every product of two bf16 values is exact in fp32; a thread sums
// each run of 32 products in fp32 (FMA, starting from zero) and adds the run's sum to an fp64
// accumulator, so a logit's error is at most gamma_31 * sum_i |x_i w_i| (gamma_n = n u /
// (1 - n u), u = 2^-24) plus the fp64 rounding, and sum_i |x_i w_i| <= ||x_t|| * ||Wr_e||
// (Cauchy-Schwarz).  The token norms are summed in fp64 while the tiles are staged.
// Tiles are staged through registers into two shared buffers: the global loads of the next
// 32-wide K chunk are in flight while the current one is multiplied.
constexpr int PR_T = 64, PR_E = 32, PR_K = 32;
constexpr float BOUND_CHUNK32 = 1.85e-6f;   // gamma_31 = 1.8477e-6, rounded up
__global__ void __launch_bounds__(128) router_gemm_kernel(const __nv_bfloat16 *__restrict__ x, int T, int H,
                                                          const __nv_bfloat16 *__restrict__ wr, int E,
                                                          const float *__restrict__ bias,
                                                          const float *__restrict__ wr_norm, double *logits,
                                                          float *labs) {
    __shared__ __align__(16) float xs[2][PR_K][PR_T + 4];   // [k][token]
    __shared__ __align__(16) float ws[2][PR_K][PR_E + 4];   // [k][expert]
    __shared__ double xn2s[2][PR_T];
    const int t0 = blockIdx.x * PR_T, e0 = blockIdx.y * PR_E;
    const int tid = threadIdx.x;
    // staging: token lt (16 K of the chunk, half kh), expert le (8 K of the chunk, quarter kq)
    const int lt = tid & 63, kh = tid >> 6, le = tid & 31, kq = tid >> 5;
    const bool tv = t0 + lt < T, ev = e0 + le < E;
    const uint4 *xp = reinterpret_cast<const uint4 *>(x + (size_t)(tv ? t0 + lt : 0) * H) + kh * 2;
    const uint4 *wp = reinterpret_cast<const uint4 *>(wr + (size_t)(ev ? e0 + le : 0) * H) + kq;
    // compute: tokens 4 tq .. 4 tq + 3, experts 4 eq .. 4 eq + 3
    const int tq = tid >> 3, eq = tid & 7;
    float c[4][4];
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) { c[i][j] = 0.0f; acc[i][j] = 0.0; }
    double xn2 = 0.0;
    uint4 rx0 = make_uint4(0, 0, 0, 0), rx1 = rx0, rw = rx0;
    auto gload = [&](int k0) {
        if (tv) {
            rx0 = __ldg(xp + k0 / 8);
            rx1 = __ldg(xp + k0 / 8 + 1);
        }
        if (ev) rw = __ldg(wp + k0 / 8);
    };
    auto stage = [&](int b) {
        const uint32_t vx[8] = {rx0.x, rx0.y, rx0.z, rx0.w, rx1.x, rx1.y, rx1.z, rx1.w};
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float lo = bf16lo(vx[q]), hi = bf16hi(vx[q]);
            xs[b][kh * 16 + 2 * q][lt] = lo;
            xs[b][kh * 16 + 2 * q + 1][lt] = hi;
            xn2 = fma((double)lo, (double)lo, xn2);
            xn2 = fma((double)hi, (double)hi, xn2);
        }
        const uint32_t vw[4] = {rw.x, rw.y, rw.z, rw.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            ws[b][kq * 8 + 2 * q][le] = bf16lo(vw[q]);
            ws[b][kq * 8 + 2 * q + 1][le] = bf16hi(vw[q]);
        }
    };
    gload(0);
    stage(0);
    __syncthreads();
    for (int k0 = 0; k0 < H; k0 += PR_K) {
        const int b = (k0 / PR_K) & 1;
        const bool more = k0 + PR_K < H;
        if (more) gload(k0 + PR_K);
#pragma unroll
        for (int kk = 0; kk < PR_K; ++kk) {
            const float4 a = *reinterpret_cast<const float4 *>(&xs[b][kk][4 * tq]);
            const float4 w = *reinterpret_cast<const float4 *>(&ws[b][kk][4 * eq]);
            const float av[4] = {a.x, a.y, a.z, a.w}, wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) c[i][j] = __fmaf_rn(av[i], wv[j], c[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) { acc[i][j] += (double)c[i][j]; c[i][j] = 0.0f; }
        if (more) stage(b ^ 1);
        __syncthreads();
    }
    xn2s[kh][lt] = xn2;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int tl = 4 * tq + i, t = t0 + tl;
        if (t >= T) continue;
        const float xn = (float)sqrt(xn2s[0][tl] + xn2s[1][tl]) * (1.0f + 1e-6f);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int e = e0 + 4 * eq + j;
            if (e >= E) continue;
            const double s = acc[i][j];
            logits[(size_t)t * E + e] = bias ? __dadd_rn(s, (double)bias[e]) : s;
            labs[(size_t)t * E + e] = xn * wr_norm[e];
        }
    }
}

// Prefill top-k + per-64-token-block counts and masks: one CTA (16 warps) per 64 tokens.
constexpr int TOPK_THREADS = 512;
template <int NPL>
__global__ void __launch_bounds__(TOPK_THREADS) topk_block_kernel(const double *logits, const float *labs, int T, int E,
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
    for (int tt = warp; tt < nt; tt += (int)(blockDim.x >> 5)) {
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
