// decode.cuh -- the batched-GEMV path of the layer as one persistent kernel.
//
// Work is cut into units handed out in dependency order from one atomic counter; a CTA
// that takes a unit whose inputs are not ready waits (bounded) on a completion counter.
// Units are dispensed in the order below and each waits only on units dispensed before
// it, so the schedule cannot deadlock.
//   R   router rows (fp64-accumulated logits); the CTA that completes the last R unit runs
//       the certified top-k of every token and the permutation, then publishes them.
//   X   x -> int16 per 256-block (one unit per token).
//   SG  shared-expert gate/up rows + SwiGLU (16 rows of each per unit).
//   G   routed gate/up + SwiGLU: (active expert slot, 32 rows of I) per unit; lane = row,
//       integer dot products of the 2-bit quants with the int16 activations (dp2a), the
//       4-bit scales and mins applied in integers, fp16 d/dmin and the x scale in fp32.
//   SD  shared-expert down rows (16 per unit).
//   D   routed down: (active slot, 128 rows of H) per unit; h of the slot's tokens is
//       quantised to int16 per 256-block in shared memory.
// The last unit (SD or D) to finish a 128-row range of H writes y for that range:
// y = sum_j w_j o_j + S, summed in slot order.  Q2_K bytes stream from HBM once per call.
#pragma once
#include "common.cuh"
#include "router.cuh"

namespace ds4 {

constexpr int DEC_WARPS = 8;
constexpr int DEC_THREADS = DEC_WARPS * 32;
#ifndef DS4_TT_DENSE
#define DS4_TT_DENSE 4
#endif
#ifndef DS4_TT_Q
#define DS4_TT_Q 4
#endif
constexpr int TT_DENSE = DS4_TT_DENSE;   // tokens per pass in the dense GEMVs
constexpr int TT_Q = DS4_TT_Q;           // tokens per pass in the Q2_K GEMVs
constexpr int SG_ROWS = 16;    // shared gate/up rows per unit (2 gate + 2 up per warp)
constexpr int SD_ROWS = 16;    // shared down rows per unit (2 per warp)
constexpr int SD_PER_RANGE = 128 / SD_ROWS;
constexpr int MAX_DECODE_T = 32;   // the decode permutation ranks T*k <= 512 pairs in shared memory

// Completion counters of one call (zeroed before every launch).
struct DecodeCtl {
    unsigned next_unit;
    unsigned router_done;
    unsigned routing_ready;
    unsigned xq_done;
    unsigned sg_done;
    unsigned abort;
    unsigned exited;
    unsigned pad;
    unsigned exp_done[MAX_EXPERTS];
    unsigned rg_done[16384 / 128];
};

struct DecodeArgs {
    int T, H, E, k, I, Is;
    const __nv_bfloat16 *x;        // [T][H]
    const __nv_bfloat16 *wr;       // [E][H]
    const float *bias;             // [E] or null
    const __nv_bfloat16 *sg, *su;  // [Is][H]
    const __nv_bfloat16 *sd;       // [H][Is]
    const uint8_t *gate, *up, *down;  // tiled Q2_K, expert-major
    size_t gu_bytes, d_bytes;         // bytes per expert matrix
    double *logits;
    float *labs;
    RouteOut ro;
    int16_t *xq;
    float *xscale;
    int *xsum;
    float *hs;   // [T][Is]
    float *h;    // [P][I]
    float *o;    // [P][H]
    float *s;    // [T][H]
    float *y;    // [T][H]
    DecodeCtl *ctl;
    int *status;
    // unit map: [0,uX) R, [uX,uSG) X, [uSG,uG) SG, [uG,uSD) G, [uSD,uD) SD, [uD,uEnd) D
    int uX, uSG, uG, uSD, uD, uEnd;
    int max_act;
    int routing_preset;   // routing comes from an earlier launch (no counter wait)
    int routing_pdl;      // that launch is this kernel's programmatic prerequisite: wait on it
    unsigned long long *trace;   // optional: 4 words per unit (unit | sm << 32, fetch, ready, end ns)
    size_t trace_stamps;         // word offset of the routing-step stamps in trace
};

__device__ __forceinline__ unsigned long long gtimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ unsigned smid() {
    unsigned r;
    asm volatile("mov.u32 %0, %smid;" : "=r"(r));
    return r;
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Thread 0 waits until *p >= target (bounded); false on timeout or abort.
__device__ bool wait_counter(const unsigned *p, unsigned target, DecodeCtl *ctl, int *status) {
    for (long long it = 0;; ++it) {
        if (ld_acquire(p) >= target) return true;
        if (ld_acquire(&ctl->abort)) return false;
        if (it > (1ll << 22)) {
            set_status(status, ST_ETIMEOUT);
            atomicExch(&ctl->abort, 1u);
            return false;
        }
        __nanosleep(it < 64 ? 32 : 256);
    }
}

// CTA-wide: all threads learn whether the wait succeeded.
__device__ bool cta_wait(const unsigned *p, unsigned target, DecodeCtl *ctl, int *status, int *s_ok,
                         unsigned long long *t_ready) {
    if (threadIdx.x == 0) {
        *s_ok = (target == 0u || wait_counter(p, target, ctl, status)) ? 1 : 0;
        *t_ready = gtimer();
    }
    __syncthreads();
    const bool ok = *s_ok != 0;
    __syncthreads();
    return ok;
}

// x -> int16 per 256-block: xq = rint(x * 32767 / amax), xscale = amax / 32767,
// xsum[sub-block] = sum of the 16 xq of each sub-block.  One warp per (token, block).
__device__ void quantize_x_warp(const __nv_bfloat16 *x, int H, int t, int blk, int16_t *xq, float *xscale, int *xsum) {
    const int lane = threadIdx.x & 31;
    const int i0 = blk * QK + lane * 8;
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)t * H + i0));
    const float f[8] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y),
                        bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w)};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = warp_max(amax);
    const float inv = amax > 0.0f ? 32767.0f / amax : 0.0f;
    int q[8], s = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        q[i] = max(-32767, min(32767, __float2int_rn(f[i] * inv)));
        s += q[i];
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    uint4 o;
    o.x = (uint32_t)(q[0] & 0xFFFF) | ((uint32_t)q[1] << 16);
    o.y = (uint32_t)(q[2] & 0xFFFF) | ((uint32_t)q[3] << 16);
    o.z = (uint32_t)(q[4] & 0xFFFF) | ((uint32_t)q[5] << 16);
    o.w = (uint32_t)(q[6] & 0xFFFF) | ((uint32_t)q[7] << 16);
    *reinterpret_cast<uint4 *>(xq + (size_t)t * H + i0) = o;
    if ((lane & 1) == 0) xsum[(size_t)t * (H / 16) + blk * 16 + lane / 2] = s;
    if (lane == 0) xscale[(size_t)t * (H / QK) + blk] = amax / 32767.0f;
}

// Same quantisation for fp32 input held in global memory, writing to shared memory.
__device__ void quantize_f32_warp(const float *src, int16_t *q_out, int *sum_out, float *scale_out) {
    const int lane = threadIdx.x & 31;
    const float4 v0 = __ldcg(reinterpret_cast<const float4 *>(src + lane * 8));
    const float4 v1 = __ldcg(reinterpret_cast<const float4 *>(src + lane * 8 + 4));
    const float f[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = warp_max(amax);
    const float inv = amax > 0.0f ? 32767.0f / amax : 0.0f;
    int q[8], s = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        q[i] = max(-32767, min(32767, __float2int_rn(f[i] * inv)));
        s += q[i];
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    uint4 o;
    o.x = (uint32_t)(q[0] & 0xFFFF) | ((uint32_t)q[1] << 16);
    o.y = (uint32_t)(q[2] & 0xFFFF) | ((uint32_t)q[3] << 16);
    o.z = (uint32_t)(q[4] & 0xFFFF) | ((uint32_t)q[5] << 16);
    o.w = (uint32_t)(q[6] & 0xFFFF) | ((uint32_t)q[7] << 16);
    *reinterpret_cast<uint4 *>(q_out + lane * 8) = o;
    if ((lane & 1) == 0) sum_out[lane / 2] = s;
    if (lane == 0) *scale_out = amax / 32767.0f;
}

// ---------------------------------------------------------------------------------------
// Dense bf16 GEMVs (lanes along K, 16-byte loads, two K steps in flight per row).

// Shared gate/up rows r and r+1 of one warp: hs[t][r] = silu(g) u for every token.
__device__ void sg_warp(const DecodeArgs &a, int r) {
    const int lane = threadIdx.x & 31;
    const __nv_bfloat16 *rows[4] = {a.sg + (size_t)r * a.H, a.sg + (size_t)(r + 1) * a.H, a.su + (size_t)r * a.H,
                                    a.su + (size_t)(r + 1) * a.H};
    for (int t0 = 0; t0 < a.T; t0 += TT_DENSE) {
        const int nt = min(TT_DENSE, a.T - t0);
        float acc[4][TT_DENSE];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int t = 0; t < TT_DENSE; ++t) acc[q][t] = 0.0f;
        for (int k0 = lane * 8; k0 < a.H; k0 += 512) {
            const bool two = k0 + 256 < a.H;
            uint4 w0[4], w1[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                w0[q] = ld_stream_v4(rows[q] + k0);
                w1[q] = two ? ld_stream_v4(rows[q] + k0 + 256) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int t = 0; t < TT_DENSE; ++t) {
                if (t < nt) {
                    const __nv_bfloat16 *xr = a.x + (size_t)(t0 + t) * a.H + k0;
                    const uint4 xa = __ldg(reinterpret_cast<const uint4 *>(xr));
                    const uint4 xb = two ? __ldg(reinterpret_cast<const uint4 *>(xr + 256)) : make_uint4(0, 0, 0, 0);
                    const uint32_t xs[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t ws[8] = {w0[q].x, w0[q].y, w0[q].z, w0[q].w, w1[q].x, w1[q].y, w1[q].z, w1[q].w};
                        float s = acc[q][t];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            s = fmaf(bf16lo(xs[i]), bf16lo(ws[i]), s);
                            s = fmaf(bf16hi(xs[i]), bf16hi(ws[i]), s);
                        }
                        acc[q][t] = s;
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT_DENSE; ++t) {
            const float g0 = warp_sum(acc[0][t]), g1 = warp_sum(acc[1][t]);
            const float u0 = warp_sum(acc[2][t]), u1 = warp_sum(acc[3][t]);
            if (lane == 0 && t < nt) {
                a.hs[(size_t)(t0 + t) * a.Is + r] = silu(g0) * u0;
                a.hs[(size_t)(t0 + t) * a.Is + r + 1] = silu(g1) * u1;
            }
        }
    }
}

// Shared down rows c and c+1 of one warp: s[t][c] = W_sd[c,:] . hs[t,:].
__device__ void sd_warp(const DecodeArgs &a, int c) {
    const int lane = threadIdx.x & 31;
    const __nv_bfloat16 *rows[2] = {a.sd + (size_t)c * a.Is, a.sd + (size_t)(c + 1) * a.Is};
    for (int t0 = 0; t0 < a.T; t0 += TT_DENSE) {
        const int nt = min(TT_DENSE, a.T - t0);
        float acc[2][TT_DENSE];
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int t = 0; t < TT_DENSE; ++t) acc[q][t] = 0.0f;
        for (int k0 = lane * 8; k0 < a.Is; k0 += 512) {
            const bool two = k0 + 256 < a.Is;
            uint4 w0[2], w1[2];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                w0[q] = ld_stream_v4(rows[q] + k0);
                w1[q] = two ? ld_stream_v4(rows[q] + k0 + 256) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int t = 0; t < TT_DENSE; ++t) {
                if (t < nt) {
                    const float *hp = a.hs + (size_t)(t0 + t) * a.Is + k0;
                    float hv[16];
                    const float4 h0 = __ldcg(reinterpret_cast<const float4 *>(hp));
                    const float4 h1 = __ldcg(reinterpret_cast<const float4 *>(hp + 4));
                    hv[0] = h0.x; hv[1] = h0.y; hv[2] = h0.z; hv[3] = h0.w;
                    hv[4] = h1.x; hv[5] = h1.y; hv[6] = h1.z; hv[7] = h1.w;
                    if (two) {
                        const float4 h2 = __ldcg(reinterpret_cast<const float4 *>(hp + 256));
                        const float4 h3 = __ldcg(reinterpret_cast<const float4 *>(hp + 260));
                        hv[8] = h2.x; hv[9] = h2.y; hv[10] = h2.z; hv[11] = h2.w;
                        hv[12] = h3.x; hv[13] = h3.y; hv[14] = h3.z; hv[15] = h3.w;
                    } else {
#pragma unroll
                        for (int i = 8; i < 16; ++i) hv[i] = 0.0f;
                    }
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        const uint32_t ws[8] = {w0[q].x, w0[q].y, w0[q].z, w0[q].w, w1[q].x, w1[q].y, w1[q].z, w1[q].w};
                        float s = acc[q][t];
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            s = fmaf(hv[2 * i], bf16lo(ws[i]), s);
                            s = fmaf(hv[2 * i + 1], bf16hi(ws[i]), s);
                        }
                        acc[q][t] = s;
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT_DENSE; ++t) {
            const float s0 = warp_sum(acc[0][t]), s1 = warp_sum(acc[1][t]);
            if (lane == 0 && t < nt) {
                a.s[(size_t)(t0 + t) * a.H + c] = s0;
                a.s[(size_t)(t0 + t) * a.H + c + 1] = s1;
            }
        }
    }
}

// ---------------------------------------------------------------------------------------
// Integer dot of one Q2_K block row (held by this lane) with one token's int16 block.
//  qs[4]: the row's four 16-byte quant chunks; sc: its 16 scale bytes;
//  xq: the token's 256 int16 values of this block (16-byte aligned), xs: its 16 sub-block sums.
//  Returns isc = sum_sb scale_sb * dot_sb and imn = sum_sb min_sb * xsum_sb.
__device__ __forceinline__ void q2k_block_dot(const uint4 (&qs)[4], const uint4 &sc, const int16_t *xq, const int *xs,
                                              int &isc, int &imn) {
    const uint32_t scw[4] = {sc.x, sc.y, sc.z, sc.w};
    isc = 0;
    imn = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t w[4] = {qs[c].x, qs[c].y, qs[c].z, qs[c].w};
        const int hh = c >> 1, l0 = (c & 1) * 16;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int sb = 8 * hh + 2 * j + (c & 1);
            const int base = 128 * hh + 32 * j + l0;
            const uint4 xa = *reinterpret_cast<const uint4 *>(xq + base);
            const uint4 xb = *reinterpret_cast<const uint4 *>(xq + base + 8);
            // the quants of plane j stay in place (byte value q * 4^j); the dot is divided by
            // 4^j afterwards, exactly, since every term is a multiple of 4^j
            const uint32_t mask = 0x03030303u << (2 * j);
            const uint32_t q0 = w[0] & mask, q1 = w[1] & mask, q2 = w[2] & mask, q3 = w[3] & mask;
            int d = dp2a_lo((int)xa.x, q0, 0);
            d = dp2a_hi((int)xa.y, q0, d);
            d = dp2a_lo((int)xa.z, q1, d);
            d = dp2a_hi((int)xa.w, q1, d);
            d = dp2a_lo((int)xb.x, q2, d);
            d = dp2a_hi((int)xb.y, q2, d);
            d = dp2a_lo((int)xb.z, q3, d);
            d = dp2a_hi((int)xb.w, q3, d);
            d >>= 2 * j;
            const uint32_t sbyte = (scw[sb >> 2] >> (8 * (sb & 3))) & 0xFFu;
            isc += (int)(sbyte & 0xFu) * d;
            imn += (int)(sbyte >> 4) * xs[sb];
        }
    }
}

struct Q2Row {
    uint4 qs[4];
    uint4 sc;
    uint32_t dm;
};

__device__ __forceinline__ void load_q2_row(Q2Row &r, const uint8_t *tile, int lane) {
#pragma unroll
    for (int c = 0; c < 4; ++c) r.qs[c] = ld_stream_v4(tile + TILE_QS + c * 512 + lane * 16);
    r.sc = ld_stream_v4(tile + TILE_SC + lane * 16);
    r.dm = ld_stream_u32(tile + TILE_DM + lane * 4);
}

// acc[t] += sum over the blocks b = b0, b0 + bstep, ... < nb of one Q2_K row (lane = row)
// dotted with token t's int16 activations; the next block's bytes are loaded while the
// current one is computed.
template <class XQ, class XS, class SC>
__device__ __forceinline__ void q2_rows_dot(const uint8_t *rowgroup, int nb, int b0, int bstep, int nt, XQ xq_of,
                                            XS xs_of, SC sc_of, float (&acc)[TT_Q]) {
    const int lane = threadIdx.x & 31;
    if (b0 >= nb) return;
    Q2Row cur, nxt;
    load_q2_row(cur, rowgroup + (size_t)b0 * TILE_BYTES, lane);
    for (int b = b0; b < nb; b += bstep) {
        const bool more = b + bstep < nb;
        if (more) load_q2_row(nxt, rowgroup + (size_t)(b + bstep) * TILE_BYTES, lane);
        const float d = h2f(cur.dm), dmin = h2f(cur.dm >> 16);
#pragma unroll
        for (int t = 0; t < TT_Q; ++t) {
            if (t < nt) {
                int isc, imn;
                q2k_block_dot(cur.qs, cur.sc, xq_of(t, b), xs_of(t, b), isc, imn);
                acc[t] = fmaf(sc_of(t, b), fmaf(d, (float)isc, -dmin * (float)imn), acc[t]);
            }
        }
        if (more) cur = nxt;
    }
}

// ---------------------------------------------------------------------------------------
struct DecSmem {
    float red[2][4][TT_Q][32];
    int s_ok, s_last, s_unit, s_next, s_routed, s_n_act;
    unsigned long long s_t_fetch, s_t_ready;
    int s_cnt[MAX_EXPERTS];
    unsigned long long s_mask[MAX_EXPERTS];
    int s_off[MAX_EXPERTS + 1];
    int s_idx[MAX_DECODE_T * MAX_TOPK];
    int s_sorted[MAX_DECODE_T * MAX_TOPK];
    int r_act[MAX_EXPERTS];        // cached routing: active experts and their pair offsets
    int r_off[MAX_EXPERTS + 1];
};

__device__ void combine_range(const DecodeArgs &a, int rg4) {
    for (int i = threadIdx.x; i < a.T * 128; i += blockDim.x) {
        const int t = i >> 7, row = rg4 * 128 + (i & 127);
        float acc = 0.0f;
        for (int j = 0; j < a.k; ++j) {
            const int p = __ldcg(a.ro.inv_pos + (size_t)t * a.k + j);
            acc = fmaf(__ldcg(a.ro.topk_w + (size_t)t * a.k + j), __ldcg(a.o + (size_t)p * a.H + row), acc);
        }
        if (a.Is > 0) acc += __ldcg(a.s + (size_t)t * a.H + row);
        a.y[(size_t)t * a.H + row] = acc;
    }
}

// Count a finished unit of a 128-row range; the last one (of max_act routed + the shared
// ones) writes y for the range.
__device__ void finish_range(const DecodeArgs &a, DecSmem &sm, int rg4) {
    __threadfence();
    __syncthreads();
    const unsigned target = (unsigned)(a.max_act + (a.Is > 0 ? SD_PER_RANGE : 0));
    if (threadIdx.x == 0) sm.s_last = (atomicAdd(&a.ctl->rg_done[rg4], 1u) == target - 1);
    __syncthreads();
    if (sm.s_last) {
        __threadfence();
        combine_range(a, rg4);
    }
    __syncthreads();
}

// Trace layout: 4 words per unit (or per routing CTA), then 32 stamp words of the routing
// step at trace_stamps.
__device__ __forceinline__ void stamp(const DecodeArgs &a, int slot) {
    if (a.trace && threadIdx.x == 0) a.trace[a.trace_stamps + slot] = gtimer();
}

// Top-k of every token (one warp per token), then the permutation for up to 64 tokens:
// each (token, slot) pair is ranked by (expert, token) against all pairs, the expert
// offsets come from a binary search in the sorted experts, and the active list from the
// first pair of each expert.
template <int NPL>
__device__ void topk_and_permute(const DecodeArgs &a, DecSmem &sm) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    stamp(a, 0);
    for (int t = warp; t < a.T; t += (int)(blockDim.x >> 5))
        warp_topk_certified<NPL>(a.logits + (size_t)t * a.E, a.labs + (size_t)t * a.E, a.E, a.k, BOUND_PAIR, a.H,
                                 a.x + (size_t)t * a.H, a.wr, a.bias, a.ro.topk_idx + (size_t)t * a.k,
                                 a.ro.topk_w + (size_t)t * a.k, a.ro.fallbacks, sm.s_idx + t * a.k,
                                 (a.trace && t == 0) ? a.trace + a.trace_stamps + 8 : nullptr);
    __syncthreads();
    stamp(a, 1);
    const int P = a.T * a.k;
    int *sorted_e = sm.s_sorted;   // [P] experts in sorted pair order
    for (int p = threadIdx.x; p < P; p += blockDim.x) {
        const int t = p / a.k, j = p - t * a.k;
        const int key = sm.s_idx[p] * MAX_DECODE_T + t;
        int pos = 0;
        for (int q = 0; q < P; ++q) pos += (sm.s_idx[q] * MAX_DECODE_T + q / a.k) < key;
        sorted_e[pos] = sm.s_idx[p];
        a.ro.sorted_token[pos] = t;
        a.ro.sorted_slot[pos] = j;
        a.ro.inv_pos[p] = pos;
    }
    __syncthreads();
    stamp(a, 14);
    for (int e = threadIdx.x; e <= a.E; e += blockDim.x) {
        int lo = 0, hi = P;
        while (lo < hi) {
            const int mid = (lo + hi) >> 1;
            if (sorted_e[mid] < e) lo = mid + 1; else hi = mid;
        }
        sm.s_off[e] = lo;
        a.ro.offsets[e] = lo;
    }
    if (warp == 0) {
        int nact = 0;
        for (int c = 0; c < P; c += 32) {
            const int i = c + lane;
            const bool first = i < P && (i == 0 || sorted_e[i] != sorted_e[i - 1]);
            const unsigned bal = __ballot_sync(0xffffffffu, first);
            if (first) a.ro.active[nact + __popc(bal & ((1u << lane) - 1))] = sorted_e[i];
            nact += __popc(bal);
        }
        if (lane == 0) *a.ro.n_active = nact;
    }
    stamp(a, 2);
}

// Routing info for G and D units: waits for the published routing, then keeps the active
// experts and the pair offsets in shared memory for the rest of the launch.
__device__ bool ensure_routing(const DecodeArgs &a, DecSmem &sm) {
    if (sm.s_routed) return true;
    // routing written by the preceding launch: wait until it has completed and its writes
    // are visible (returns at once when this launch has no programmatic prerequisite)
    if (a.routing_pdl) asm volatile("griddepcontrol.wait;" ::: "memory");
    if (!cta_wait(&a.ctl->routing_ready, a.routing_preset ? 0u : 1u, a.ctl, a.status, &sm.s_ok, &sm.s_t_ready))
        return false;
    const int n_act = *(volatile int *)a.ro.n_active;
    for (int i = threadIdx.x; i < n_act; i += blockDim.x) sm.r_act[i] = __ldcg(a.ro.active + i);
    for (int i = threadIdx.x; i <= a.E; i += blockDim.x) sm.r_off[i] = __ldcg(a.ro.offsets + i);
    if (threadIdx.x == 0) {
        sm.s_n_act = n_act;
        sm.s_routed = 1;
    }
    __syncthreads();
    return true;
}

// L2 prefetch of the weights unit u will stream (issued by warp 0, one piece per lane).
// Routed units need the routing, which must already be cached in shared memory.
__device__ void prefetch_unit(const DecodeArgs &a, const DecSmem &sm, int u) {
    const int lane = threadIdx.x & 31;
    if (u < 0 || u >= a.uEnd) return;
    if (u < a.uX) {
        const int e0 = u * DEC_WARPS;
        prefetch_range_l2(a.wr + (size_t)e0 * a.H, (size_t)min(DEC_WARPS, a.E - e0) * a.H * 2, lane, 32);
    } else if (u < a.uSG) {
        return;
    } else if (u < a.uG) {
        const int r0 = (u - a.uSG) * SG_ROWS;
        const size_t bytes = (size_t)min(SG_ROWS, a.Is - r0) * a.H * 2;
        prefetch_range_l2(a.sg + (size_t)r0 * a.H, bytes, lane, 16);
        prefetch_range_l2(a.su + (size_t)r0 * a.H, bytes, lane ^ 16, 16);
    } else if (u < a.uSD) {
        if (!sm.s_routed) return;
        const int RG = a.I / TILE_ROWS, v = u - a.uG, slot = v / RG, rg = v % RG;
        if (slot >= sm.s_n_act) return;
        const int e = sm.r_act[slot], nb = a.H / QK;
        const size_t grp = (size_t)rg * nb * TILE_BYTES;
        prefetch_range_l2(a.gate + (size_t)e * a.gu_bytes + grp, (size_t)nb * TILE_BYTES, lane, 16);
        prefetch_range_l2(a.up + (size_t)e * a.gu_bytes + grp, (size_t)nb * TILE_BYTES, lane ^ 16, 16);
    } else if (u < a.uD) {
        const int c0 = (u - a.uSD) * SD_ROWS;
        prefetch_range_l2(a.sd + (size_t)c0 * a.Is, (size_t)SD_ROWS * a.Is * 2, lane, 32);
    } else {
        if (!sm.s_routed) return;
        const int RG4 = a.H / 128, v = u - a.uD, slot = v / RG4, rg4 = v % RG4;
        if (slot >= sm.s_n_act) return;
        const int e = sm.r_act[slot], nbI = a.I / QK;
        prefetch_range_l2(a.down + (size_t)e * a.d_bytes + (size_t)rg4 * 4 * nbI * TILE_BYTES,
                          (size_t)4 * nbI * TILE_BYTES, lane, 32);
    }
}

template <int NPL>
__device__ void run_unit(const DecodeArgs &a, DecSmem &sm, unsigned char *dsm_raw, int u) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    DecodeCtl *ctl = a.ctl;
    if (u < a.uX) {  // ------------------------------------------------------------ R
        const int e = u * DEC_WARPS + warp;
        if (e < a.E) router_row_warp<TT_DENSE>(a.x, a.T, a.H, a.wr, a.bias, e, a.E, a.logits, a.labs);
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) sm.s_last = (atomicAdd(&ctl->router_done, 1u) == (unsigned)a.uX - 1);
        __syncthreads();
        if (sm.s_last) {
            stamp(a, 4);
            __threadfence();
            topk_and_permute<NPL>(a, sm);
            __threadfence();
            __syncthreads();
            if (threadIdx.x == 0) atomicExch(&ctl->routing_ready, 1u);
            stamp(a, 3);
        }
    } else if (u < a.uSG) {  // ------------------------------------------------------ X
        const int t = u - a.uX;
        for (int blk = warp; blk < a.H / QK; blk += DEC_WARPS) quantize_x_warp(a.x, a.H, t, blk, a.xq, a.xscale, a.xsum);
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) atomicAdd(&ctl->xq_done, 1u);
    } else if (u < a.uG) {  // ------------------------------------------------------- SG
        const int r0 = (u - a.uSG) * SG_ROWS;
        const int r = r0 + warp * 2;
        if (r < a.Is) sg_warp(a, r);
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) atomicAdd(&ctl->sg_done, 1u);
    } else if (u < a.uSD) {  // ------------------------------------------------------ G
        const int RG = a.I / TILE_ROWS;
        const int v = u - a.uG, slot = v / RG, rg = v % RG;
        if (!ensure_routing(a, sm)) return;
        if (slot >= sm.s_n_act) return;
        const int e = sm.r_act[slot];
        const int p0 = sm.r_off[e], p1 = sm.r_off[e + 1];
        const int mat = warp >> 2, kq = warp & 3, nb = a.H / QK;
        const size_t grp = (size_t)rg * nb * TILE_BYTES;
        if (!cta_wait(&ctl->xq_done, (unsigned)a.T, ctl, a.status, &sm.s_ok, &sm.s_t_ready)) return;
        const uint8_t *rowgroup = (mat == 0 ? a.gate : a.up) + (size_t)e * a.gu_bytes + grp;
        const int H = a.H;
        int16_t *sxq = reinterpret_cast<int16_t *>(dsm_raw);                          // [TT_Q][H]
        int *sxs = reinterpret_cast<int *>(dsm_raw + TT_Q * H * 2);                    // [TT_Q][H/16]
        float *sxc = reinterpret_cast<float *>(dsm_raw + TT_Q * H * 2 + TT_Q * (H / 16) * 4);  // [TT_Q][H/256]
        for (int pc = p0; pc < p1; pc += TT_Q) {
            const int nt = min(TT_Q, p1 - pc);
            // the tokens' int16 activations, sub-block sums and scales -> shared memory
            for (int t = 0; t < nt; ++t) {
                const int tk = __ldcg(a.ro.sorted_token + pc + t);
                const uint4 *src = reinterpret_cast<const uint4 *>(a.xq + (size_t)tk * H);
                for (int i = threadIdx.x; i < H / 8; i += blockDim.x)
                    reinterpret_cast<uint4 *>(sxq + t * H)[i] = __ldcg(src + i);
                for (int i = threadIdx.x; i < H / 16; i += blockDim.x) sxs[t * (H / 16) + i] = __ldcg(a.xsum + (size_t)tk * (H / 16) + i);
                for (int i = threadIdx.x; i < nb; i += blockDim.x) sxc[t * nb + i] = __ldcg(a.xscale + (size_t)tk * nb + i);
            }
            __syncthreads();
            float acc[TT_Q];
#pragma unroll
            for (int t = 0; t < TT_Q; ++t) acc[t] = 0.0f;
            q2_rows_dot(
                rowgroup, nb, kq, 4, nt, [&](int t, int b) { return (const int16_t *)(sxq + t * H + b * QK); },
                [&](int t, int b) { return (const int *)(sxs + t * (H / 16) + b * 16); },
                [&](int t, int b) { return sxc[t * nb + b]; }, acc);
#pragma unroll
            for (int t = 0; t < TT_Q; ++t) sm.red[mat][kq][t][lane] = acc[t];
            __syncthreads();
            if (threadIdx.x < nt * 32) {
                const int t = threadIdx.x >> 5, r = threadIdx.x & 31;
                const float g = sm.red[0][0][t][r] + sm.red[0][1][t][r] + sm.red[0][2][t][r] + sm.red[0][3][t][r];
                const float uu = sm.red[1][0][t][r] + sm.red[1][1][t][r] + sm.red[1][2][t][r] + sm.red[1][3][t][r];
                a.h[(size_t)(pc + t) * a.I + rg * TILE_ROWS + r] = silu(g) * uu;
            }
            __syncthreads();
        }
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) atomicAdd(&ctl->exp_done[slot], 1u);
    } else if (u < a.uD) {  // ------------------------------------------------------ SD
        const int v = u - a.uSD;
        const int c0 = v * SD_ROWS;
        if (!cta_wait(&ctl->sg_done, (unsigned)(a.uG - a.uSG), ctl, a.status, &sm.s_ok, &sm.s_t_ready)) return;
        sd_warp(a, c0 + warp * 2);
        if (!ensure_routing(a, sm)) return;
        finish_range(a, sm, c0 / 128);
    } else {  // ----------------------------------------------------------------- D
        const int RG4 = a.H / 128;
        const int v = u - a.uD, slot = v / RG4, rg4 = v % RG4;
        if (!ensure_routing(a, sm)) return;
        if (slot < sm.s_n_act) {
            const int e = sm.r_act[slot];
            const int p0 = sm.r_off[e], p1 = sm.r_off[e + 1];
            const int nbI = a.I / QK;
            const uint8_t *base = a.down + (size_t)e * a.d_bytes + (size_t)rg4 * 4 * nbI * TILE_BYTES;
            if (!cta_wait(&ctl->exp_done[slot], (unsigned)(a.I / TILE_ROWS), ctl, a.status, &sm.s_ok, &sm.s_t_ready))
                return;
            int16_t *hq = reinterpret_cast<int16_t *>(dsm_raw);                              // [TT_Q][I]
            int *hsum = reinterpret_cast<int *>(dsm_raw + TT_Q * a.I * 2);                    // [TT_Q][I/16]
            float *hscale = reinterpret_cast<float *>(dsm_raw + TT_Q * a.I * 2 + TT_Q * (a.I / 16) * 4);
            const int rgl = warp & 3, kh = warp >> 2;
            const uint8_t *rowgroup = base + (size_t)rgl * nbI * TILE_BYTES;
            for (int pc = p0; pc < p1; pc += TT_Q) {
                const int nt = min(TT_Q, p1 - pc);
                for (int wi = warp; wi < nt * nbI; wi += DEC_WARPS) {
                    const int t = wi / nbI, blk = wi % nbI;
                    quantize_f32_warp(a.h + (size_t)(pc + t) * a.I + blk * QK, hq + t * a.I + blk * QK,
                                      hsum + t * (a.I / 16) + blk * 16, hscale + t * nbI + blk);
                }
                __syncthreads();
                float acc[TT_Q];
#pragma unroll
                for (int t = 0; t < TT_Q; ++t) acc[t] = 0.0f;
                const int I = a.I;
                q2_rows_dot(
                    rowgroup, nbI, kh, 2, nt, [&](int t, int b) { return (const int16_t *)(hq + t * I + b * QK); },
                    [&](int t, int b) { return (const int *)(hsum + t * (I / 16) + b * 16); },
                    [&](int t, int b) { return hscale[t * nbI + b]; }, acc);
#pragma unroll
                for (int t = 0; t < TT_Q; ++t) sm.red[kh][rgl][t][lane] = acc[t];
                __syncthreads();
                for (int i = threadIdx.x; i < nt * 128; i += blockDim.x) {
                    const int t = i >> 7, rr = i & 127;
                    const int gl = rr >> 5, r = rr & 31;
                    a.o[(size_t)(pc + t) * a.H + rg4 * 128 + rr] = sm.red[0][gl][t][r] + sm.red[1][gl][t][r];
                }
                __syncthreads();
            }
        }
        finish_range(a, sm, rg4);
    }
}

template <int NPL>
__global__ void __launch_bounds__(DEC_THREADS, 2) decode_kernel(DecodeArgs a) {
    extern __shared__ __align__(16) unsigned char dsm_raw[];
    __shared__ DecSmem sm;
    DecodeCtl *ctl = a.ctl;
    if (threadIdx.x == 0) {
        sm.s_routed = 0;
        sm.s_unit = (int)atomicAdd(&ctl->next_unit, 1u);
        sm.s_next = (int)atomicAdd(&ctl->next_unit, 1u);
    }
    __syncthreads();
    if (a.routing_preset && !a.routing_pdl) ensure_routing(a, sm);
    if (threadIdx.x < 32) prefetch_unit(a, sm, sm.s_unit);
    for (;;) {
        const int u = sm.s_unit;
        if (u >= a.uEnd) break;
        unsigned next2 = 0;
        if (threadIdx.x == 0) {
            // units are handed out two ahead: the one after next is requested now, and the
            // next unit's weights start moving into L2 while this one computes
            next2 = atomicAdd(&ctl->next_unit, 1u);
            sm.s_t_fetch = sm.s_t_ready = gtimer();
        }
        if (threadIdx.x < 32) prefetch_unit(a, sm, sm.s_next);
        __syncthreads();
        run_unit<NPL>(a, sm, dsm_raw, u);
        __syncthreads();
        if (threadIdx.x == 0) {
            if (a.trace) {
                unsigned long long *r = a.trace + 4 * (size_t)u;
                r[0] = (unsigned long long)u | ((unsigned long long)smid() << 32);
                r[1] = sm.s_t_fetch;
                r[2] = sm.s_t_ready;
                r[3] = gtimer();
            }
            sm.s_unit = sm.s_next;
            sm.s_next = (int)next2;
        }
        __syncthreads();
    }
    // The CTA that leaves last resets the counters for the next call (no CTA of this
    // launch touches them any more).
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) sm.s_last = (atomicAdd(&ctl->exited, 1u) == gridDim.x - 1);
    __syncthreads();
    if (sm.s_last) {
        for (int i = threadIdx.x; i < MAX_EXPERTS; i += blockDim.x) ctl->exp_done[i] = 0u;
        for (int i = threadIdx.x; i < 16384 / 128; i += blockDim.x) ctl->rg_done[i] = 0u;
        if (threadIdx.x == 0) {
            ctl->next_unit = 0u; ctl->router_done = 0u; ctl->routing_ready = 0u; ctl->xq_done = 0u;
            ctl->sg_done = 0u; ctl->abort = 0u; ctl->exited = 0u;
        }
    }
}

// Routing of up to MAX_DECODE_T tokens as its own small launch: CTA (b, g) computes router
// rows W*b .. +W-1 for tokens TT_DENSE*g .. +TT_DENSE-1 (one pass of register-held tokens
// per warp); the CTA that finishes last runs the certified top-k of every token (one warp
// per token) and the permutation, then resets the counter for the next call.  W is 4 for a
// single pass of tokens (the rows then spread over E/4 SMs) and 16 above it (16 warps for
// the top-k of up to 64 tokens).  A CTA first copies its tokens into shared memory with all
// loads in flight at once, so the row loops read x there instead of waiting on global
// loads one group at a time.  The launch lets its dependent launch start at once (the
// streaming kernel begins with the shared expert, which does not need the routing).
constexpr int ROUTE_WARPS = 16;
constexpr int ROUTE_WARPS_1 = 4;
inline size_t route_dyn_smem(int H) { return (size_t)TT_DENSE * H * 2; }   // the CTA's tokens, bf16
template <int NPL, int W>
__global__ void __launch_bounds__(W * 32) route_kernel(DecodeArgs a) {
    __shared__ DecSmem sm;
    extern __shared__ __align__(16) unsigned char route_xs[];
    asm volatile("griddepcontrol.launch_dependents;");
    const unsigned long long t_start = gtimer();
    const int warp = threadIdx.x >> 5;
    const int e = blockIdx.x * W + warp;
    const int t0 = blockIdx.y * TT_DENSE, nt = min(TT_DENSE, a.T - t0);
    __nv_bfloat16 *xs = reinterpret_cast<__nv_bfloat16 *>(route_xs);
    if (nt > 0) {   // H is a multiple of 256, so the rows are whole 16-byte vectors
        const uint4 *src = reinterpret_cast<const uint4 *>(a.x + (size_t)t0 * a.H);
        uint4 *dst = reinterpret_cast<uint4 *>(route_xs);
        for (int i = threadIdx.x; i < nt * a.H / 8; i += blockDim.x) dst[i] = __ldg(src + i);
    }
    __syncthreads();
    if (e < a.E && nt > 0)
        router_row_warp<TT_DENSE, true>(xs, nt, a.H, a.wr, a.bias, e, a.E, a.logits + (size_t)t0 * a.E,
                                        a.labs + (size_t)t0 * a.E);
    __threadfence();
    __syncthreads();
    const unsigned cta = blockIdx.y * gridDim.x + blockIdx.x;
    if (threadIdx.x == 0) {
        sm.s_last = (atomicAdd(&a.ctl->router_done, 1u) == gridDim.x * gridDim.y - 1);
        if (a.trace && 4 * (size_t)cta + 3 < (size_t)a.trace_stamps) {   // per-CTA record: block | sm << 32, start, rows done, counted
            unsigned long long *r = a.trace + 4 * (size_t)cta;
            r[0] = (unsigned long long)cta | ((unsigned long long)smid() << 32);
            r[1] = t_start;
            r[2] = gtimer();
            r[3] = gtimer();
        }
    }
    __syncthreads();
    if (!sm.s_last) return;
    stamp(a, 4);
    __threadfence();
    topk_and_permute<NPL>(a, sm);
    if (threadIdx.x == 0) a.ctl->router_done = 0u;
    stamp(a, 3);
}

inline size_t decode_dyn_smem(int I, int H) {
    const int K = I > H ? I : H;
    return (size_t)TT_Q * K * 2 + (size_t)TT_Q * (K / 16) * 4 + (size_t)TT_Q * (K / QK) * 4;
}

}  // namespace ds4
