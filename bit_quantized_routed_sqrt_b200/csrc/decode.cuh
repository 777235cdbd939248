// decode.cuh -- the batched-GEMV path of the layer (three kernels per forward).
//
//  K1  router rows (fp64-accumulated logits) + the last router CTA's certified top-k and
//      permutation; x quantised to int16 per 256-block; shared-expert gate/up + SwiGLU.
//  K2  routed gate/up + SwiGLU: lane = weight row, integer dot products of the 2-bit
//      quants with the int16 activations (dp2a), per-sub-block 4-bit scales and mins
//      applied in integers, fp16 d/dmin and the activation scale in fp32.
//  K3  routed down (h quantised to int16 per 256-block in shared memory), shared-expert
//      down, and the weighted combine done by the last unit of each 128-row range.
// All Q2_K bytes stream from HBM exactly once per call; see common.cuh for the tile layout.
#pragma once
#include "common.cuh"
#include "router.cuh"

namespace ds4 {

struct DecodeArgs {
    int T, H, E, k, I, Is;
    const __nv_bfloat16 *x;        // [T][H]
    const __nv_bfloat16 *wr;       // [E][H]
    const float *bias;             // [E] or null
    const __nv_bfloat16 *sg, *su;  // [Is][H]
    const __nv_bfloat16 *sd;       // [H][Is]
    const uint8_t *gate, *up, *down;  // tiled Q2_K, expert-major
    size_t gu_bytes, d_bytes;         // bytes per expert matrix
    // workspace
    double *logits;
    float *labs;
    RouteOut ro;
    int16_t *xq;
    float *xscale;
    int *xsum;
    float *hs;        // [T][Is]
    float *h;         // [P][I]
    float *o;         // [P][H]
    float *s;         // [T][H]
    float *y;         // [T][H]
    unsigned *router_done;  // [1]
    unsigned *rg_done;      // [H/128]
    int n_router_ctas, n_xq_ctas, n_shared_ctas;
    int do_shared;          // 0: routing only
};

constexpr int K1_WARPS = 4;
constexpr int ROUTER_RW = 2;   // router rows per warp
constexpr int TT_DENSE = 4;    // tokens per pass in the dense GEMVs

// x -> int16 per 256-block: xq = rint(x * 32767 / amax), xscale = amax / 32767,
// xsum[sub-block] = sum of the 16 xq of each sub-block.  One warp per (token, block).
__device__ void quantize_x_warp(const __nv_bfloat16 *x, int H, int t, int blk, int16_t *xq, float *xscale, int *xsum) {
    const int lane = threadIdx.x & 31;
    const int i0 = blk * QK + lane * 8;
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(x + (size_t)t * H + i0));
    float f[8] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y), bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w)};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = warp_max(amax);
    const float inv = amax > 0.0f ? 32767.0f / amax : 0.0f;
    int q[8];
    int s = 0;
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

// Dense bf16 GEMV for the shared expert's gate and up rows r (one warp): h[t][r] = silu(g) u.
__device__ void shared_gateup_warp(const DecodeArgs &a, int r) {
    const int lane = threadIdx.x & 31;
    const __nv_bfloat16 *gw = a.sg + (size_t)r * a.H, *uw = a.su + (size_t)r * a.H;
    for (int t0 = 0; t0 < a.T; t0 += TT_DENSE) {
        const int nt = min(TT_DENSE, a.T - t0);
        float g[TT_DENSE], u[TT_DENSE];
#pragma unroll
        for (int t = 0; t < TT_DENSE; ++t) { g[t] = 0.0f; u[t] = 0.0f; }
        for (int k0 = lane * 8; k0 < a.H; k0 += 256) {
            const uint4 gv = ld_stream_v4(gw + k0), uv = ld_stream_v4(uw + k0);
            const uint32_t gs[4] = {gv.x, gv.y, gv.z, gv.w}, us[4] = {uv.x, uv.y, uv.z, uv.w};
#pragma unroll
            for (int t = 0; t < TT_DENSE; ++t) {
                if (t < nt) {
                    const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)(t0 + t) * a.H + k0));
                    const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float x0 = bf16lo(xs[q]), x1 = bf16hi(xs[q]);
                        g[t] = fmaf(x0, bf16lo(gs[q]), fmaf(x1, bf16hi(gs[q]), g[t]));
                        u[t] = fmaf(x0, bf16lo(us[q]), fmaf(x1, bf16hi(us[q]), u[t]));
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < TT_DENSE; ++t) {
            const float gs = warp_sum(g[t]), us = warp_sum(u[t]);
            if (lane == 0 && t < nt) a.hs[(size_t)(t0 + t) * a.Is + r] = silu(gs) * us;
        }
    }
}

// K1: grid = [router CTAs][x-quant CTAs][shared gate/up CTAs], K1_WARPS warps each.
template <int NPL>
__global__ void __launch_bounds__(K1_WARPS * 32) k1_router_shared_kernel(DecodeArgs a) {
    __shared__ int s_last;
    __shared__ int s_cnt[MAX_EXPERTS];
    __shared__ unsigned long long s_mask[MAX_EXPERTS];
    __shared__ int s_off[MAX_EXPERTS + 1];
    __shared__ int s_idx[64 * MAX_TOPK];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int b = blockIdx.x;
    if (b < a.n_router_ctas) {
        const int e0 = (b * K1_WARPS + warp) * ROUTER_RW;
        if (e0 < a.E) router_rows_warp<ROUTER_RW, TT_DENSE>(a.x, a.T, a.H, a.wr, a.bias, e0, a.E, a.logits, a.labs);
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) s_last = (atomicAdd(a.router_done, 1u) == (unsigned)a.n_router_ctas - 1);
        __syncthreads();
        if (!s_last) return;
        __threadfence();
        // last router CTA: certified top-k of every token, then the permutation (T <= 64)
        for (int t = warp; t < a.T; t += K1_WARPS) {
            warp_topk_certified<NPL>(a.logits + (size_t)t * a.E, a.labs + (size_t)t * a.E, a.E, a.k, BOUND_PAIR, a.H,
                                     a.x + (size_t)t * a.H, a.wr, a.bias, a.ro.topk_idx + (size_t)t * a.k,
                                     a.ro.topk_w + (size_t)t * a.k, a.ro.fallbacks);
            __syncwarp();
            if (lane < a.k) s_idx[t * a.k + lane] = a.ro.topk_idx[(size_t)t * a.k + lane];
        }
        for (int e = threadIdx.x; e < a.E; e += blockDim.x) { s_cnt[e] = 0; s_mask[e] = 0ull; }
        __syncthreads();
        block_count_masks(s_idx, a.T, a.k, s_cnt, s_mask);
        __syncthreads();
        if (warp == 0) warp_scan_active(s_cnt, a.E, s_off, a.ro.active, a.ro.n_active);
        __syncthreads();
        for (int e = threadIdx.x; e <= a.E; e += blockDim.x) a.ro.offsets[e] = s_off[e];
        for (int p = threadIdx.x; p < a.T * a.k; p += blockDim.x) {
            const int t = p / a.k, j = p % a.k;
            const int e = s_idx[p];
            const int pos = s_off[e] + __popcll(s_mask[e] & ((1ull << t) - 1ull));
            a.ro.sorted_token[pos] = t;
            a.ro.sorted_slot[pos] = j;
            a.ro.inv_pos[p] = pos;
        }
        if (threadIdx.x == 0) *a.router_done = 0u;
        return;
    }
    b -= a.n_router_ctas;
    if (b < a.n_xq_ctas) {
        // (token, block) pairs, one per warp
        const int nbk = a.H / QK;
        for (int wi = b * K1_WARPS + warp; wi < a.T * nbk; wi += a.n_xq_ctas * K1_WARPS)
            quantize_x_warp(a.x, a.H, wi / nbk, wi % nbk, a.xq, a.xscale, a.xsum);
        return;
    }
    b -= a.n_xq_ctas;
    for (int r = b * K1_WARPS + warp; r < a.Is; r += a.n_shared_ctas * K1_WARPS) shared_gateup_warp(a, r);
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
            const uint32_t q0 = (w[0] >> (2 * j)) & 0x03030303u, q1 = (w[1] >> (2 * j)) & 0x03030303u;
            const uint32_t q2 = (w[2] >> (2 * j)) & 0x03030303u, q3 = (w[3] >> (2 * j)) & 0x03030303u;
            int d = dp2a_lo((int)xa.x, q0, 0);
            d = dp2a_hi((int)xa.y, q0, d);
            d = dp2a_lo((int)xa.z, q1, d);
            d = dp2a_hi((int)xa.w, q1, d);
            d = dp2a_lo((int)xb.x, q2, d);
            d = dp2a_hi((int)xb.y, q2, d);
            d = dp2a_lo((int)xb.z, q3, d);
            d = dp2a_hi((int)xb.w, q3, d);
            const uint32_t sbyte = (scw[sb >> 2] >> (8 * (sb & 3))) & 0xFFu;
            isc += (int)(sbyte & 0xFu) * d;
            imn += (int)(sbyte >> 4) * xs[sb];
        }
    }
}

constexpr int K2_WARPS = 8;
constexpr int TT_Q = 4;   // tokens per pass in the Q2_K GEMVs

// K2: routed gate/up + SwiGLU.  Unit = (active expert a, 32-row group of I); warp w takes
// matrix w/4 (gate, up) and the blocks b = w%4, w%4 + 4, ... of the H/256 input blocks.
__global__ void __launch_bounds__(K2_WARPS * 32) k2_gateup_kernel(DecodeArgs a) {
    __shared__ float red[2][4][TT_Q][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int mat = warp >> 2, kq = warp & 3;
    const int nb = a.H / QK, RG = a.I / TILE_ROWS;
    const int n_act = *a.ro.n_active;
    const int n_units = n_act * RG;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int ai = u / RG, rg = u % RG;
        const int e = a.ro.active[ai];
        const int p0 = a.ro.offsets[e], p1 = a.ro.offsets[e + 1];
        const uint8_t *base = (mat == 0 ? a.gate : a.up) + (size_t)e * a.gu_bytes + (size_t)rg * nb * TILE_BYTES;
        for (int pc = p0; pc < p1; pc += TT_Q) {
            const int nt = min(TT_Q, p1 - pc);
            int tok[TT_Q];
#pragma unroll
            for (int t = 0; t < TT_Q; ++t) tok[t] = a.ro.sorted_token[pc + min(t, nt - 1)];
            float acc[TT_Q];
#pragma unroll
            for (int t = 0; t < TT_Q; ++t) acc[t] = 0.0f;
            for (int b = kq; b < nb; b += 4) {
                const uint8_t *tile = base + (size_t)b * TILE_BYTES;
                uint4 qs[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) qs[c] = ld_stream_v4(tile + TILE_QS + c * 512 + lane * 16);
                const uint4 sc = ld_stream_v4(tile + TILE_SC + lane * 16);
                const uint32_t dm = ld_stream_u32(tile + TILE_DM + lane * 4);
                const float d = h2f(dm), dmin = h2f(dm >> 16);
#pragma unroll
                for (int t = 0; t < TT_Q; ++t) {
                    if (t < nt) {
                        int isc, imn;
                        q2k_block_dot(qs, sc, a.xq + (size_t)tok[t] * a.H + b * QK, a.xsum + (size_t)tok[t] * (a.H / 16) + b * 16,
                                      isc, imn);
                        const float xsc = __ldg(a.xscale + (size_t)tok[t] * nb + b);
                        acc[t] = fmaf(xsc, fmaf(d, (float)isc, -dmin * (float)imn), acc[t]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < TT_Q; ++t) red[mat][kq][t][lane] = acc[t];
            __syncthreads();
            if (threadIdx.x < nt * 32) {
                const int t = threadIdx.x >> 5, r = threadIdx.x & 31;
                const float g = red[0][0][t][r] + red[0][1][t][r] + red[0][2][t][r] + red[0][3][t][r];
                const float uu = red[1][0][t][r] + red[1][1][t][r] + red[1][2][t][r] + red[1][3][t][r];
                a.h[(size_t)(pc + t) * a.I + rg * TILE_ROWS + r] = silu(g) * uu;
            }
            __syncthreads();
        }
    }
}

// K3 unit counts: routed units (active expert, 128-row range of H) and shared units
// (128-row range, 16-row part).  The last unit to finish a range writes y for it.
constexpr int K3_WARPS = 8;
constexpr int SH_PARTS = 8;

__global__ void __launch_bounds__(K3_WARPS * 32) k3_down_combine_kernel(DecodeArgs a) {
    extern __shared__ __align__(16) unsigned char k3_smem[];
    __shared__ float red[2][4][TT_Q][32];
    __shared__ int s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nbI = a.I / QK, RG4 = a.H / 128;
    int16_t *hq = reinterpret_cast<int16_t *>(k3_smem);                       // [TT_Q][I]
    int *hsum = reinterpret_cast<int *>(k3_smem + TT_Q * a.I * 2);            // [TT_Q][I/16]
    float *hscale = reinterpret_cast<float *>(k3_smem + TT_Q * a.I * 2 + TT_Q * (a.I / 16) * 4);  // [TT_Q][I/256]
    const int n_act = *a.ro.n_active;
    const int shared_parts = a.Is > 0 ? SH_PARTS : 0;
    const int n_routed = n_act * RG4;
    const int n_units = n_routed + RG4 * shared_parts;
    const unsigned target = (unsigned)(n_act + shared_parts);
    int cached_e = -1, cached_pc = -1;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        int rg4;
        if (u < n_routed) {
            const int ai = u / RG4;
            rg4 = u % RG4;
            const int e = a.ro.active[ai];
            const int p0 = a.ro.offsets[e], p1 = a.ro.offsets[e + 1];
            const int rgl = warp & 3, kh = warp >> 2;
            const uint8_t *base = a.down + (size_t)e * a.d_bytes + (size_t)(rg4 * 4 + rgl) * nbI * TILE_BYTES;
            for (int pc = p0; pc < p1; pc += TT_Q) {
                const int nt = min(TT_Q, p1 - pc);
                if (cached_e != e || cached_pc != pc) {
                    __syncthreads();
                    // quantise h of pairs pc .. pc+nt-1 per 256-block (one warp per (pair, block))
                    for (int wi = warp; wi < nt * nbI; wi += K3_WARPS) {
                        const int t = wi / nbI, blk = wi % nbI;
                        const float *src = a.h + (size_t)(pc + t) * a.I + blk * QK + lane * 8;
                        const float4 v0 = __ldcg(reinterpret_cast<const float4 *>(src));
                        const float4 v1 = __ldcg(reinterpret_cast<const float4 *>(src + 4));
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
                        *reinterpret_cast<uint4 *>(hq + t * a.I + blk * QK + lane * 8) = o;
                        if ((lane & 1) == 0) hsum[t * (a.I / 16) + blk * 16 + lane / 2] = s;
                        if (lane == 0) hscale[t * nbI + blk] = amax / 32767.0f;
                    }
                    cached_e = e;
                    cached_pc = pc;
                    __syncthreads();
                }
                float acc[TT_Q];
#pragma unroll
                for (int t = 0; t < TT_Q; ++t) acc[t] = 0.0f;
                for (int b = kh; b < nbI; b += 2) {
                    const uint8_t *tile = base + (size_t)b * TILE_BYTES;
                    uint4 qs[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c) qs[c] = ld_stream_v4(tile + TILE_QS + c * 512 + lane * 16);
                    const uint4 sc = ld_stream_v4(tile + TILE_SC + lane * 16);
                    const uint32_t dm = ld_stream_u32(tile + TILE_DM + lane * 4);
                    const float d = h2f(dm), dmin = h2f(dm >> 16);
#pragma unroll
                    for (int t = 0; t < TT_Q; ++t) {
                        if (t < nt) {
                            int isc, imn;
                            q2k_block_dot(qs, sc, hq + t * a.I + b * QK, hsum + t * (a.I / 16) + b * 16, isc, imn);
                            acc[t] = fmaf(hscale[t * nbI + b], fmaf(d, (float)isc, -dmin * (float)imn), acc[t]);
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < TT_Q; ++t) red[kh][rgl][t][lane] = acc[t];
                __syncthreads();
                if (threadIdx.x < nt * 128) {
                    const int t = threadIdx.x >> 7, rr = threadIdx.x & 127;
                    const int gl = rr >> 5, r = rr & 31;
                    a.o[(size_t)(pc + t) * a.H + rg4 * 128 + rr] = red[0][gl][t][r] + red[1][gl][t][r];
                }
                __syncthreads();
            }
        } else {
            const int v = u - n_routed;
            rg4 = v / shared_parts;
            const int part = v % shared_parts;
            // 16 rows per part, 2 per warp
            for (int rr = warp * 2; rr < warp * 2 + 2; ++rr) {
                const int row = rg4 * 128 + part * 16 + rr;
                const __nv_bfloat16 *wrow = a.sd + (size_t)row * a.Is;
                for (int t0 = 0; t0 < a.T; t0 += TT_DENSE) {
                    const int nt = min(TT_DENSE, a.T - t0);
                    float acc[TT_DENSE];
#pragma unroll
                    for (int t = 0; t < TT_DENSE; ++t) acc[t] = 0.0f;
                    for (int k0 = lane * 8; k0 < a.Is; k0 += 256) {
                        const uint4 wv = ld_stream_v4(wrow + k0);
                        const float w8[8] = {bf16lo(wv.x), bf16hi(wv.x), bf16lo(wv.y), bf16hi(wv.y),
                                             bf16lo(wv.z), bf16hi(wv.z), bf16lo(wv.w), bf16hi(wv.w)};
#pragma unroll
                        for (int t = 0; t < TT_DENSE; ++t) {
                            if (t < nt) {
                                const float *hp = a.hs + (size_t)(t0 + t) * a.Is + k0;
                                const float4 h0 = __ldcg(reinterpret_cast<const float4 *>(hp));
                                const float4 h1 = __ldcg(reinterpret_cast<const float4 *>(hp + 4));
                                acc[t] = fmaf(w8[0], h0.x, fmaf(w8[1], h0.y, fmaf(w8[2], h0.z, fmaf(w8[3], h0.w, acc[t]))));
                                acc[t] = fmaf(w8[4], h1.x, fmaf(w8[5], h1.y, fmaf(w8[6], h1.z, fmaf(w8[7], h1.w, acc[t]))));
                            }
                        }
                    }
#pragma unroll
                    for (int t = 0; t < TT_DENSE; ++t) {
                        const float sres = warp_sum(acc[t]);
                        if (lane == 0 && t < nt) a.s[(size_t)(t0 + t) * a.H + row] = sres;
                    }
                }
            }
        }
        // completion of this unit's 128-row range; the last one combines
        __threadfence();
        __syncthreads();
        if (threadIdx.x == 0) s_last = (atomicAdd(a.rg_done + rg4, 1u) == target - 1);
        __syncthreads();
        if (s_last) {
            __threadfence();
            for (int i = threadIdx.x; i < a.T * 128; i += blockDim.x) {
                const int t = i >> 7, row = rg4 * 128 + (i & 127);
                float acc = 0.0f;
                for (int j = 0; j < a.k; ++j) {
                    const int p = __ldcg(a.ro.inv_pos + (size_t)t * a.k + j);
                    acc = fmaf(__ldcg(a.ro.topk_w + (size_t)t * a.k + j), __ldcg(a.o + (size_t)p * a.H + row), acc);
                }
                if (shared_parts) acc += __ldcg(a.s + (size_t)t * a.H + row);
                a.y[(size_t)t * a.H + row] = acc;
            }
            if (threadIdx.x == 0) a.rg_done[rg4] = 0u;
        }
    }
}

}  // namespace ds4
