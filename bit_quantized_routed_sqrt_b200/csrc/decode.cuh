// decode.cuh -- the batched-GEMV path of the layer (T <= 32 tokens) as ONE persistent,
// cooperative launch: one CTA per SM, warp-specialised.
//
//   warp 0      producer: claims work units from a global counter (in unit order) and
//               streams each unit's weight bytes into a ring of shared-memory slots with
//               bulk copies (cp.async.bulk, 43 KB per slot).  It never waits on another
//               unit's result -- only on a free slot, and once on the routing.
//   warp 1      scheduler: after the router rows are done, the certified top-k (the same
//               selection for every CTA), the permutation and the unit table in shared
//               memory; CTA 0 also publishes the routing outputs.  Then a second epilogue
//               warp (the units of the second partial-sum buffer).
//   warp 2      epilogue: reduces the consumer warps' partial sums of a finished unit,
//               applies SwiGLU (and the int16 re-quantisation of h) or the routing weight,
//               writes the unit's rows, and publishes the counts of finished units in
//               batches; once every down unit of the launch is done, each CTA writes y for
//               its share of the 64-row ranges of H (y = S + sum_j w_j o_j in slot order).
//   warps 3-18  consumers: first the router rows of this CTA (split along K over the 16
//               warps) and its share of the int16 quantisation of x; then, slot by slot,
//               dot products of the streamed
//               weights with the activations: warp w takes tile w of a Q2_K piece (lane =
//               weight row) or (row, K segment) w of a dense bf16 piece.
//
// Unit kinds:
//   SG  shared gate/up: R rows of gate + the same R rows of up (two dense pieces)
//   G   routed gate/up: (expert group, 32 rows of I): the Q2_K tiles of gate, then of up
//   SD  shared down: 2R rows of H (two dense pieces); needs every SG unit
//   D   routed down: (expert group, 64 rows of H); needs the G units of its group
// Unit order, in four phases (each unit waits only on units before it, so the schedule
// cannot deadlock):
//   A   the SG units: they need no routing and cover its latency;
//   B   the G units, group by group (the interleave formula can mix SG units in, one after
//       every two G units; the plan mixes none);
//   C0  the SD units that the mixing of C1 has no room for (usually none);
//   C1  the D units, group by group, with the SD units mixed in, one after every two D units.
// A D unit waits only for its own group's G units, which phase B finished long before
// (groups run in the same order in both phases), so no CTA waits at the boundary for the
// last G units of the launch; the SD units need every SG unit, all of them early in B.
// Mixing the dense bf16 units (cheap to compute per byte) among the Q2_K units (whose dot
// products bound the SM's integer pipe) keeps both the HBM and the SM busy.
// An expert group is one active expert with up to DK_TU of its tokens.  Dependencies only
// gate the consumers: the producer keeps streaming the weights of later units (they do not
// depend on the activations), so the HBM stays busy while a phase boundary resolves.
//
// Activations travel with the weights: each piece's slot starts with an activation area
// that the producer fills in the same bulk copy batch -- the int16 records of x (G; x
// quantised per 256-block, its sub-block sums and scales), every token's bf16 x (SG), the
// routed h records (D; h re-quantised to int16 with a scale per 32 rows, sums, scales) or
// every token's fp32 shared h (SD).  SD and D inputs are staged only when the producer finds
// them published (one acquire load per group, or once for the shared h); otherwise the
// consumers wait for the count and read them from global memory.  Int16 values are limited
// to +-8191 so the Q2_K dot keeps one integer accumulator per bit plane without overflow.
//
// Every wait is bounded in time; a timeout sets ETIMEOUT and an abort flag that every
// role checks, and a CTA drains its own bulk copies before it returns.
#pragma once
#include <algorithm>
#include <cstddef>
#include "common.cuh"
#include "mbar.cuh"
#include "router.cuh"

namespace ds4 {

constexpr int MAX_DECODE_T = 32;
constexpr int DK_CW = 16;                          // consumer warps
constexpr int DK_W_PROD = 0, DK_W_SCHED = 1, DK_W_EPI = 2, DK_W_CONS = 3;
constexpr int DK_WARPS = DK_W_CONS + DK_CW;        // 19
constexpr int DK_THREADS = DK_WARPS * 32;          // 608
constexpr int DK_XA = 18560;                       // activation area at the start of a slot
constexpr int DK_WOFF = DK_XA;                     // weights start here within a slot
constexpr int DK_SLOT = DK_XA + 16 * TILE_BYTES;   // + 43008 B: 16 Q2_K tiles, or <= 32 KB of dense rows
constexpr int DK_NSLOT = 3;
constexpr int DK_TU = 2;                           // tokens per routed unit
constexpr int DK_TR = 4;                           // tokens per router item
constexpr int DK_TRED = 2;                         // T up to this: every CTA runs the top-k itself
constexpr int DK_MAXP = MAX_DECODE_T * MAX_TOPK;   // 512 (token, slot) pairs
constexpr int DK_QMAX = 8191;                      // int16 activation range
constexpr int DK_RANGE = 64;                       // rows of H per combine range (one D unit)
constexpr int DK_MAX_RANGES = 16384 / DK_RANGE;
constexpr int DK_DENSE_ELEMS = 16384;              // dense piece: rows * K <= this (32 KB of bf16)
constexpr int DK_PBUF = 2;                         // partial-sum buffers between consumers and epilogue

// Global control words of one launch; zero before the launch, reset by the last CTA to exit.
struct DecCtl {
    unsigned next_unit;    // unit claims
    unsigned route_done;   // router / x-quantisation items finished
    unsigned topk_next;    // token claims of the distributed top-k
    unsigned topk_done;
    unsigned sg_done;      // SG units finished
    unsigned abort;
    unsigned exited;
    unsigned grp_done[DK_MAXP];          // G units finished, per expert group
    unsigned rng_done[DK_MAX_RANGES];    // SD and D units finished, per 64-row range of H
};

// Launch constants (host-computed; nothing here depends on the routing).
struct DecPlan {
    int nbH, nbI;          // 256-blocks along H and along I
    int RSG, SSG;          // dense rows per SG piece and K segments per row (RSG * SSG = 16)
    int RSD, SSD;          // the same for SD pieces (K = Is)
    int nSG, nSD;          // shared units
    int nA, nB;            // SG units in phase A and mixed into phase B
    int nC0, nC1;          // SD units in the run of phase C0 and mixed into phase C1
    int RGI, RPH;          // 32-row groups of I (G units per group), 64-row ranges of H (D units per group)
    int ppGm;              // G pieces per matrix: ceil(nbH / 16)
    int ppD;               // D pieces: ceil(2 nbI / 16)
    int nTR;               // token chunks of the router items
    int n_route_items;     // E * nTR router items + T * nbH x-quantisation items
    int sd_per_range;      // SD units per 64-row range
    int xrec;              // bytes of one token's int16 record: x (H), sub-block sums (H/16), scales (H/256)
    int xs_off, xc_off;    // offsets of the sums and the scales in a record
    int stage_g;           // G pieces carry their tokens' records (nt * xrec <= DK_XA)
    int stage_sg;          // SG pieces carry the bf16 rows of every token (T * 2H <= DK_XA)
    int hrec;              // bytes of one pair's h record: int16 h (I), sub-block sums (I/16), scales (I/32)
    int hs_off, hc_off;    // offsets of the sums and the scales in an h record
    int stage_d;           // D pieces can carry their pairs' h records (nt * hrec <= DK_XA)
    int stage_sd;          // SD pieces can carry every token's fp32 h_s row (T * 4 Is <= DK_XA)
};

// Rows of a dense piece: the largest power of two <= 16 with rows * K <= 16384.
__host__ __device__ inline int dense_rows(int K) {
    int r = 16;
    while (r > 1 && r * K > DK_DENSE_ELEMS) r >>= 1;
    return r;
}

inline DecPlan make_dec_plan(int T, int H, int E, int k, int I, int Is) {
    DecPlan p{};
    p.nbH = H / QK;
    p.nbI = I / QK;
    p.RSG = dense_rows(H);
    p.SSG = 16 / p.RSG;
    p.RSD = Is > 0 ? dense_rows(Is) : 16;
    p.SSD = 16 / p.RSD;
    p.nSG = Is > 0 ? Is / p.RSG : 0;
    p.nSD = Is > 0 ? H / (2 * p.RSD) : 0;
    p.RGI = I / TILE_ROWS;
    p.RPH = H / DK_RANGE;
    p.ppGm = (p.nbH + 15) / 16;
    p.ppD = (2 * p.nbI + 15) / 16;
    p.nTR = (T + DK_TR - 1) / DK_TR;
    p.n_route_items = E * p.nTR + T * p.nbH;
    p.sd_per_range = Is > 0 ? DK_RANGE / (2 * p.RSD) : 0;
    // every launch has at least k expert groups (the first token's k distinct experts), so
    // phase B holds at least RGI * k G units and phase C1 at least RPH * k D units: the
    // shared units mixed in (one per two routed units) never outnumber them
    // every SG unit runs in phase A, while the routing resolves (dense and Q2_K pieces take
    // about as long per byte here, so mixing SG units into phase B buys nothing); likewise
    // every SD unit runs in phase C0, before the D units: the consumers then do not switch
    // between the two dot products piece by piece, and the last groups' G units get the
    // SD units' time to finish (single token: 63.9 against 65.3 us with them mixed)
    p.nB = 0;
    p.nA = p.nSG - p.nB;
    p.nC1 = 0;
    p.nC0 = p.nSD - p.nC1;
    p.xs_off = 2 * H;
    p.xc_off = p.xs_off + H / 4;
    p.xrec = (p.xc_off + H / 64 + 15) / 16 * 16;
    p.stage_g = DK_TU * p.xrec <= DK_XA;
    p.stage_sg = T * 2 * H <= DK_XA;
    p.hs_off = 2 * I;
    p.hc_off = p.hs_off + I / 4;
    p.hrec = (p.hc_off + I / 8 + 15) / 16 * 16;
    p.stage_d = DK_TU * p.hrec <= DK_XA;
    p.stage_sd = Is > 0 && T * 4 * Is <= DK_XA;
    return p;
}

struct DecArgs {
    int T, H, E, k, I, Is;
    DecPlan pl;
    const __nv_bfloat16 *x;        // [T][H]
    const __nv_bfloat16 *wr;       // [E][H]
    const float *bias;             // [E] or null
    const __nv_bfloat16 *sg, *su;  // [Is][H]
    const __nv_bfloat16 *sd;       // [H][Is]
    const uint8_t *gate, *up, *down;  // tiled Q2_K, expert-major
    size_t gu_bytes, d_bytes;         // bytes per expert matrix
    double *logits;                // [T][E]
    float *labs;                   // [T][E]
    RouteOut ro;
    uint8_t *xrec;                 // [T][pl.xrec]: int16 x, its sub-block sums and block scales
    float *hs;                     // [T][Is]
    uint8_t *hrec;                 // [P][pl.hrec]: routed h re-quantised to int16, its sub-block sums and scales
    float *o;                      // [P][H]: w * routed expert output, pair order
    float *s;                      // [T][H]: shared expert output
    float *y;                      // [T][H]
    DecCtl *ctl;
    int *status;
    int route_only;                // routing outputs only (no expert work)
    int test_timeout;              // test hook: the first D unit waits on a count that is never reached
    long long wait_ns;             // limit of every bounded wait
    unsigned long long *trace;     // optional timeline (layout: dk_trace_cta / dk_trace_tail)
    int trace_units;               // unit records available in trace
};

// Work units
enum : int { U_SG = 0, U_G = 1, U_SD = 2, U_D = 3, U_END = 4 };

struct Unit {
    int type;
    int a;   // SG: first row; G, D: group; SD: first row
    int b;   // G: 32-row group of I; D: 64-row range of H
};

// ---------------------------------------------------------------------------------------
// Shared memory of a CTA (after the ring).
struct DecTable {
    int ok, NG;
    int nG, nD;            // G and D units
    int uC, uC1, uEnd;     // first unit of phases C0 and C1, and the end
    int topi[DK_MAXP];             // [t * k + j] selected expert
    float topw[DK_MAXP];           // [t * k + j] its weight
    unsigned mask[MAX_EXPERTS];    // tokens of each expert (bit t)
    int off[MAX_EXPERTS + 1];      // pair offsets
    short grp_e[DK_MAXP], grp_p0[DK_MAXP];
    signed char grp_nt[DK_MAXP];
    signed char pair_slot[DK_MAXP];
    short pair_tok[DK_MAXP];
    short inv[DK_MAXP];            // [t * k + j] pair position
};

constexpr int DK_PART_FLOATS = 2 * DK_CW * DK_TU * 32;   // partials of one unit (2 sets)
static_assert(2 * DK_CW * MAX_DECODE_T <= DK_PART_FLOATS, "dense partials fit the buffer");

struct DecSmem {
    unsigned long long full[DK_NSLOT], empty[DK_NSLOT], pfull[DK_PBUF], pempty[DK_PBUF], route_bar, items_bar;
    int meta_unit[DK_NSLOT], meta_piece[DK_NSLOT];
    int meta_staged[DK_NSLOT];     // 1: the piece carries its SD or D unit's activations
    Unit meta_un[DK_NSLOT];        // the piece's unit, decoded once by the producer
    int last_issue[DK_NSLOT];      // index of the last copy issued into each slot (-1: none)
    int cons_pos[DK_CW];           // ring positions each consumer warp has finished with
    int part_unit[DK_PBUF];
    Unit part_un[DK_PBUF];
    alignas(16) float part[DK_PBUF][DK_PART_FLOATS];   // also the fp64 router partial sums
    double tk_v[MAX_EXPERTS], tk_m[MAX_EXPERTS];       // the scheduler's top-k: logits, bounds
    DecTable tb;
};
static_assert(offsetof(DecSmem, part) % 16 == 0, "partials hold doubles");

constexpr size_t DK_SMEM = (size_t)DK_NSLOT * DK_SLOT + sizeof(DecSmem) + 128;
static_assert(DK_SMEM <= 227 * 1024, "shared memory of one CTA");

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
// Trace layout: 4 words per unit (unit | ns the consumers spent on it << 32, first copy
// issued, consumers started, epilogue done), then 8 words per CTA (start, its router rows
// done, routing seen, top-k done, table ready, exit, 0, 0), then a 16-word tail (the four phase
// bounds at 0..3, the top-k step stamps of CTA 0 at 8..13), then 8 more words per unit
// (consumers' partials written, epilogue started, CTA | staged << 16, pieces 0 and 1 seen
// landed by the consumers, piece 1 issued, piece 0 computed, SM cycles of its epilogue).
__device__ __forceinline__ unsigned long long *dk_trace_cta(const DecArgs &a) {
    return a.trace + 4 * (size_t)a.trace_units + 8 * (size_t)blockIdx.x;
}
__device__ __forceinline__ unsigned long long *dk_trace_tail(const DecArgs &a) {
    return a.trace + 4 * (size_t)a.trace_units + 8 * (size_t)gridDim.x;
}
__device__ __forceinline__ unsigned long long *dk_trace_ext(const DecArgs &a, int u) {
    return dk_trace_tail(a) + 16 + 8 * (size_t)u;
}
__device__ __forceinline__ unsigned ld_relaxed(const unsigned *p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void dk_abort(const DecArgs &a) {
    set_status(a.status, ST_ETIMEOUT);
    atomicExch(&a.ctl->abort, 1u);
}

// Wait (one thread) until *p >= target, bounded by a.wait_ns; false on timeout or abort.
// The successful exit is an acquire load (it orders the caller's later reads).
__device__ bool dk_poll(const DecArgs &a, const unsigned *p, unsigned target, long long limit_ns) {
    const unsigned long long t0 = gtimer();
    for (int it = 0;; ++it) {
        if (ld_acquire(p) >= target) return true;
        if (ld_relaxed(&a.ctl->abort)) return false;
        if ((long long)(gtimer() - t0) > limit_ns) {
            dk_abort(a);
            return false;
        }
        __nanosleep(it < 16 ? 32 : 128);
    }
}

// Mbarrier phase wait of one thread, bounded by a.wait_ns; false on timeout or abort.
__device__ bool dk_wait(const DecArgs &a, uint32_t bar, uint32_t parity) {
    if (mbar_try_spin(bar, parity)) return true;
    const unsigned long long t0 = gtimer();
    for (int it = 0;; ++it) {
        if (mbar_try_spin(bar, parity)) return true;
        if ((it & 7) == 7) {
            if (ld_relaxed(&a.ctl->abort)) return false;
            if ((long long)(gtimer() - t0) > a.wait_ns) {
                dk_abort(a);
                return false;
            }
        }
    }
}
// Warp-uniform version: lane 0 waits, every lane gets the result.
__device__ __forceinline__ bool dk_wait_warp(const DecArgs &a, uint32_t bar, uint32_t parity) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = dk_wait(a, bar, parity) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}
// The other lanes' later reads are ordered after lane 0's acquire by the warp barrier.
__device__ __forceinline__ bool dk_poll_warp(const DecArgs &a, const unsigned *p, unsigned target, long long limit_ns) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = dk_poll(a, p, target, limit_ns) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}
// Add to a global count with release semantics (the warp's earlier global writes, ordered
// before by __syncwarp, become visible no later than the count).  A release needs no
// invalidation of the SM's L1, which an acquire-release fence would cost every warp that
// reads activations through it.
__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Count a finished item (after the warp's global writes).
__device__ __forceinline__ void dk_count(unsigned *p) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) red_release_add(p, 1u);
    __syncwarp();
}

// ---------------------------------------------------------------------------------------
// Work units



__device__ __forceinline__ Unit decode_unit(const DecPlan &pl, const DecTable &tb, int u) {
    Unit r;
    int sg = -1, g = -1, sd = -1, d = -1;
    if (u < pl.nA) {
        sg = u;
    } else if (u < tb.uC) {
        const int p = u - pl.nA;
        if (p % 3 == 2 && p / 3 < pl.nB) sg = pl.nA + p / 3;
        else g = p - min(pl.nB, p / 3);
    } else if (u < tb.uC1) {
        sd = u - tb.uC;
    } else if (u < tb.uEnd) {
        const int p = u - tb.uC1;
        if (p % 3 == 2 && p / 3 < pl.nC1) sd = pl.nC0 + p / 3;
        else d = p - min(pl.nC1, p / 3);
    }
    if (sg >= 0) { r.type = U_SG; r.a = sg * pl.RSG; r.b = 0; }
    else if (g >= 0) { r.type = U_G; r.a = g / pl.RGI; r.b = g % pl.RGI; }
    else if (sd >= 0) { r.type = U_SD; r.a = sd * 2 * pl.RSD; r.b = 0; }
    else if (d >= 0) { r.type = U_D; r.a = d / pl.RPH; r.b = d % pl.RPH; }
    else { r.type = U_END; r.a = r.b = 0; }
    return r;
}

__device__ __forceinline__ int unit_pieces(const DecPlan &pl, int type) {
    return type == U_G ? 2 * pl.ppGm : type == U_D ? pl.ppD : 2;
}

// Source bytes of piece pi of unit un.
__device__ __forceinline__ void piece_src(const DecArgs &a, const DecTable &tb, const Unit &un, int pi,
                                          const uint8_t *&src, uint32_t &bytes) {
    const DecPlan &pl = a.pl;
    if (un.type == U_SG) {
        const __nv_bfloat16 *m = pi == 0 ? a.sg : a.su;
        src = reinterpret_cast<const uint8_t *>(m + (size_t)un.a * a.H);
        bytes = (uint32_t)(pl.RSG * a.H * 2);
    } else if (un.type == U_SD) {
        src = reinterpret_cast<const uint8_t *>(a.sd + (size_t)(un.a + pi * pl.RSD) * a.Is);
        bytes = (uint32_t)(pl.RSD * a.Is * 2);
    } else if (un.type == U_G) {
        const int mat = pi / pl.ppGm, b0 = (pi % pl.ppGm) * 16;
        const int nt = min(16, pl.nbH - b0);
        const int e = tb.grp_e[un.a];
        src = (mat == 0 ? a.gate : a.up) + (size_t)e * a.gu_bytes + ((size_t)un.b * pl.nbH + b0) * TILE_BYTES;
        bytes = (uint32_t)(nt * TILE_BYTES);
    } else {
        const int t0 = pi * 16, nt = min(16, 2 * pl.nbI - t0);
        const int e = tb.grp_e[un.a];
        src = a.down + (size_t)e * a.d_bytes + ((size_t)un.b * 2 * pl.nbI + t0) * TILE_BYTES;
        bytes = (uint32_t)(nt * TILE_BYTES);
    }
}

// ---------------------------------------------------------------------------------------
// Routing items (consumer warps, before the ring)

// x -> int16 per 256-block (|q| <= DK_QMAX), the 16 sub-block sums and the block scale.
__device__ __forceinline__ void dk_quantize_x(const DecArgs &a, int t, int blk) {
    const int lane = threadIdx.x & 31;
    const int i0 = blk * QK + lane * 8;
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)t * a.H + i0));
    const float f[8] = {bf16lo(v.x), bf16hi(v.x), bf16lo(v.y), bf16hi(v.y),
                        bf16lo(v.z), bf16hi(v.z), bf16lo(v.w), bf16hi(v.w)};
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = warp_max(amax);
    const float inv = amax > 0.0f ? (float)DK_QMAX / amax : 0.0f;
    int q[8], s = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        q[i] = max(-DK_QMAX, min(DK_QMAX, __float2int_rn(f[i] * inv)));
        s += q[i];
    }
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    uint4 o;
    o.x = (uint32_t)(q[0] & 0xFFFF) | ((uint32_t)q[1] << 16);
    o.y = (uint32_t)(q[2] & 0xFFFF) | ((uint32_t)q[3] << 16);
    o.z = (uint32_t)(q[4] & 0xFFFF) | ((uint32_t)q[5] << 16);
    o.w = (uint32_t)(q[6] & 0xFFFF) | ((uint32_t)q[7] << 16);
    uint8_t *rec = a.xrec + (size_t)t * a.pl.xrec;
    *reinterpret_cast<uint4 *>(rec + (size_t)i0 * 2) = o;
    if ((lane & 1) == 0) reinterpret_cast<int *>(rec + a.pl.xs_off)[blk * 16 + lane / 2] = s;
    if (lane == 0) reinterpret_cast<float *>(rec + a.pl.xc_off)[blk] = amax / (float)DK_QMAX;
}

// The router rows of this CTA (e = blockIdx.x + gridDim.x * j), for every token, computed by
// all 16 consumer warps: a task is (row, chunk of DK_TR tokens, K slice); each lane sums
// pairs of exact bf16 products in fp32 (one rounding per pair) into fp64, with the sum of
// |x_i w_i| for the bound; the slices meet in shared memory and are added in fp64.  Two
// rows per round.  Then this CTA's share of the int16 quantisation of x.  `consumer bar`:
// named barrier 1 over the 512 consumer threads.
__device__ __forceinline__ void cons_bar() { asm volatile("bar.sync 1, 512;" ::: "memory"); }

// T1: one token (the token loops hold one iteration).
template <bool T1>
__device__ __forceinline__ void route_rows_cta(const DecArgs &a, DecSmem &sm, int w) {
    constexpr int TRN = T1 ? 1 : DK_TR;   // token slots per router item this build handles
    const int lane = threadIdx.x & 31;
    const int G = gridDim.x, c = blockIdx.x, nbH = a.pl.nbH, nTR = a.pl.nTR;
    const int nrows = c < a.E ? (a.E - 1 - c) / G + 1 : 0;
    const int S = min(8, nbH), bps = (nbH + S - 1) / S;   // K slices per row, 256-blocks per slice
    double *psum = reinterpret_cast<double *>(&sm.part[0][0]);   // [2][nTR][8][DK_TR]
    float *pabs = reinterpret_cast<float *>(psum + 2 * 8 * 8 * DK_TR);
    for (int j0 = 0; j0 < nrows; j0 += 2) {
        const int nr = min(2, nrows - j0), ntask = nr * nTR * S;
        for (int task = w; task < ntask; task += DK_CW) {
            const int sl = task % S, tc = (task / S) % nTR, rr = task / (S * nTR);
            const int e = c + G * (j0 + rr);
            const int t0 = tc * DK_TR, nt = min(DK_TR, a.T - t0);
            const __nv_bfloat16 *row = a.wr + (size_t)e * a.H;
            double acc[TRN];
            float ab[TRN];
#pragma unroll
            for (int t = 0; t < TRN; ++t) { acc[t] = 0.0; ab[t] = 0.0f; }
            const int k1 = min(nbH, (sl + 1) * bps) * QK;
#pragma unroll 2
            for (int k = sl * bps * QK + lane * 8; k < k1; k += QK) {
                const uint4 wv = ld_stream_v4(row + k);
                const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
                for (int t = 0; t < TRN; ++t) {
                    if (t < nt) {
                        const uint4 xv = __ldg(reinterpret_cast<const uint4 *>(a.x + (size_t)(t0 + t) * a.H + k));
                        const uint32_t xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float x0 = bf16lo(xs[q]), x1 = bf16hi(xs[q]);
                            const float w0 = bf16lo(ws[q]), w1 = bf16hi(ws[q]);
                            acc[t] += (double)__fmaf_rn(x1, w1, __fmul_rn(x0, w0));
                            ab[t] = __fmaf_rn(fabsf(x0), fabsf(w0), __fmaf_rn(fabsf(x1), fabsf(w1), ab[t]));
                        }
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < TRN; ++t) {
                const double sm_ = warp_sum(acc[t]);
                const float sa = warp_sum(ab[t]);
                if (lane == 0) {
                    psum[((rr * nTR + tc) * 8 + sl) * DK_TR + t] = sm_;
                    pabs[((rr * nTR + tc) * 8 + sl) * DK_TR + t] = sa;
                }
            }
        }
        cons_bar();
        // (row, token chunk) w: lane t < DK_TR adds the slices of token 4 tc + t
        if (w < nr * nTR && lane < DK_TR) {
            const int rr = w / nTR, tc = w % nTR, t = tc * DK_TR + lane;
            if (t < a.T) {
                const int e = c + G * (j0 + rr);
                double sv = 0.0;
                float sa = 0.0f;
                for (int sl = 0; sl < S; ++sl) {
                    sv += psum[((rr * nTR + tc) * 8 + sl) * DK_TR + lane];
                    sa += pabs[((rr * nTR + tc) * 8 + sl) * DK_TR + lane];
                }
                a.logits[(size_t)t * a.E + e] = a.bias ? __dadd_rn(sv, (double)a.bias[e]) : sv;
                a.labs[(size_t)t * a.E + e] = sa;
            }
        }
        cons_bar();
        if (w == 0 && lane == 0) red_release_add(&a.ctl->route_done, (unsigned)(nr * nTR));
    }
    // int16 x: blocks v = c + G * j of the T * nbH blocks, one warp each
    int done = 0;
    for (int v = c + G * w; v < a.T * nbH; v += G * DK_CW) {
        dk_quantize_x(a, v / nbH, v % nbH);
        ++done;
    }
    __syncwarp();
    if (done && lane == 0) red_release_add(&a.ctl->route_done, (unsigned)done);
}

// ---------------------------------------------------------------------------------------
// Dot products of one piece

// One Q2_K tile (lane = row of the tile) with NT tokens' int16 activations of its block.
// PER32 = false: one scale per 256-block (xs_scale[t] given); the four bit planes keep
//   separate integer accumulators (unshifted) that are joined exactly at the end.
// PER32 = true: one scale per 32 activations (sc32[t][g]); each 32-group is joined and
//   scaled in fp32.
// q: int16 activations of the block (256 values); qs: their 16 sub-block sums.
// Activation operands of the Q2_K dot: in shared memory (32-bit addresses) or through the
// generic address space.
template <bool SMEM>
__device__ __forceinline__ uint4 act_v4(uintptr_t a) {
    if (SMEM) return lds_v4((uint32_t)a);
    return *reinterpret_cast<const uint4 *>(a);
}
template <bool SMEM>
__device__ __forceinline__ int act_i32(uintptr_t a) {
    if (SMEM) return (int)lds_u32((uint32_t)a);
    return *reinterpret_cast<const int *>(a);
}
template <bool SMEM>
__device__ __forceinline__ float act_f32(uintptr_t a) {
    if (SMEM) return __uint_as_float(lds_u32((uint32_t)a));
    return *reinterpret_cast<const float *>(a);
}

template <int NT, bool PER32, bool SMEM = false>
__device__ __forceinline__ void q2k_tile_dot(uint32_t tile, const uintptr_t (&q)[NT], const uintptr_t (&qs)[NT],
                                             const uintptr_t (&sc32)[NT], const float (&xs_scale)[NT], float (&acc)[NT]) {
    const int lane = threadIdx.x & 31;
    const uint4 scv = lds_v4(tile + TILE_SC + lane * 16);
    const uint32_t dm = lds_u32(tile + TILE_DM + lane * 4);
    const float d = h2f(dm), dmin = h2f(dm >> 16);
    int iscj[NT][4];
    int imn[NT];
    float facc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        imn[t] = 0;
        facc[t] = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) iscj[t][j] = 0;
    }
    // the two 128-weight halves run as a loop (not unrolled): half the code, which keeps
    // the instruction working set of the SM's warps small
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
        const uint4 qa = lds_v4(tile + TILE_QS + (uint32_t)(2 * hh) * 512 + lane * 16);
        const uint4 qb = lds_v4(tile + TILE_QS + (uint32_t)(2 * hh + 1) * 512 + lane * 16);
        const uint32_t sw0 = hh ? scv.z : scv.x, sw1 = hh ? scv.w : scv.y;   // scale bytes of sub-blocks 8hh..8hh+7
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int gsc[NT], gmn[NT];
#pragma unroll
            for (int t = 0; t < NT; ++t) { gsc[t] = 0; gmn[t] = 0; }
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
                const uint4 qw = cc ? qb : qa;
                const int sl = 2 * j + cc;                     // sub-block of (chunk 2hh + cc, plane j) within the half
                const int sb = 8 * hh + sl;
                const int base = 128 * hh + 32 * j + 16 * cc;  // its first weight
                const uint32_t mask = 0x03030303u << (2 * j);
                const uint32_t m0 = qw.x & mask, m1 = qw.y & mask, m2 = qw.z & mask, m3 = qw.w & mask;
                const uint32_t sbyte = ((sl < 4 ? sw0 : sw1) >> (8 * (sl & 3))) & 0xFFu;
                const int s_sc = (int)(sbyte & 0xFu), s_mn = (int)(sbyte >> 4);
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const uint4 xa = act_v4<SMEM>(q[t] + 2 * base);
                    const uint4 xb = act_v4<SMEM>(q[t] + 2 * base + 16);
                    // plane j stays in place (byte = q * 4^j); the sum carries the factor 4^j
                    int dd = dp2a_lo((int)xa.x, m0, 0);
                    dd = dp2a_hi((int)xa.y, m0, dd);
                    dd = dp2a_lo((int)xa.z, m1, dd);
                    dd = dp2a_hi((int)xa.w, m1, dd);
                    dd = dp2a_lo((int)xb.x, m2, dd);
                    dd = dp2a_hi((int)xb.y, m2, dd);
                    dd = dp2a_lo((int)xb.z, m3, dd);
                    dd = dp2a_hi((int)xb.w, m3, dd);
                    const int xsum = act_i32<SMEM>(qs[t] + 4 * sb);
                    if (PER32) {
                        gsc[t] += s_sc * dd;
                        gmn[t] += s_mn * xsum;
                    } else {
                        iscj[t][j] += s_sc * dd;
                        imn[t] += s_mn * xsum;
                    }
                }
            }
            if (PER32) {
                const float dj = d * (1.0f / (float)(1 << (2 * j)));
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    facc[t] = fmaf(act_f32<SMEM>(sc32[t] + 4 * (4 * hh + j)), fmaf(dj, (float)gsc[t], -dmin * (float)gmn[t]),
                                   facc[t]);
            }
        }
    }
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        if (PER32) {
            acc[t] += facc[t];
        } else {
            const int isc = iscj[t][0] + (iscj[t][1] >> 2) + (iscj[t][2] >> 4) + (iscj[t][3] >> 6);
            acc[t] = fmaf(xs_scale[t], fmaf(d, (float)isc, -dmin * (float)imn[t]), acc[t]);
        }
    }
}

// Dense bf16 piece: warp handles row `row`, inputs [k0, k0 + len) (len <= 1024, multiple of
// 8); activations of token t start at act + t * ld.  Lane t of the result holds token t's sum.
// TC > 0: the token count is TC, known at compile time.
template <bool ACT_F32, bool XSMEM = false, int TC = 0>
__device__ __forceinline__ float dense_seg_dot(uint32_t rowbase, int k0, int len, const void *act, int ld, int T_,
                                               uint32_t xs_smem = 0) {
    const int lane = threadIdx.x & 31;
    const int T = TC > 0 ? TC : T_;
    uint4 wv[4];
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int k = it * 256 + lane * 8;
        wv[it] = k < len ? lds_v4(rowbase + (uint32_t)(k0 + k) * 2) : make_uint4(0, 0, 0, 0);
    }
    float mine = 0.0f;
    for (int t = 0; t < T; ++t) {
        float p = 0.0f;
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int k = it * 256 + lane * 8;
            if (k < len) {
                float xv[8];
                if (ACT_F32) {
                    float4 x0, x1;
                    if (XSMEM) {
                        const uint32_t xa = xs_smem + (uint32_t)((t * ld + k0 + k) * 4);
                        const uint4 r0 = lds_v4(xa), r1 = lds_v4(xa + 16);
                        x0 = make_float4(__uint_as_float(r0.x), __uint_as_float(r0.y), __uint_as_float(r0.z), __uint_as_float(r0.w));
                        x1 = make_float4(__uint_as_float(r1.x), __uint_as_float(r1.y), __uint_as_float(r1.z), __uint_as_float(r1.w));
                    } else {
                        const float *xp = reinterpret_cast<const float *>(act) + (size_t)t * ld + k0 + k;
                        x0 = *reinterpret_cast<const float4 *>(xp);
                        x1 = *reinterpret_cast<const float4 *>(xp + 4);
                    }
                    xv[0] = x0.x; xv[1] = x0.y; xv[2] = x0.z; xv[3] = x0.w;
                    xv[4] = x1.x; xv[5] = x1.y; xv[6] = x1.z; xv[7] = x1.w;
                } else {
                    uint4 xr;
                    if (XSMEM) {
                        xr = lds_v4(xs_smem + (uint32_t)((t * ld + k0 + k) * 2));
                    } else {
                        const __nv_bfloat16 *xp = reinterpret_cast<const __nv_bfloat16 *>(act) + (size_t)t * ld + k0 + k;
                        xr = __ldg(reinterpret_cast<const uint4 *>(xp));
                    }
                    xv[0] = bf16lo(xr.x); xv[1] = bf16hi(xr.x); xv[2] = bf16lo(xr.y); xv[3] = bf16hi(xr.y);
                    xv[4] = bf16lo(xr.z); xv[5] = bf16hi(xr.z); xv[6] = bf16lo(xr.w); xv[7] = bf16hi(xr.w);
                }
                const uint32_t ws[4] = {wv[it].x, wv[it].y, wv[it].z, wv[it].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    p = fmaf(bf16lo(ws[i]), xv[2 * i], p);
                    p = fmaf(bf16hi(ws[i]), xv[2 * i + 1], p);
                }
            }
        }
        p = warp_sum(p);
        if (lane == t) mine = p;
    }
    return mine;
}

// ---------------------------------------------------------------------------------------
// Consumer warp state of the unit in progress
struct ConsState {
    float acc[2][DK_TU];   // Q2_K units: per set and token, lane = row
    float pd[2];           // dense units: per set, lane t = token t
};

// G tile: the group's tokens' records in the slot's activation area (staged) or in global
// memory.
template <int NT, bool STAGED>
__device__ __forceinline__ void g_tile(const DecArgs &a, const DecTable &tb, uint32_t slot, uint32_t tile, int grp, int b,
                                       int set, ConsState &cs) {
    const DecPlan &pl = a.pl;
    const int p0 = tb.grp_p0[grp];
    uintptr_t q[NT], qs[NT], sc32[NT];
    float xsc[NT], acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const uintptr_t rec = STAGED ? (uintptr_t)(slot + (uint32_t)(t * pl.xrec))
                                     : reinterpret_cast<uintptr_t>(a.xrec + (size_t)tb.pair_tok[p0 + t] * pl.xrec);
        q[t] = rec + (uintptr_t)b * QK * 2;
        qs[t] = rec + pl.xs_off + (uintptr_t)b * 64;
        sc32[t] = 0;
        xsc[t] = act_f32<STAGED>(rec + pl.xc_off + (uintptr_t)b * 4);
        acc[t] = 0.0f;
    }
    q2k_tile_dot<NT, false, STAGED>(tile, q, qs, sc32, xsc, acc);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        if (set == 0) cs.acc[0][t] += acc[t];
        else cs.acc[1][t] += acc[t];
    }
}

// D tile: the group's pairs' h records in the slot's activation area (staged) or in global
// memory.
template <int NT, bool STAGED>
__device__ __forceinline__ void d_tile(const DecArgs &a, const DecTable &tb, uint32_t slot, uint32_t tile, int grp, int b,
                                       int set, ConsState &cs) {
    const DecPlan &pl = a.pl;
    const int p0 = tb.grp_p0[grp];
    uintptr_t q[NT], qs[NT], sc32[NT];
    float xsc[NT], acc[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const uintptr_t rec = STAGED ? (uintptr_t)(slot + (uint32_t)(t * pl.hrec))
                                     : reinterpret_cast<uintptr_t>(a.hrec + (size_t)(p0 + t) * pl.hrec);
        q[t] = rec + (uintptr_t)b * QK * 2;
        qs[t] = rec + pl.hs_off + (uintptr_t)b * 64;
        sc32[t] = rec + pl.hc_off + (uintptr_t)b * 32;
        xsc[t] = 0.0f;
        acc[t] = 0.0f;
    }
    q2k_tile_dot<NT, true, STAGED>(tile, q, qs, sc32, xsc, acc);
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        if (set == 0) cs.acc[0][t] += acc[t];
        else cs.acc[1][t] += acc[t];
    }
}

// Compute warp w's share of piece pi of unit un held in slot `slot`; `staged`: the piece
// carries the activations of its SD or D unit (the producer found the unit's inputs ready).
// T1: the launch has one token (every group has one token; the dense dots know T = 1), the
// build whose code holds only those paths.
template <bool T1>
__device__ __forceinline__ void consume_piece(const DecArgs &a, const DecTable &tb, const Unit &un, int pi, uint32_t slot, int w,
                                              bool staged, ConsState &cs) {
    const DecPlan &pl = a.pl;
    if (un.type == U_SG || un.type == U_SD) {
        const int R = un.type == U_SG ? pl.RSG : pl.RSD, S = 16 / R;
        const int K = un.type == U_SG ? a.H : a.Is;
        const int row = w / S, seg = w % S;
        const int len = K / S, k0 = seg * len;
        const uint32_t rowbase = slot + DK_WOFF + (uint32_t)row * K * 2;
        float v;
        if (un.type == U_SD) {
            if (staged) v = dense_seg_dot<true, true, T1 ? 1 : 0>(rowbase, k0, len, a.hs, a.Is, a.T, slot);
            else v = dense_seg_dot<true, false, T1 ? 1 : 0>(rowbase, k0, len, a.hs, a.Is, a.T);
        }
        else if (pl.stage_sg) v = dense_seg_dot<false, true, T1 ? 1 : 0>(rowbase, k0, len, a.x, a.H, a.T, slot);
        else v = dense_seg_dot<false, false, T1 ? 1 : 0>(rowbase, k0, len, a.x, a.H, a.T);
        cs.pd[pi] = v;
        return;
    }
    const int nt = tb.grp_nt[un.a];
    if (un.type == U_G) {
        const int mat = pi / pl.ppGm, b0 = (pi % pl.ppGm) * 16;
        const int b = b0 + w;
        if (b >= pl.nbH) return;
        const uint32_t tile = slot + DK_WOFF + (uint32_t)w * TILE_BYTES;
        if (pl.stage_g) {
            if (T1 || nt == 1) g_tile<1, true>(a, tb, slot, tile, un.a, b, mat, cs);
            else g_tile<2, true>(a, tb, slot, tile, un.a, b, mat, cs);
        } else {
            if (T1 || nt == 1) g_tile<1, false>(a, tb, slot, tile, un.a, b, mat, cs);
            else g_tile<2, false>(a, tb, slot, tile, un.a, b, mat, cs);
        }
    } else {
        const int tq = pi * 16 + w;
        if (tq >= 2 * pl.nbI) return;
        const int rl = tq / pl.nbI, b = tq % pl.nbI;
        const uint32_t tile = slot + DK_WOFF + (uint32_t)w * TILE_BYTES;
        if (staged) {
            if (T1 || nt == 1) d_tile<1, true>(a, tb, slot, tile, un.a, b, rl, cs);
            else d_tile<2, true>(a, tb, slot, tile, un.a, b, rl, cs);
        } else {
            if (T1 || nt == 1) d_tile<1, false>(a, tb, slot, tile, un.a, b, rl, cs);
            else d_tile<2, false>(a, tb, slot, tile, un.a, b, rl, cs);
        }
    }
}

// Partials of a finished unit into part[] (layout by unit kind):
//   Q2_K: [set][warp][token < DK_TU][lane]     dense: [set][warp][token < 32]
__device__ __forceinline__ void write_partials(const Unit &un, float *part, int w, const ConsState &cs) {
    const int lane = threadIdx.x & 31;
    if (un.type == U_SG || un.type == U_SD) {
        part[(0 * DK_CW + w) * 32 + lane] = cs.pd[0];
        part[(1 * DK_CW + w) * 32 + lane] = cs.pd[1];
    } else {
#pragma unroll
        for (int s = 0; s < 2; ++s)
#pragma unroll
            for (int t = 0; t < DK_TU; ++t) part[((s * DK_CW + w) * DK_TU + t) * 32 + lane] = cs.acc[s][t];
    }
}

// ---------------------------------------------------------------------------------------
// Scheduler: routing table

__device__ __forceinline__ void build_table(const DecArgs &a, DecTable &tb) {
    const int lane = threadIdx.x & 31;
    const int E = a.E, k = a.k, P = a.T * a.k;
    for (int e = lane; e < E; e += 32) tb.mask[e] = 0u;
    __syncwarp();
    for (int p = lane; p < P; p += 32) atomicOr(&tb.mask[tb.topi[p]], 1u << (p / k));
    __syncwarp();
    int base = 0, gbase = 0;
    for (int c = 0; c < E; c += 32) {
        const int e = c + lane;
        const unsigned m = e < E ? tb.mask[e] : 0u;
        const int cnt = __popc(m), ng = (cnt + DK_TU - 1) / DK_TU;
        int ic = cnt, ig = ng;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int nc = __shfl_up_sync(0xffffffffu, ic, o), ngv = __shfl_up_sync(0xffffffffu, ig, o);
            if (lane >= o) { ic += nc; ig += ngv; }
        }
        const int off = base + ic - cnt, g0 = gbase + ig - ng;
        if (e < E) tb.off[e] = off;
        for (int q = 0; q < ng; ++q) {
            tb.grp_e[g0 + q] = (short)e;
            tb.grp_p0[g0 + q] = (short)(off + q * DK_TU);
            tb.grp_nt[g0 + q] = (signed char)min(DK_TU, cnt - q * DK_TU);
        }
        base += __shfl_sync(0xffffffffu, ic, 31);
        gbase += __shfl_sync(0xffffffffu, ig, 31);
    }
    if (lane == 0) {
        tb.off[E] = base;
        tb.NG = gbase;
    }
    __syncwarp();
    for (int p = lane; p < P; p += 32) {
        const int e = tb.topi[p], t = p / k, j = p - t * k;
        const int pos = tb.off[e] + __popc(tb.mask[e] & ((1u << t) - 1u));
        tb.pair_tok[pos] = (short)t;
        tb.pair_slot[pos] = (signed char)j;
        tb.inv[p] = (short)pos;
    }
    __syncwarp();
    if (lane == 0) {
        const DecPlan &pl = a.pl;
        tb.nG = tb.NG * pl.RGI;
        tb.nD = tb.NG * pl.RPH;
        tb.uC = pl.nA + tb.nG + pl.nB;
        tb.uC1 = tb.uC + pl.nC0;
        tb.uEnd = tb.uC1 + tb.nD + pl.nC1;
        tb.ok = 1;
    }
    __syncwarp();
}

// The table for T <= DK_TRED tokens (then every expert has at most DK_TU tokens, one group
// each): lane p ranks pair p by (expert, token) among the P <= 32 pairs.  The per-expert
// masks and offsets of all E experts are not needed by the work units (see publish_small).
__device__ __forceinline__ void build_table_small(const DecArgs &a, DecTable &tb) {
    const int lane = threadIdx.x & 31;
    const int k = a.k, P = a.T * a.k;
    const int e = lane < P ? tb.topi[lane] : 0x7fff;
    const int t = lane < P ? lane / k : 0;
    const int key = lane < P ? e * MAX_DECODE_T + t : 0x7fffffff;
    int pos = 0;
    for (int q = 0; q < P; ++q) pos += __shfl_sync(0xffffffffu, key, q) < key;
    if (lane < P) {
        tb.pair_tok[pos] = (short)t;
        tb.pair_slot[pos] = (signed char)(lane - t * k);
        tb.inv[lane] = (short)pos;
        tb.grp_e[pos] = (short)e;   // expert of each position, compacted below
    }
    __syncwarp();
    const int pe = lane < P ? tb.grp_e[lane] : -1;
    const int prev = __shfl_up_sync(0xffffffffu, pe, 1);
    const bool first = lane < P && (lane == 0 || prev != pe);
    const unsigned bal = __ballot_sync(0xffffffffu, first);
    const int nxt = __shfl_down_sync(0xffffffffu, pe, 1);
    __syncwarp();
    if (first) {
        const int g = __popc(bal & ((1u << lane) - 1u));
        tb.grp_e[g] = (short)pe;
        tb.grp_p0[g] = (short)lane;
        tb.grp_nt[g] = (signed char)((lane + 1 < P && nxt == pe) ? 2 : 1);
    }
    __syncwarp();
    if (lane == 0) {
        const DecPlan &pl = a.pl;
        tb.NG = __popc(bal);
        tb.nG = tb.NG * pl.RGI;
        tb.nD = tb.NG * pl.RPH;
        tb.uC = pl.nA + tb.nG + pl.nB;
        tb.uC1 = tb.uC + pl.nC0;
        tb.uEnd = tb.uC1 + tb.nD + pl.nC1;
        tb.ok = 1;
    }
    __syncwarp();
}

// CTA 0, after build_table_small: the routing outputs (top-k, offsets of all E experts,
// permutation, active experts).
__device__ __forceinline__ void publish_small(const DecArgs &a, const DecTable &tb) {
    const int lane = threadIdx.x & 31;
    const int P = a.T * a.k;
    if (lane < P) {
        a.ro.topk_idx[lane] = tb.topi[lane];
        a.ro.topk_w[lane] = tb.topw[lane];
        a.ro.sorted_token[lane] = tb.pair_tok[lane];
        a.ro.sorted_slot[lane] = tb.pair_slot[lane];
        a.ro.inv_pos[lane] = tb.inv[lane];
    }
    const int pe = lane < P ? tb.topi[lane] : 0x7fffffff;
    for (int e = 0; e <= a.E; e += 32) {
        int off = 0;
        for (int q = 0; q < P; ++q) off += __shfl_sync(0xffffffffu, pe, q) < e + lane;
        if (e + lane <= a.E) a.ro.offsets[e + lane] = off;
    }
    for (int g = lane; g < tb.NG; g += 32) a.ro.active[g] = tb.grp_e[g];
    if (lane == 0) *a.ro.n_active = tb.NG;
}

// CTA 0 publishes the routing: top-k (where this CTA computed it), offsets, permutation,
// active experts.
__device__ __forceinline__ void publish_routing(const DecArgs &a, const DecTable &tb, bool with_topk) {
    const int lane = threadIdx.x & 31;
    const int E = a.E, P = a.T * a.k;
    if (with_topk)
        for (int p = lane; p < P; p += 32) {
            a.ro.topk_idx[p] = tb.topi[p];
            a.ro.topk_w[p] = tb.topw[p];
        }
    for (int e = lane; e <= E; e += 32) a.ro.offsets[e] = tb.off[e];
    for (int p = lane; p < P; p += 32) {
        a.ro.sorted_token[p] = tb.pair_tok[p];
        a.ro.sorted_slot[p] = tb.pair_slot[p];
        a.ro.inv_pos[p] = tb.inv[p];
    }
    int nact = 0;
    for (int c = 0; c < E; c += 32) {
        const int e = c + lane;
        const bool act = e < E && tb.mask[e] != 0u;
        const unsigned bal = __ballot_sync(0xffffffffu, act);
        if (act) a.ro.active[nact + __popc(bal & ((1u << lane) - 1u))] = e;
        nact += __popc(bal);
    }
    if (lane == 0) *a.ro.n_active = nact;
}

template <bool TR, bool T1>
__device__ __forceinline__ void scheduler_role(const DecArgs &a, DecSmem &sm) {
    const int lane = threadIdx.x & 31;
    DecTable &tb = sm.tb;
    const int T = a.T, k = a.k, E = a.E;
    const bool redundant = T1 || T <= DK_TRED;
    bool ok = dk_poll_warp(a, &a.ctl->route_done, (unsigned)a.pl.n_route_items, a.wait_ns);
    if (TR && a.trace && lane == 0) dk_trace_cta(a)[2] = gtimer();
    // few tokens: every CTA selects every token itself, into its table; otherwise tokens are
    // claimed from a counter and published.  One call site: the selection is large code.
    for (int it = 0; ok; ++it) {
        int t = it;
        if (!redundant) {
            if (lane == 0) t = (int)atomicAdd(&a.ctl->topk_next, 1u);
            t = __shfl_sync(0xffffffffu, t, 0);
        }
        if (t >= T) break;
        warp_topk_fast<8>(a.logits + (size_t)t * E, a.labs + (size_t)t * E, E, k, BOUND_PAIR, a.H,
                          a.x + (size_t)t * a.H, a.wr, a.bias,
                          redundant ? tb.topi + t * k : a.ro.topk_idx + (size_t)t * k,
                          redundant ? tb.topw + t * k : a.ro.topk_w + (size_t)t * k,
                          (!redundant || blockIdx.x == 0) ? a.ro.fallbacks : nullptr, sm.tk_v, sm.tk_m,
                          (TR && a.trace && redundant && blockIdx.x == 0 && t == 0) ? dk_trace_tail(a) + 8 : nullptr);
        if (!redundant) dk_count(&a.ctl->topk_done);
    }
    if (ok && !redundant) {
        ok = dk_poll_warp(a, &a.ctl->topk_done, (unsigned)T, a.wait_ns);
        if (ok)
            for (int p = lane; p < T * k; p += 32) {
                tb.topi[p] = __ldcg(a.ro.topk_idx + p);
                tb.topw[p] = __ldcg(a.ro.topk_w + p);
            }
        __syncwarp();
    }
    if (TR && a.trace && lane == 0) dk_trace_cta(a)[3] = gtimer();
    if (ok) {
        // selection maps a non-finite logit to an in-range expert, so indices are in range
        if (redundant) build_table_small(a, tb);
        else build_table(a, tb);
    } else if (lane == 0) {
        tb.ok = 0;
        tb.NG = 0;
        tb.nG = tb.nD = 0;
        tb.uC = tb.uC1 = tb.uEnd = a.pl.nA;
    }
    __syncwarp();
    if (TR && a.trace && lane == 0) {
        dk_trace_cta(a)[4] = gtimer();
        if (blockIdx.x == 0) {
            unsigned long long *b = dk_trace_tail(a);
            b[0] = (unsigned long long)a.pl.nA;
            b[1] = (unsigned long long)tb.uC;
            b[2] = (unsigned long long)tb.uC1;
            b[3] = (unsigned long long)tb.uEnd;
            b[4] = (unsigned long long)tb.NG;
        }
    }
    if (lane == 0) mbar_arrive(smem_u32(&sm.route_bar));
    // the routing outputs, after the work has been released
    if (ok && blockIdx.x == 0) {
        if (redundant) publish_small(a, tb);
        else publish_routing(a, tb, false);
    }
}

// ---------------------------------------------------------------------------------------
// Producer

template <bool TR>
__device__ __forceinline__ void producer_role(const DecArgs &a, DecSmem &sm, uint32_t ring) {
    const int lane = threadIdx.x & 31;
    const DecPlan &pl = a.pl;
    DecTable &tb = sm.tb;
    int i = 0;   // copies issued (ring position; 32-bit: the slot and phase divisions stay cheap)
    if (!a.route_only) {
        bool routed = false;
        int limit = pl.nA;    // units known before the routing (phase A)
        int d_ver = -1;       // expert group whose G units are known done (groups never decrease)
        bool sd_ver = false;  // every SG unit known done
        int u = 0, u_next = 0;
        if (lane == 0) {
            u = (int)atomicAdd(&a.ctl->next_unit, 1u);
            u_next = (int)atomicAdd(&a.ctl->next_unit, 1u);
        }
        u = __shfl_sync(0xffffffffu, u, 0);
        u_next = __shfl_sync(0xffffffffu, u_next, 0);
        for (;;) {
            if (u >= limit && !routed) {
                if (!dk_wait_warp(a, smem_u32(&sm.route_bar), 0)) break;
                // the int16 token records written by other CTAs' generic stores are read by
                // bulk copies (the async proxy) from here on
                asm volatile("fence.proxy.async.global;" ::: "memory");
                routed = true;
                limit = tb.uEnd;
            }
            if (u >= limit) break;
            if (lane == 0 && ld_relaxed(&a.ctl->abort)) u = -1;
            if (__shfl_sync(0xffffffffu, u, 0) < 0) break;
            const Unit un = decode_unit(pl, tb, u);
            if (TR && a.trace && lane == 0 && u < a.trace_units) {
                a.trace[4 * (size_t)u + 1] = gtimer();
                dk_trace_ext(a, u)[2] = blockIdx.x;
            }
            // An SD or D unit carries its inputs in its slots (where they fit), so its
            // consumers neither poll nor read them from global memory: the producer waits
            // until they are published (usually they are: they were computed a phase
            // earlier), then a proxy fence lets the bulk copies (async proxy) see the other
            // CTAs' generic writes.  Waiting here rather than in the consumers costs nothing
            // they would not wait anyway, and keeps the slow global-input path rare.
            bool ustage = false;
            if ((un.type == U_D && pl.stage_d) || (un.type == U_SD && pl.stage_sd)) {
                if (un.type == U_D ? un.a == d_ver : sd_ver) {
                    ustage = true;
                } else {
                    int ok = 0;
                    if (lane == 0) {
                        ok = un.type == U_D
                                 ? dk_poll(a, &a.ctl->grp_done[un.a], (unsigned)pl.RGI + (a.test_timeout ? 1u : 0u),
                                           a.test_timeout ? 2000000ll : a.wait_ns)
                                 : dk_poll(a, &a.ctl->sg_done, (unsigned)pl.nSG, a.wait_ns);
                        if (ok) asm volatile("fence.proxy.async.global;" ::: "memory");
                    }
                    if (!__shfl_sync(0xffffffffu, ok, 0)) break;   // timed out or aborted
                    ustage = true;
                    if (un.type == U_D) d_ver = un.a;
                    else sd_ver = true;
                }
            }
            if (TR && a.trace && lane == 0 && u < a.trace_units) dk_trace_ext(a, u)[2] = blockIdx.x | (ustage ? 0x10000u : 0u);
            const int np = unit_pieces(pl, un.type);
            bool fail = false;
            for (int pi = 0; pi < np; ++pi, ++i) {
                const int s = (int)(i % DK_NSLOT);
                if (i >= DK_NSLOT && !dk_wait_warp(a, smem_u32(&sm.empty[s]), (uint32_t)((i / DK_NSLOT - 1) & 1))) {
                    fail = true;
                    break;
                }
                const uint8_t *src;
                uint32_t bytes;
                piece_src(a, tb, un, pi, src, bytes);
                if (lane == 0) {
                    if (TR && a.trace && pi == 1 && u < a.trace_units) dk_trace_ext(a, u)[5] = gtimer();
                    sm.meta_unit[s] = u;
                    sm.meta_piece[s] = pi;
                    sm.meta_staged[s] = ustage ? 1 : 0;
                    sm.meta_un[s] = un;
                    sm.last_issue[s] = (int)i;
                    const uint32_t fb = smem_u32(&sm.full[s]), dst = ring + (uint32_t)s * DK_SLOT;
                    // the piece's activations go to the front of the slot: the group's token
                    // records (G) or every token's bf16 row (SG)
                    int nstage = 0;
                    uint32_t sbytes = 0;
                    if (un.type == U_G && pl.stage_g) {
                        nstage = tb.grp_nt[un.a];
                        sbytes = (uint32_t)(nstage * pl.xrec);
                    } else if (un.type == U_SG && pl.stage_sg) {
                        sbytes = (uint32_t)(a.T * a.H * 2);
                    } else if (ustage && un.type == U_D) {
                        nstage = tb.grp_nt[un.a];
                        sbytes = (uint32_t)(nstage * pl.hrec);
                    } else if (ustage) {
                        sbytes = (uint32_t)(a.T * a.Is * 4);
                    }
                    mbar_expect_tx(fb, bytes + sbytes);
                    if (un.type == U_G && pl.stage_g) {
                        const int p0 = tb.grp_p0[un.a];
                        for (int t = 0; t < nstage; ++t)
                            bulk_g2s(dst + (uint32_t)(t * pl.xrec), a.xrec + (size_t)tb.pair_tok[p0 + t] * pl.xrec,
                                     (uint32_t)pl.xrec, fb);
                    } else if (ustage && un.type == U_D) {
                        const int p0 = tb.grp_p0[un.a];
                        for (int t = 0; t < nstage; ++t)
                            bulk_g2s(dst + (uint32_t)(t * pl.hrec), a.hrec + (size_t)(p0 + t) * pl.hrec, (uint32_t)pl.hrec, fb);
                    } else if (ustage) {
                        bulk_g2s(dst, a.hs, sbytes, fb);
                    } else if (sbytes) {
                        bulk_g2s(dst, a.x, sbytes, fb);
                    }
                    bulk_g2s(dst + DK_WOFF, src, bytes, fb);
                }
                __syncwarp();
                // one slot in flight until this CTA's router rows are done: the rows' loads
                // then wait behind little streaming in the memory queues
                if (i == 0) {
                    if (!dk_wait_warp(a, smem_u32(&sm.items_bar), 0)) {
                        fail = true;
                        ++i;
                        break;
                    }
                    if (TR && a.trace && lane == 0) dk_trace_cta(a)[1] = gtimer();
                }
            }
            if (fail) break;
            u = u_next;
            if (lane == 0) u_next = (int)atomicAdd(&a.ctl->next_unit, 1u);
            u_next = __shfl_sync(0xffffffffu, u_next, 0);
        }
    }
    // end marker
    const int s = (int)(i % DK_NSLOT);
    if (i < DK_NSLOT || dk_wait_warp(a, smem_u32(&sm.empty[s]), (uint32_t)((i / DK_NSLOT - 1) & 1))) {
        if (lane == 0) {
            sm.meta_unit[s] = -1;
            sm.meta_piece[s] = 0;
            mbar_arrive(smem_u32(&sm.full[s]));
        }
    }
    __syncwarp();
}

// ---------------------------------------------------------------------------------------
// Consumers

template <bool TR, bool T1>
__device__ __forceinline__ void consumer_role(const DecArgs &a, DecSmem &sm, uint32_t ring) {
    const int lane = threadIdx.x & 31;
    const int w = (int)(threadIdx.x >> 5) - DK_W_CONS;
    const DecPlan &pl = a.pl;
    const DecTable &tb = sm.tb;
    route_rows_cta<T1>(a, sm, w);
    if (lane == 0) mbar_arrive(smem_u32(&sm.items_bar));
    // phase A units need no routing: the ring starts at once and waits for the routing
    // table at the first unit past phase A
    bool routed = false;
    bool sg_ok = false;
    int g_ok = -1;   // group whose G units are known to be done
    ConsState cs;
    unsigned long long t_unit = 0;   // trace: when this warp started the current unit
    int i = 0;
    int n_units = 0;
    bool alive = true;
    for (;; ++i) {
        const int s = (int)(i % DK_NSLOT);
        if (!dk_wait_warp(a, smem_u32(&sm.full[s]), (uint32_t)((i / DK_NSLOT) & 1))) { alive = false; break; }
        const int u = sm.meta_unit[s], pi = sm.meta_piece[s];
        if (u < 0) break;
        const bool staged = sm.meta_staged[s] != 0;
        if (TR && a.trace && w == 0 && lane == 0 && pi < 2 && u < a.trace_units) dk_trace_ext(a, u)[3 + pi] = gtimer();
        if (u >= pl.nA && !routed) {
            if (!dk_wait_warp(a, smem_u32(&sm.route_bar), 0)) { alive = false; break; }
            routed = true;
        }
        const Unit un = sm.meta_un[s];
        if (pi == 0) {
            if (un.type == U_SD && !sg_ok && !staged) {
                if (!dk_poll_warp(a, &a.ctl->sg_done, (unsigned)pl.nSG, a.wait_ns)) { alive = false; break; }
                sg_ok = true;
            }
            // a D unit needs the G units of its own group only (this CTA claims units in
            // increasing order, so the groups of its D units never decrease)
            if (un.type == U_D && un.a != g_ok && !staged) {
                const unsigned target = (unsigned)pl.RGI + (a.test_timeout ? 1u : 0u);
                if (!dk_poll_warp(a, &a.ctl->grp_done[un.a], target, a.test_timeout ? 2000000ll : a.wait_ns)) {
                    alive = false;
                    break;
                }
                g_ok = un.a;
            }
            if (TR && a.trace && w == 0 && lane == 0 && u < a.trace_units) a.trace[4 * (size_t)u + 2] = t_unit = gtimer();
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                cs.pd[q] = 0.0f;
#pragma unroll
                for (int t = 0; t < DK_TU; ++t) cs.acc[q][t] = 0.0f;
            }
        }
        consume_piece<T1>(a, tb, un, pi, ring + (uint32_t)s * DK_SLOT, w, staged, cs);
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.empty[s]));
        if (TR && a.trace && w == 0 && lane == 0 && pi == 0 && u < a.trace_units) dk_trace_ext(a, u)[6] = gtimer();
        if (pi == unit_pieces(pl, un.type) - 1) {
            if (TR && a.trace && w == 0 && lane == 0 && u < a.trace_units)
                a.trace[4 * (size_t)u] = (unsigned long long)u | ((gtimer() - t_unit) << 32);
            const int buf = n_units % DK_PBUF, use = n_units / DK_PBUF;
            if (use > 0 && !dk_wait_warp(a, smem_u32(&sm.pempty[buf]), (uint32_t)((use - 1) & 1))) {
                alive = false;
                break;
            }
            write_partials(un, sm.part[buf], w, cs);
            if (w == 0 && lane == 0) {
                sm.part_unit[buf] = u;
                sm.part_un[buf] = un;
                if (TR && a.trace && u < a.trace_units) dk_trace_ext(a, u)[0] = gtimer();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.pfull[buf]));
            ++n_units;
        }
    }
    if (lane == 0) sm.cons_pos[w] = (int)i;
    // end of both epilogue queues
    for (int n = n_units; alive && n < n_units + DK_PBUF; ++n) {
        const int buf = n % DK_PBUF, use = n / DK_PBUF;
        if (use == 0 || dk_wait_warp(a, smem_u32(&sm.pempty[buf]), (uint32_t)((use - 1) & 1))) {
            if (w == 0 && lane == 0) sm.part_unit[buf] = -1;
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.pfull[buf]));
        } else {
            alive = false;
        }
    }
}

// ---------------------------------------------------------------------------------------
// Epilogue

// y for one 64-row range of H, all tokens: S + sum_j o[inv_pos(t, j)] in slot order.
// Every load of a token is issued before the additions (they would otherwise be k + 1
// dependent L2 round trips per half), and the sum keeps the slot order.
template <bool T1>
__device__ __forceinline__ void combine_range(const DecArgs &a, const DecTable &tb, int range) {
    const int lane = threadIdx.x & 31;
    const int T = T1 ? 1 : a.T;
    for (int t = 0; t < T; ++t) {
        float v[2][MAX_TOPK + 1];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int row = range * DK_RANGE + h * 32 + lane;
            v[h][0] = a.Is > 0 ? __ldcg(a.s + (size_t)t * a.H + row) : 0.0f;
#pragma unroll
            for (int j = 0; j < MAX_TOPK; ++j)
                v[h][j + 1] = j < a.k ? __ldcg(a.o + (size_t)tb.inv[t * a.k + j] * a.H + row) : 0.0f;
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            float acc = v[h][0];
#pragma unroll
            for (int j = 0; j < MAX_TOPK; ++j)
                if (j < a.k) acc += v[h][j + 1];
            a.y[(size_t)t * a.H + range * DK_RANGE + h * 32 + lane] = acc;
        }
    }
}

// A down unit's rows of range r are written: count it at once (an acquire-release add,
// which publishes this warp's rows and, for the last unit of the range, makes every other
// unit's rows visible).  True for the unit that completes the range -- its SD units and one
// D unit per expert group --, whose epilogue warp then writes y for it, so the combine runs
// as the ranges finish instead of after a launch-wide count.
__device__ __forceinline__ bool epi_range_done(const DecArgs &a, const DecTable &tb, int r) {
    __syncwarp();
    int last = 0;
    if ((threadIdx.x & 31) == 0) {
        unsigned old;
        asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], 1;" : "=r"(old) : "l"(&a.ctl->rng_done[r]) : "memory");
        last = old + 1u == (unsigned)(a.pl.sd_per_range + tb.NG);
    }
    return __shfl_sync(0xffffffffu, last, 0) != 0;
}

// Finished units whose completion is not yet published: shared gate/up, and routed gate/up
// of one expert group.  (Down units count per range at once: see epi_range_done.)
struct EpiCounts {
    unsigned sg, gn;
    int grp;
};
__device__ __forceinline__ void red_relaxed_add(unsigned *p, unsigned v) {
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// One fence, then relaxed adds: each add after the fence is a release of the warp's earlier
// writes (ordered before the fence by __syncwarp), so the whole batch costs one fence.
__device__ __forceinline__ void epi_flush(const DecArgs &a, EpiCounts &c) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0 && (c.sg | c.gn)) {
        __threadfence();
        if (c.sg) red_relaxed_add(&a.ctl->sg_done, c.sg);
        if (c.gn) red_relaxed_add(&a.ctl->grp_done[c.grp], c.gn);
    }
    c.sg = c.gn = 0;
    __syncwarp();
}
__device__ __forceinline__ void epi_count_g(const DecArgs &a, EpiCounts &c, int grp) {
    if (c.gn && c.grp != grp) epi_flush(a, c);
    c.grp = grp;
    ++c.gn;
}
// SiLU with the fast exponential and division (within a few ulp; h is re-quantised to
// int16 right after).
__device__ __forceinline__ float silu_fast(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// Returns the 64-row range of H whose rows this unit (SD or D) wrote, else -1.
template <bool T1>
__device__ __forceinline__ int epilogue_unit(const DecArgs &a, const DecTable &tb, const Unit &un, const float *part_p, EpiCounts &cnt) {
    const int lane = threadIdx.x & 31;
    // partial sums by shared-memory address: part(i) = element i of the buffer
    const uint32_t pbase = smem_u32(part_p);
    auto part = [&](int i) { return lds_f32(pbase + 4u * (uint32_t)i); };
    const DecPlan &pl = a.pl;
    if (un.type == U_SG) {
        // lanes take the (row, token) pairs; the segments of a row add in order
        const int S = pl.SSG, T = T1 ? 1 : a.T;
        for (int i = lane; i < pl.RSG * T; i += 32) {
            const int r = i / T, t = i - r * T;
            float g = 0.0f, u = 0.0f;
            for (int s = 0; s < S; ++s) {
                g += part((0 * DK_CW + r * S + s) * 32 + t);
                u += part((1 * DK_CW + r * S + s) * 32 + t);
            }
            a.hs[(size_t)t * a.Is + un.a + r] = silu_fast(g) * u;
        }
        ++cnt.sg;
    } else if (un.type == U_SD) {
        const int S = pl.SSD, T = T1 ? 1 : a.T, R = pl.RSD;
        for (int i = lane; i < 2 * R * T; i += 32) {
            const int sr = i / T, t = i - sr * T, set = sr / R, r = sr - set * R;
            float v = 0.0f;
            for (int s = 0; s < S; ++s) v += part((set * DK_CW + r * S + s) * 32 + t);
            a.s[(size_t)t * a.H + un.a + set * R + r] = v;
        }
        return un.a / DK_RANGE;
    } else if (un.type == U_G) {
        const int nt = T1 ? 1 : tb.grp_nt[un.a], p0 = tb.grp_p0[un.a];
        for (int t = 0; t < nt; ++t) {
            float g = 0.0f, u = 0.0f;
#pragma unroll 4
            for (int w = 0; w < DK_CW; ++w) {
                g += part(((0 * DK_CW + w) * DK_TU + t) * 32 + lane);
                u += part(((1 * DK_CW + w) * DK_TU + t) * 32 + lane);
            }
            const float h = silu_fast(g) * u;
            // |h| of non-negative floats orders like its bits: one warp reduction
            const float amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(h))));
            const float inv = amax > 0.0f ? (float)DK_QMAX / amax : 0.0f;
            const int q = max(-DK_QMAX, min(DK_QMAX, __float2int_rn(h * inv)));
            int s16;   // the sums of the two 16-row sub-blocks
            if (lane < 16) s16 = __reduce_add_sync(0x0000FFFFu, q);
            else s16 = __reduce_add_sync(0xFFFF0000u, q);
            uint8_t *rec = a.hrec + (size_t)(p0 + t) * pl.hrec;
            reinterpret_cast<int16_t *>(rec)[un.b * 32 + lane] = (int16_t)q;
            if ((lane & 15) == 0) reinterpret_cast<int *>(rec + pl.hs_off)[un.b * 2 + (lane >> 4)] = s16;
            if (lane == 0) reinterpret_cast<float *>(rec + pl.hc_off)[un.b] = amax / (float)DK_QMAX;
        }
        epi_count_g(a, cnt, un.a);
    } else if (un.type == U_D) {
        const int nt = T1 ? 1 : tb.grp_nt[un.a], p0 = tb.grp_p0[un.a];
        for (int t = 0; t < nt; ++t) {
            const int p = p0 + t;
            const float wgt = tb.topw[tb.pair_tok[p] * a.k + tb.pair_slot[p]];
#pragma unroll
            for (int rl = 0; rl < 2; ++rl) {
                float v = 0.0f;
#pragma unroll 4
                for (int w = 0; w < DK_CW; ++w) v += part(((rl * DK_CW + w) * DK_TU + t) * 32 + lane);
                a.o[(size_t)p * a.H + un.b * DK_RANGE + rl * 32 + lane] = wgt * v;
            }
        }
        return un.b;
    }
    return -1;
}

// Units are taken in the order the consumers finished them.  Counts are published in
// batches: whenever no finished unit is waiting, and after every fourth unit.  The warp
// whose down unit completed a 64-row range writes y for it once the partial buffer is
// free again.
// Two epilogue warps: `which` = 0 (the epilogue warp) takes the units of partial buffer 0,
// which = 1 (the scheduler warp, once the routing is out) those of buffer 1; each in order.
template <bool TR, bool T1>
__device__ __forceinline__ void epilogue_role(const DecArgs &a, DecSmem &sm, int which) {
    const int lane = threadIdx.x & 31;
    EpiCounts cnt;
    cnt.sg = cnt.gn = 0;
    cnt.grp = 0;
    for (int n = which;; n += DK_PBUF) {
        const int buf = which;
        const uint32_t par = (uint32_t)((n / DK_PBUF) & 1), bar = smem_u32(&sm.pfull[buf]);
        int ready = lane == 0 ? (mbar_try_spin(bar, par) ? 1 : 0) : 0;
        if (!__shfl_sync(0xffffffffu, ready, 0)) {
            epi_flush(a, cnt);
            if (!dk_wait_warp(a, bar, par)) break;
        }
        const int u = sm.part_unit[buf];
        if (u < 0) break;
        if (TR && a.trace && lane == 0 && u < a.trace_units) dk_trace_ext(a, u)[1] = gtimer();
        const Unit un = sm.part_un[buf];
        const long long c0 = clock64();
        const int rng = epilogue_unit<T1>(a, sm.tb, un, sm.part[buf], cnt);
        if (TR && a.trace && lane == 0 && u < a.trace_units) {
            a.trace[4 * (size_t)u + 3] = gtimer();
            dk_trace_ext(a, u)[7] = (unsigned long long)(clock64() - c0);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sm.pempty[buf]));
        // a G unit's count goes out at once (the D units of its group wait for it); the
        // others in batches; a down unit's range count once its partial buffer is free (the
        // count's round trip to L2 does not hold the consumers), and the unit that completes
        // a range writes y for it
        if (cnt.gn || cnt.sg >= 4) epi_flush(a, cnt);
        if (rng >= 0 && epi_range_done(a, sm.tb, rng)) combine_range<T1>(a, sm.tb, rng);
    }
    epi_flush(a, cnt);
}

// ---------------------------------------------------------------------------------------

// 96 registers: the register file is split among the SM's four schedulers (16K each) and
// 19 warps put 5 on one of them, so 5 * 32 * r <= 16384 bounds r below 102.
// Builds: TR writes the timeline (handles created with DS4MOE_FLAG_TRACE), the others have
// no trace code at all; T1 (launches of one token) holds only the one-token consumer paths.
// Shorter hot loops measured faster: 72.0 us per single-token forward with the trace code
// in, 69.0 without it, 66.9 with the one-token build.
template <bool TR, bool T1>
__global__ void __maxnreg__(96) decode_kernel(DecArgs a) {
    extern __shared__ __align__(128) unsigned char dk_raw[];
    const uint32_t ring = (smem_u32(dk_raw) + 127u) & ~127u;
    unsigned char *base = dk_raw + (ring - smem_u32(dk_raw));
    DecSmem &sm = *reinterpret_cast<DecSmem *>(base + (size_t)DK_NSLOT * DK_SLOT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < DK_NSLOT; ++s) {
            mbar_init(smem_u32(&sm.full[s]), 1);
            mbar_init(smem_u32(&sm.empty[s]), DK_CW);
            sm.last_issue[s] = -1;
        }
        for (int b = 0; b < DK_PBUF; ++b) {
            mbar_init(smem_u32(&sm.pfull[b]), DK_CW);
            mbar_init(smem_u32(&sm.pempty[b]), 1);
        }
        mbar_init(smem_u32(&sm.route_bar), 1);
        mbar_init(smem_u32(&sm.items_bar), DK_CW);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (TR && a.trace) dk_trace_cta(a)[0] = gtimer();
    }
    __syncthreads();
    if (warp == DK_W_PROD) producer_role<TR>(a, sm, ring);
    else if (warp == DK_W_SCHED) {
        scheduler_role<TR, T1>(a, sm);
        epilogue_role<TR, T1>(a, sm, 1);
    } else if (warp == DK_W_EPI) epilogue_role<TR, T1>(a, sm, 0);
    else consumer_role<TR, T1>(a, sm, ring);
    __syncthreads();
    // drain: every bulk copy this CTA issued has landed before its shared memory is released
    // (copies at positions every consumer warp has passed have landed already)
    if (threadIdx.x == 0) {
        int passed = sm.cons_pos[0];
        for (int w = 1; w < DK_CW; ++w) passed = min(passed, sm.cons_pos[w]);
        for (int s = 0; s < DK_NSLOT; ++s) {
            const int li = sm.last_issue[s];
            if (li < passed) continue;
            const uint32_t bar = smem_u32(&sm.full[s]), par = (uint32_t)((li / DK_NSLOT) & 1);
            const unsigned long long t0 = gtimer();
            while (!mbar_try_spin(bar, par) && (long long)(gtimer() - t0) < a.wait_ns) {
            }
        }
        if (TR && a.trace) dk_trace_cta(a)[5] = gtimer();
    }
    // the CTA that leaves last resets the control words for the next launch
    __shared__ int s_last;
    if (threadIdx.x == 0) {
        __threadfence();
        s_last = atomicAdd(&a.ctl->exited, 1u) == gridDim.x - 1;
    }
    __syncthreads();
    if (s_last) {
        __threadfence();
        for (int g = threadIdx.x; g < DK_MAXP; g += blockDim.x) a.ctl->grp_done[g] = 0u;
        for (int r = threadIdx.x; r < DK_MAX_RANGES; r += blockDim.x) a.ctl->rng_done[r] = 0u;
        if (threadIdx.x == 0) {
            a.ctl->next_unit = 0u; a.ctl->route_done = 0u; a.ctl->topk_next = 0u; a.ctl->topk_done = 0u;
            a.ctl->sg_done = 0u; a.ctl->abort = 0u; a.ctl->exited = 0u;
        }
    }
    (void)lane;
}

}  // namespace ds4
