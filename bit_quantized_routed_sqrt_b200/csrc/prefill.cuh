// prefill.cuh -- the grouped tensor-core path of the layer (large T).
//
// After routing, the tokens of every active expert are contiguous rows of X (fp16, pair
// order) and the shared expert's tokens follow them.  Two persistent tcgen05 GEMM launches
// then run over a tile list (expert, 128 weight rows, up to N tokens):
//   GEMM1  g = W_gate x, u = W_up x  ->  H = silu(g) * u (fp16)
//   GEMM2  o = W_down h * routing weight  ->  O (fp32, one row per (token, slot) pair)
// and a combine launch sums each token's k rows of O plus its shared-expert row.
//
// Inside a GEMM CTA (one per SM, 16 warps), a ring of K-step stages, each holding the
// activation tile (TMA; GEMM1 up to 128 tokens, GEMM2 up to 256) and the weight tile
// (dequantised here, or TMA for the dense shared expert; GEMM1 gate|up, GEMM2 down) of one
// 64-wide K step (GEMM1 3 stages, GEMM2 4), and a ring of raw Q2_K block columns (bulk
// copies).  A stage has one `full` barrier, which the MMA warp waits on, and one `empty`
// barrier, which one MMA commit releases and every filling role waits on: a barrier wait
// costs a round trip to shared memory even when the phase is already complete, so the
// MMA warp does one wait and one commit per step.
//   warp 0     producer: TMA loads of the activation tile of each step (128B swizzle, only
//              the 64-row boxes holding the tile's tokens) and bulk copies of the raw Q2_K
//              tiles of each 256-wide block column;
//   warp 1     allocates tensor memory and issues tcgen05.mma into two accumulator
//              buffers, so the epilogue of one tile overlaps the next tile;
//   warp 2     loader: TMA loads of the weight tiles of the (dense fp16) shared expert, and
//              on every step the relay of the activation tile's arrival (its own tx
//              barrier) to the stage's full barrier;
//   warps 4-7  epilogue: tcgen05.ld of the accumulators, SwiGLU or routing-weight scaling;
//   warps 8-15 dequantise Q2_K -> fp16 straight into the swizzled K-major operand layout:
//              per 8 weights, w & (0x03030303 << 2j) keeps the quants of plane j in place,
//              prmt joins each byte with the exponent byte of 2^(10-2j) (fp16 2^(10-2j) + q),
//              one hsub2 gives q exactly, one hfma2 gives d*scale*q - dmin*min rounded once
//              to fp16.
// Every mbarrier wait is bounded; on a timeout the CTA records ETIMEOUT, drains its own
// copies and MMAs (waits that ignore the abort flag but have their own limit), frees
// tensor memory and returns.
// Each barrier is waited on by parity, which tells apart only two consecutive phases: every
// waiter therefore waits on every phase of its barriers in order.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "mbar.cuh"

namespace ds4 {

constexpr int PF_THREADS = 512;
constexpr int PF_BK = 64;                 // K per stage (one 128-byte swizzle atom of fp16)
constexpr int PF_M = 128;                 // weight rows per tile (MMA M)
constexpr int PF_N1 = 128;                // tokens per GEMM1 tile (two accumulators of 128 columns)
constexpr int PF_N2 = 256;                // tokens per GEMM2 tile (one accumulator of 256 columns)
constexpr int PF_A_BYTES = PF_M * PF_BK * 2;      // 16 KiB per weight matrix and step
constexpr int PF_BBOX = 64;               // activation rows per TMA box: a tile loads only the boxes its tokens need
constexpr int PF_BAR_BYTES = 512;

// Ring shapes of each GEMM.  GEMM1 dequantises two matrices (gate, up) per step for up to
// 128 tokens; GEMM2 one matrix (down) for up to 256 tokens, which halves the dequantisation
// per token where an expert has more than 128 tokens.
template <int G>
struct PfCfg {
    static constexpr int NMAT = G == 1 ? 2 : 1;
    static constexpr int BN = G == 1 ? PF_N1 : PF_N2;
    static constexpr int B_BYTES = BN * PF_BK * 2;           // activation tile: 16 or 32 KiB
    static constexpr int STAGES = G == 1 ? 3 : 4;            // K steps in flight
    static constexpr int RAWS = 2;                           // raw Q2_K block columns in flight
    static constexpr int ASTAGE_BYTES = NMAT * PF_A_BYTES;
    static constexpr int RAW_BYTES = (NMAT * 4 * TILE_BYTES + 1023) / 1024 * 1024;   // one 256-wide block column
    static constexpr int N_BARS = 4 * STAGES + 2 * RAWS + 5;
    static constexpr size_t SMEM = 1024 + STAGES * (B_BYTES + ASTAGE_BYTES) + RAWS * RAW_BYTES + PF_BAR_BYTES;
};
static_assert(PfCfg<1>::SMEM <= 227 * 1024 && PfCfg<2>::SMEM <= 227 * 1024, "shared memory per CTA");
static_assert(PfCfg<1>::N_BARS * 8 + 16 <= PF_BAR_BYTES && PfCfg<2>::N_BARS * 8 + 16 <= PF_BAR_BYTES, "barrier area");
static_assert(PF_N1 % PF_BBOX == 0 && PF_N2 % PF_BBOX == 0 && PF_BBOX % 8 == 0, "activation boxes tile the stage");

struct PfTile {
    int expert;    // expert id for Q2_K tiles; -1 for the shared expert
    int m0;        // first weight row (output feature)
    int b_row;     // first activation row (pair position, or P + token for the shared expert)
    int n;         // tokens in the tile
    int quant;     // 1: Q2_K weights (dequantised here); 0: fp16 weights by TMA
    int K;         // reduction length
    int pad0, pad1;
};

struct PfArgs {
    const PfTile *tiles;
    const int *n_tiles;
    int gemm;                 // 1 or 2
    const uint8_t *wq0, *wq1; // Q2_K tiled matrices (gate, up) or (down, -)
    size_t wq_bytes;          // bytes per expert matrix
    __half *out16;            // GEMM1 output (H rows), row stride ld_out
    float *out32;             // GEMM2 output (O rows), row stride ld_out
    int ld_out;
    const float *row_scale;   // GEMM2: weight of each activation row
    int *status;
    // checks: limits of what the kernel may touch (violations set EDEVICE, record, and skip)
    size_t out_elems;         // elements of out16 / out32
    size_t wq_total;          // bytes of each Q2_K weight array (all experts)
    int b_rows_total;         // rows of the activation tensor map
    int *dbg;                 // [8]: first violation (code, tile, a, b)
};

__device__ __forceinline__ void pf_report(const PfArgs &p, int code, int t, long long a, long long b) {
    set_status(p.status, ST_EDEVICE);
    if (p.dbg && atomicCAS(p.dbg, 0, code) == 0) {
        p.dbg[1] = t;
        p.dbg[2] = (int)a;
        p.dbg[3] = (int)(a >> 32);
        p.dbg[4] = (int)b;
        p.dbg[5] = (int)(b >> 32);
        p.dbg[6] = blockIdx.x;
        p.dbg[7] = threadIdx.x;
    }
}
// A tile every role can process: 1 <= n <= the GEMM's tile width, K a positive multiple of
// 256, rows in range.
__device__ __forceinline__ bool pf_tile_ok(const PfArgs &p, const PfTile &tile, int t) {
    const bool ok = tile.n >= 1 && tile.n <= (p.gemm == 1 ? PF_N1 : PF_N2) && tile.K >= QK && tile.K % QK == 0 && tile.K <= 16384 &&
                    tile.m0 >= 0 && tile.m0 % PF_M == 0 && tile.b_row >= 0 && tile.b_row < p.b_rows_total;
    if (!ok && threadIdx.x % 32 == 0) pf_report(p, 1, t, tile.n | ((long long)tile.K << 32), tile.b_row);
    return ok;
}

// ------------------------------------------------------------------ PTX wrappers
// Bounded wait for the completion of the barrier phase of the given parity (about two
// seconds); false on timeout (recorded) or when another role of the CTA gave up.  Roles off
// the critical path pass backoff_ns, so that while they wait they leave the issue slots to
// the dequantising warps.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort, int *status,
                                          int *dbg = nullptr, int who = 0, uint32_t iter = 0,
                                          unsigned backoff_ns = 0) {
    long long t0 = 0;
    for (int i = 0;; ++i) {
        if (mbar_try_spin(bar, parity)) return true;
        if (backoff_ns) __nanosleep(backoff_ns);
        if ((i & 15) == 15) {
            if (*abort) return false;
            const long long now = clock64();
            if (t0 == 0) {
                t0 = now;
            } else if (now - t0 > 4000000000ll) {
                set_status(status, ST_ETIMEOUT);
                if (dbg && atomicCAS(dbg, 0, 100 + who) == 0) {
                    dbg[1] = (int)iter;
                    dbg[2] = (int)parity;
                    dbg[3] = (int)(bar & 0xFFFF);
                    dbg[6] = blockIdx.x;
                    dbg[7] = threadIdx.x;
                }
                *abort = 1;
                return false;
            }
        }
    }
}
// Wait for copies or MMAs already issued by this CTA (they complete without any other
// role's help), ignoring the abort flag; bounded by about half a second.
__device__ __forceinline__ bool mbar_drain(uint32_t bar, uint32_t parity, int *status) {
    const long long t0 = clock64();
    for (int i = 0;; ++i) {
        if (mbar_try_spin(bar, parity)) return true;
        if ((i & 15) == 15 && clock64() - t0 > 1000000000ll) {
            set_status(status, ST_ETIMEOUT);
            return false;
        }
    }
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
    return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Instruction descriptor of kind::f16: fp16 A and B (K-major), fp32 D, M = 128, N.
__device__ __forceinline__ uint32_t f16_idesc(int N) {
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(PF_M >> 4) << 24);
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\ttcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// Constants of quant plane j (bits 2j, 2j+1 of each quant byte).  A byte masked in place
// holds q * 4^j; joined with the exponent byte 0x64 - 8j it is the fp16 number
// 2^(10-2j) + q exactly (the mantissa's unit at 2^(10-2j) is 4^-j), so subtracting the
// plane's base 2^(10-2j) leaves q exactly, without a shift.
struct Plane {
    uint32_t mask;    // 0x03030303 << 2j
    uint32_t magic;   // exponent byte of 2^(10-2j) in every byte
    uint32_t base;    // fp16 pair (2^(10-2j), 2^(10-2j))
};
__device__ __forceinline__ Plane plane_of(int j) {
    Plane pl;
    pl.mask = 0x03030303u << (2 * j);
    pl.magic = 0x64646464u - 0x08080808u * (uint32_t)j;
    pl.base = (0x6400u - 0x0800u * (uint32_t)j) * 0x10001u;
    return pl;
}
// 8 consecutive-l quants of one plane (bytes of words wa, wb) -> 8 fp16 weights
// d*sc*q - dmin*m, each rounded once.
__device__ __forceinline__ uint4 dequant8(uint32_t wa, uint32_t wb, const Plane &pl, __half2 dsc, __half2 ndmm) {
    const uint32_t qa = wa & pl.mask, qb = wb & pl.mask;
    const __half2 base = *reinterpret_cast<const __half2 *>(&pl.base);
    uint32_t o[4];
    const uint32_t src[4] = {prmt(qa, pl.magic, 0x5140u), prmt(qa, pl.magic, 0x7362u),
                             prmt(qb, pl.magic, 0x5140u), prmt(qb, pl.magic, 0x7362u)};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        __half2 q = __hsub2(*reinterpret_cast<const __half2 *>(&src[i]), base);
        __half2 w = __hfma2(q, dsc, ndmm);
        o[i] = *reinterpret_cast<uint32_t *>(&w);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

// ------------------------------------------------------------------ GEMM kernel
template <int G>
__global__ void __launch_bounds__(PF_THREADS, 1)
    pf_gemm_kernel(const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_a0,
                   const __grid_constant__ CUtensorMap tm_a1, PfArgs p) {
    using C = PfCfg<G>;
    extern __shared__ __align__(1024) uint8_t pf_smem_raw[];
    uint8_t *base = pf_smem_raw + ((1024u - (smem_u32(pf_smem_raw) & 1023u)) & 1023u);
    uint8_t *b_base = base;
    uint8_t *a_base = b_base + C::STAGES * C::B_BYTES;
    uint8_t *raw_base = a_base + C::STAGES * C::ASTAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(raw_base + C::RAWS * C::RAW_BYTES);
    // barrier map
    uint64_t *full = bars;                       // [S] 8 dequant warps + the loader's relay, every step
    uint64_t *empty = full + C::STAGES;          // [S] MMA commit
    uint64_t *full_b = empty + C::STAGES;        // [S] producer expect_tx + activation TMA bytes
    uint64_t *full_at = full_b + C::STAGES;      // [S] dense weight TMA: loader expect_tx + bytes
    uint64_t *raw_full = full_at + C::STAGES;    // [R] producer expect_tx + copy bytes
    uint64_t *raw_empty = raw_full + C::RAWS;    // [R] 8 dequant warps
    uint64_t *acc_full = raw_empty + C::RAWS;    // [2] MMA commit
    uint64_t *acc_empty = acc_full + 2;          // [2] 4 epilogue warps
    uint64_t *drain = acc_empty + 2;             // MMA commit at exit
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(drain + 2);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr bool g1 = G == 1;
    constexpr int nmat = C::NMAT;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(smem_u32(full + s), 8 + 1);
            mbar_init(smem_u32(empty + s), 1);
            mbar_init(smem_u32(full_b + s), 1);
            mbar_init(smem_u32(full_at + s), 1);
        }
        for (int r = 0; r < C::RAWS; ++r) {
            mbar_init(smem_u32(raw_full + r), 1);
            mbar_init(smem_u32(raw_empty + r), 8);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(acc_full + b), 1);
            mbar_init(smem_u32(acc_empty + b), 4);
        }
        mbar_init(smem_u32(drain), 1);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(tmem_holder))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const int n_tiles = *p.n_tiles;

    if (warp == 0) {
        // ------------------------------------------------------------------- producer
        // The whole warp runs the loop, so the copies' operands are warp-uniform values; one
        // elected lane issues each copy.
        uint32_t it = 0, rit = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
            const PfTile tile = p.tiles[t];
            if (!pf_tile_ok(p, tile, t)) { ok = false; *abort = 1; break; }
            const int nk = tile.K / PF_BK;
            const int nb = tile.K / QK;
            for (int ks = 0; ks < nk && ok; ++ks) {
                if (tile.quant && (ks & 3) == 0) {
                    const size_t last = ((size_t)(tile.m0 / TILE_ROWS + 3) * nb + (ks >> 2)) * TILE_BYTES +
                                        (size_t)tile.expert * p.wq_bytes + TILE_BYTES;
                    if (tile.expert < 0 || last > p.wq_total) {
                        if (lane == 0) pf_report(p, 2, t, (long long)last, tile.expert);
                        ok = false;
                        *abort = 1;
                        break;
                    }
                    const uint32_t r = rit % C::RAWS;
                    if (!(ok = mbar_wait(smem_u32(raw_empty + r), ((rit / C::RAWS) & 1) ^ 1, abort, p.status, p.dbg, 1, rit, 64))) break;
                    if (elect_one()) {
                        mbar_expect_tx(smem_u32(raw_full + r), (uint32_t)(nmat * 4 * TILE_BYTES));
                        for (int mat = 0; mat < nmat; ++mat) {
                            const uint8_t *w = (mat == 0 ? p.wq0 : p.wq1) + (size_t)tile.expert * p.wq_bytes;
                            for (int rg = 0; rg < 4; ++rg)
                                bulk_g2s(smem_u32(raw_base + r * C::RAW_BYTES + (mat * 4 + rg) * TILE_BYTES),
                                         w + ((size_t)(tile.m0 / TILE_ROWS + rg) * nb + (ks >> 2)) * TILE_BYTES,
                                         TILE_BYTES, smem_u32(raw_full + r));
                        }
                    }
                    __syncwarp();
                    ++rit;
                }
                // activation tile of this K step
                const uint32_t sb = it % C::STAGES;
                if (!(ok = mbar_wait(smem_u32(empty + sb), ((it / C::STAGES) & 1) ^ 1, abort, p.status, p.dbg, 2, it, 64))) break;
                // only the boxes of rows that hold this tile's tokens; the MMA reads N =
                // n rounded up to 16 rows, which never passes the last box
                const int nbox = (tile.n + PF_BBOX - 1) / PF_BBOX;
                if (elect_one()) {
                    mbar_expect_tx(smem_u32(full_b + sb), (uint32_t)(nbox * PF_BBOX * PF_BK * 2));
                    for (int j = 0; j < nbox; ++j)
                        tma_load_2d(smem_u32(b_base + sb * C::B_BYTES + j * PF_BBOX * PF_BK * 2), &tm_b, ks * PF_BK,
                                    tile.b_row + j * PF_BBOX, smem_u32(full_b + sb));
                }
                __syncwarp();
                ++it;
            }
        }
        if (!ok) {
            // make sure no copy of this CTA is still writing shared memory
            for (uint32_t i = it > C::STAGES ? it - C::STAGES : 0; i < it; ++i)
                mbar_drain(smem_u32(full_b + i % C::STAGES), (i / C::STAGES) & 1, p.status);
            for (uint32_t i = rit > C::RAWS ? rit - C::RAWS : 0; i < rit; ++i)
                mbar_drain(smem_u32(raw_full + i % C::RAWS), (i / C::RAWS) & 1, p.status);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------------- MMA
        // The whole warp runs the loop, so the MMA operands (descriptors, TMEM addresses) are
        // warp-uniform values; one elected lane issues each MMA and commit.
        uint32_t it = 0, tc = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
            const PfTile tile = p.tiles[t];
            if (!pf_tile_ok(p, tile, t)) break;
            const int nk = tile.K / PF_BK;
            const uint32_t b = tc & 1;
            if (!(ok = mbar_wait(smem_u32(acc_empty + b), ((tc >> 1) & 1) ^ 1, abort, p.status, p.dbg, 11, tc, 32))) break;
            tc_fence_after();
            const int N = (tile.n + 15) & ~15;
            const uint32_t idesc = f16_idesc(N);
            const uint32_t d0 = tmem + b * 256, d1 = tmem + b * 256 + 128;
            for (int ks = 0; ks < nk && ok; ++ks) {
                const uint32_t ss = it % C::STAGES;
                if (!(ok = mbar_wait(smem_u32(full + ss), (it / C::STAGES) & 1, abort, p.status, p.dbg, 12, it))) break;
                tc_fence_after();
                // descriptors of the stage's K = 16 slices: the start address field (in
                // 16-byte units, below 2^14 for any shared-memory address) advances by 2
                const uint64_t b0 = sw128_desc(smem_u32(b_base + ss * C::B_BYTES));
                const uint64_t a0 = sw128_desc(smem_u32(a_base + ss * C::ASTAGE_BYTES));
                const uint64_t a1 = a0 + (PF_A_BYTES >> 4);
                if (elect_one()) {
#pragma unroll
                    for (int kk = 0; kk < PF_BK / 16; ++kk) {
                        const uint32_t acc = (ks | kk) != 0;
                        tc_mma(d0, a0 + 2 * kk, b0 + 2 * kk, idesc, acc);
                        if (g1) tc_mma(d1, a1 + 2 * kk, b0 + 2 * kk, idesc, acc);
                    }
                    tc_commit(smem_u32(empty + ss));
                }
                __syncwarp();
                ++it;
            }
            if (ok && elect_one()) tc_commit(smem_u32(acc_full + b));
            __syncwarp();
            ++tc;
        }
        // every MMA issued by this warp has completed once the drain barrier fires
        if (elect_one()) tc_commit(smem_u32(drain));
        __syncwarp();
        mbar_drain(smem_u32(drain), 0, p.status);
    } else if (warp == 2) {
        // --------------------------------------------------------------------- loader
        if (lane == 0) {
            uint32_t it = 0;
            uint32_t dpar = 0, dany = 0;   // bit s: parity of the next dense fill of stage s; any fill yet
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                const PfTile tile = p.tiles[t];
                if (!pf_tile_ok(p, tile, t)) break;
                const int nk = tile.K / PF_BK;
                for (int ks = 0; ks < nk && ok; ++ks) {
                    const uint32_t ss = it % C::STAGES, ph = (it / C::STAGES) & 1;
                    if (!(ok = mbar_wait(smem_u32(empty + ss), ph ^ 1, abort, p.status, p.dbg, 3, it))) break;
                    uint32_t dfill = 2;   // parity of this step's dense fill; 2: none
                    if (!tile.quant) {
                        uint8_t *st = a_base + ss * C::ASTAGE_BYTES;
                        mbar_expect_tx(smem_u32(full_at + ss), (uint32_t)(nmat * PF_A_BYTES));
                        tma_load_2d(smem_u32(st), &tm_a0, ks * PF_BK, tile.m0, smem_u32(full_at + ss));
                        if (g1) tma_load_2d(smem_u32(st + PF_A_BYTES), &tm_a1, ks * PF_BK, tile.m0, smem_u32(full_at + ss));
                        dfill = (dpar >> ss) & 1;
                        dpar ^= 1u << ss;
                        dany |= 1u << ss;
                    }
                    // relay: the stage is full once the activation tile (and a dense weight
                    // tile) has landed and the dequantising warps have arrived
                    if (!(ok = mbar_wait(smem_u32(full_b + ss), ph, abort, p.status, p.dbg, 4, it))) break;
                    if (dfill != 2 && !(ok = mbar_wait(smem_u32(full_at + ss), dfill, abort, p.status, p.dbg, 5, it))) break;
                    mbar_arrive(smem_u32(full + ss));
                    ++it;
                }
            }
            if (!ok)
                for (int ss = 0; ss < C::STAGES; ++ss)
                    if ((dany >> ss) & 1) mbar_drain(smem_u32(full_at + ss), ((dpar >> ss) & 1) ^ 1, p.status);
        }
    } else if (warp >= 4 && warp < 8) {
        // ----------------------------------------------------------------- epilogue
        const int q = warp - 4;
        uint32_t tc = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
            const PfTile tile = p.tiles[t];
            if (!pf_tile_ok(p, tile, t)) break;
            const uint32_t b = tc & 1;
            if (!mbar_wait(smem_u32(acc_full + b), (tc >> 1) & 1, abort, p.status, p.dbg, 21, tc, 256)) break;
            tc_fence_after();
            const int m = q * 32 + lane;
            const int N = (tile.n + 15) & ~15;
            const uint32_t row_addr = tmem + ((uint32_t)(q * 32) << 16) + b * 256;
            for (int c0 = 0; c0 < N; c0 += 16) {
                uint32_t ra[16];
                tc_ld16(row_addr + c0, ra);
                if (g1) {
                    uint32_t ru[16];
                    tc_ld16(row_addr + 128 + c0, ru);
                    tc_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int n = c0 + j;
                        const size_t oi = (size_t)(tile.b_row + n) * p.ld_out + tile.m0 + m;
                        if (n < tile.n) {
                            const float g = __uint_as_float(ra[j]), u = __uint_as_float(ru[j]);
                            const float hv = silu(g) * u;
                            // h is stored in fp16: a value beyond its range is reported, not
                            // silently turned into an infinity
                            if (!(fabsf(hv) <= 65504.0f)) pf_report(p, 5, t, (long long)oi, tile.m0 + m);
                            if (oi < p.out_elems) p.out16[oi] = __float2half_rn(hv);
                            else pf_report(p, 3, t, (long long)oi, tile.m0 + m);
                        }
                    }
                } else {
                    tc_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int n = c0 + j;
                        const size_t oi = (size_t)(tile.b_row + n) * p.ld_out + tile.m0 + m;
                        if (n < tile.n) {
                            if (oi < p.out_elems && tile.b_row + n < p.b_rows_total)
                                p.out32[oi] = __uint_as_float(ra[j]) * __ldg(p.row_scale + tile.b_row + n);
                            else
                                pf_report(p, 4, t, (long long)oi, tile.b_row + n);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(acc_empty + b));
            ++tc;
        }
    } else if (warp >= 8) {
        // ----------------------------------------------------------------- dequant
        // Thread td owns weight row `row` of every tile and the 32-wide half `hf` of every K
        // step, in each of the step's matrices; its offsets inside the raw tiles and the
        // swizzled operand rows are fixed.
        const int td = threadIdx.x - 256;
        const int row = td >> 1, hf = td & 1, rr = row & 31;
        const uint32_t q_off = (uint32_t)((row >> 5) * TILE_BYTES + TILE_QS + rr * 16);
        const uint32_t s_off = (uint32_t)((row >> 5) * TILE_BYTES + TILE_SC + rr * 16);
        const uint32_t d_off = (uint32_t)((row >> 5) * TILE_BYTES + TILE_DM + rr * 4);
        const uint32_t a_off = (uint32_t)((row >> 3) * 1024 + (row & 7) * 128);
        const uint32_t sw = row & 7, cb = 4 * hf;   // first 16-byte chunk of this half in the 64-wide row
        const uint32_t o0 = ((cb + 0) ^ sw) << 4, o1 = ((cb + 1) ^ sw) << 4, o2 = ((cb + 2) ^ sw) << 4,
                       o3 = ((cb + 3) ^ sw) << 4;
        float dq[nmat], nmq[nmat];   // d and -dmin of this row's current block, per matrix
#pragma unroll
        for (int m = 0; m < nmat; ++m) dq[m] = nmq[m] = 0.0f;
        const uint32_t a_s = smem_u32(a_base), raw_s = smem_u32(raw_base);
        uint32_t ait = 0, rit = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
            const PfTile tile = p.tiles[t];
            if (!pf_tile_ok(p, tile, t)) break;
            const int nk = tile.K / PF_BK;
            for (int ks = 0; ks < nk && ok; ++ks) {
                uint32_t r = 0;
                const int q4 = ks & 3, hh = q4 >> 1;
                uint4 c0[nmat], c1[nmat];
                uint32_t scw[nmat], dmw[nmat];
                auto read_raw = [&](int m) {
                    const uint32_t tl = raw_s + r * C::RAW_BYTES + m * 4 * TILE_BYTES;
                    c0[m] = lds_v4(tl + q_off + hh * 1024);
                    c1[m] = lds_v4(tl + q_off + hh * 1024 + 512);
                    scw[m] = lds_u32(tl + s_off + 4 * q4) >> (16 * hf);
                    dmw[m] = q4 == 0 ? lds_u32(tl + d_off) : 0u;
                };
                // With one matrix (GEMM2) the step's quants and scales are read before the
                // wait for the weight stage, so the reads overlap the wait; with two (GEMM1)
                // each matrix's reads just before its conversion measured faster.
                constexpr bool read_early = nmat == 1;
                if (tile.quant) {
                    r = rit % C::RAWS;
                    if ((ks & 3) == 0 && !(ok = mbar_wait(smem_u32(raw_full + r), (rit / C::RAWS) & 1, abort, p.status, p.dbg, 31, rit))) break;
                    if (read_early)
#pragma unroll
                        for (int m = 0; m < nmat; ++m) read_raw(m);
                }
                const uint32_t sa = ait % C::STAGES;
                if (!(ok = mbar_wait(smem_u32(empty + sa), ((ait / C::STAGES) & 1) ^ 1, abort, p.status, p.dbg, 32, ait))) break;
                if (tile.quant) {
                    const uint32_t st = a_s + sa * C::ASTAGE_BYTES;
                    const Plane pl = plane_of(2 * (q4 & 1) + hf);
#pragma unroll
                    for (int m = 0; m < nmat; ++m) {
                        if (!read_early) read_raw(m);
                        if (q4 == 0) {   // d, dmin hold for the whole 256-wide block
                            dq[m] = h2f(dmw[m]);
                            nmq[m] = -h2f(dmw[m] >> 16);
                        }
                        // scale bytes of the sub-blocks of this half: l < 16 and l >= 16
                        const uint32_t s0 = scw[m] & 0xFFu, s1 = (scw[m] >> 8) & 0xFFu;
                        const __half2 dsc0 = __float2half2_rn(dq[m] * (float)(s0 & 15u));
                        const __half2 ndm0 = __float2half2_rn(nmq[m] * (float)(s0 >> 4));
                        const __half2 dsc1 = __float2half2_rn(dq[m] * (float)(s1 & 15u));
                        const __half2 ndm1 = __float2half2_rn(nmq[m] * (float)(s1 >> 4));
                        const uint32_t arow = st + m * PF_A_BYTES + a_off;
                        sts_v4(arow + o0, dequant8(c0[m].x, c0[m].y, pl, dsc0, ndm0));
                        sts_v4(arow + o1, dequant8(c0[m].z, c0[m].w, pl, dsc0, ndm0));
                        sts_v4(arow + o2, dequant8(c1[m].x, c1[m].y, pl, dsc1, ndm1));
                        sts_v4(arow + o3, dequant8(c1[m].z, c1[m].w, pl, dsc1, ndm1));
                    }
                    fence_proxy_async();
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(full + sa));
                if (tile.quant && (ks & 3) == 3) {
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(raw_empty + r));
                    ++rit;
                }
                ++ait;
            }
        }
    }
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

// ------------------------------------------------------------------ router logits on tcgen05
// Prefill router: logits[t][e] = sum_i x[t,i] Wr[e,i] (+ bias_e) for a tile of 128 experts
// (MMA M, A = Wr, K-major) x 32 tokens (MMA N, B = x, K-major), both bf16 by TMA with the
// 128-byte swizzle.  Each 64-wide K chunk is one group of four kind::f16 MMAs accumulating
// in fp32 into one of two TMEM buffers (32 columns each); the epilogue warps (one TMEM lane
// = one expert each) read every chunk's sums and add them in fp64, so only the tensor
// core's own sum of 64 exact products (each bf16 x bf16 product is exact in fp32) carries
// an fp32 error.  That error is bounded, per chunk, by 64 units of 2^-23 of the chunk's
// sum of |products| -- as if every product were added with its own truncation, the
// tensor core's worst case -- so |fast - exact| <= BOUND_MMA * sum_i |x_i Wr_i| (plus the
// fp64 additions), and sum_i |x_i Wr_i| <= ||x_t|| ||Wr_e|| (Cauchy-Schwarz).  Warps 2-3
// sum the squares of the tile's tokens in fp64 meanwhile.
//   warp 0  producer: TMA of the Wr and x tiles of every K chunk (RM_STAGES-deep ring)
//   warp 1  MMA: allocates TMEM, four MMAs per chunk into buffer (chunk & 1)
//   warps 2-3  token norms;  warps 4-7  epilogue.
constexpr int RM_M = 128, RM_N = 32, RM_BK = 64, RM_STAGES = 4;
constexpr int RM_THREADS = 256;
constexpr int RM_A_BYTES = RM_M * RM_BK * 2;   // 16 KiB
constexpr int RM_B_BYTES = RM_N * RM_BK * 2;   // 4 KiB
constexpr size_t RM_SMEM = 1024 + RM_STAGES * (RM_A_BYTES + RM_B_BYTES) + 512;
constexpr float BOUND_MMA = 7.7e-6f;           // 64 * 2^-23 = 7.63e-6, rounded up

// Instruction descriptor of kind::f16 with bf16 A and B (K-major), fp32 D, M = 128, N.
__device__ __forceinline__ uint32_t bf16_idesc(int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(RM_M >> 4) << 24);
}
__device__ __forceinline__ void tc_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

struct RouterArgs {
    const __nv_bfloat16 *x;   // [T][H] (token norms)
    int T, H, E;
    const float *bias;        // [E] or null
    const float *wr_norm;     // [E], rounded up
    double *logits;           // [T][E]
    float *labs;              // [T][E]: a bound of sum_i |x_i Wr_i|
    int *status;
    int *dbg;
};

__global__ void __launch_bounds__(RM_THREADS, 1)
    router_mma_kernel(const __grid_constant__ CUtensorMap tm_wr, const __grid_constant__ CUtensorMap tm_xr, RouterArgs p) {
    extern __shared__ __align__(1024) uint8_t rm_smem_raw[];
    uint8_t *base = rm_smem_raw + ((1024u - (smem_u32(rm_smem_raw) & 1023u)) & 1023u);
    uint8_t *a_base = base;
    uint8_t *b_base = a_base + RM_STAGES * RM_A_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(b_base + RM_STAGES * RM_B_BYTES);
    uint64_t *full = bars;                   // [S] expect_tx + TMA bytes
    uint64_t *empty = full + RM_STAGES;      // [S] MMA commit
    uint64_t *acc_full = empty + RM_STAGES;  // [2] MMA commit
    uint64_t *acc_empty = acc_full + 2;      // [2] 4 epilogue warps
    uint64_t *drain = acc_empty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort = reinterpret_cast<volatile int *>(drain + 2);
    double *xn2 = reinterpret_cast<double *>(drain + 4);   // [RM_N] token sums of squares

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.y * RM_M, n0 = blockIdx.x * RM_N;
    const int nk = p.H / RM_BK;
    if (threadIdx.x == 0) {
        for (int s = 0; s < RM_STAGES; ++s) {
            mbar_init(smem_u32(full + s), 1);
            mbar_init(smem_u32(empty + s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(acc_full + b), 1);
            mbar_init(smem_u32(acc_empty + b), 4);
        }
        mbar_init(smem_u32(drain), 1);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 64;" ::"r"(smem_u32(tmem_holder))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        uint32_t c = 0;
        bool ok = true;
        for (; c < (uint32_t)nk; ++c) {
            const uint32_t s = c % RM_STAGES;
            if (!(ok = mbar_wait(smem_u32(empty + s), ((c / RM_STAGES) & 1) ^ 1, abort, p.status, p.dbg, 41, c, 64))) break;
            if (elect_one()) {
                mbar_expect_tx(smem_u32(full + s), (uint32_t)(RM_A_BYTES + RM_B_BYTES));
                tma_load_2d(smem_u32(a_base + s * RM_A_BYTES), &tm_wr, (int)c * RM_BK, m0, smem_u32(full + s));
                tma_load_2d(smem_u32(b_base + s * RM_B_BYTES), &tm_xr, (int)c * RM_BK, n0, smem_u32(full + s));
            }
            __syncwarp();
        }
        if (!ok)
            for (uint32_t i = c > RM_STAGES ? c - RM_STAGES : 0; i < c; ++i)
                mbar_drain(smem_u32(full + i % RM_STAGES), (i / RM_STAGES) & 1, p.status);
    } else if (warp == 1) {
        const uint32_t idesc = bf16_idesc(RM_N);
        bool ok = true;
        for (uint32_t c = 0; c < (uint32_t)nk && ok; ++c) {
            const uint32_t s = c % RM_STAGES, b = c & 1;
            if (!(ok = mbar_wait(smem_u32(acc_empty + b), ((c >> 1) & 1) ^ 1, abort, p.status, p.dbg, 42, c, 32))) break;
            if (!(ok = mbar_wait(smem_u32(full + s), (c / RM_STAGES) & 1, abort, p.status, p.dbg, 43, c))) break;
            tc_fence_after();
            const uint32_t ast = smem_u32(a_base + s * RM_A_BYTES), bst = smem_u32(b_base + s * RM_B_BYTES);
            if (elect_one()) {
#pragma unroll
                for (int kk = 0; kk < RM_BK / 16; ++kk)
                    tc_mma(tmem + b * RM_N, sw128_desc(ast + kk * 32), sw128_desc(bst + kk * 32), idesc, kk != 0);
                tc_commit(smem_u32(empty + s));
                tc_commit(smem_u32(acc_full + b));
            }
            __syncwarp();
        }
        if (elect_one()) tc_commit(smem_u32(drain));
        __syncwarp();
        mbar_drain(smem_u32(drain), 0, p.status);
    } else if (warp == 2 || warp == 3) {
        // token norms: warp 2 the first 16 tokens of the tile, warp 3 the next 16
        for (int i = 0; i < RM_N / 2; ++i) {
            const int tl = (warp - 2) * (RM_N / 2) + i, t = n0 + tl;
            double ss = 0.0;
            if (t < p.T)
                for (int k = lane * 8; k < p.H; k += 256) {
                    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p.x + (size_t)t * p.H + k));
                    const uint32_t vs[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const double lo = bf16lo(vs[q]), hi = bf16hi(vs[q]);
                        ss = fma(lo, lo, ss);
                        ss = fma(hi, hi, ss);
                    }
                }
            ss = warp_sum(ss);
            if (lane == 0) xn2[tl] = ss;
        }
    } else if (warp >= 4) {
        const int q = warp - 4;
        double acc[RM_N];
#pragma unroll
        for (int j = 0; j < RM_N; ++j) acc[j] = 0.0;
        bool ok = true;
        for (uint32_t c = 0; c < (uint32_t)nk; ++c) {
            const uint32_t b = c & 1;
            if (!(ok = mbar_wait(smem_u32(acc_full + b), (c >> 1) & 1, abort, p.status, p.dbg, 44, c))) break;
            tc_fence_after();
            float v[32];
            tc_ld32(tmem + ((uint32_t)(q * 32) << 16) + b * RM_N, v);
            tc_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(acc_empty + b));
#pragma unroll
            for (int j = 0; j < RM_N; ++j) acc[j] += (double)v[j];
        }
        // the norms of warps 2-3 are complete once every CTA thread passes this barrier
        asm volatile("bar.sync 1, 192;" ::: "memory");
        const int e = m0 + q * 32 + lane;
        if (ok && e < p.E) {
            const float wn = p.wr_norm[e];
            const double be = p.bias ? (double)p.bias[e] : 0.0;
#pragma unroll
            for (int j = 0; j < RM_N; ++j) {
                const int t = n0 + j;
                if (t < p.T) {
                    p.logits[(size_t)t * p.E + e] = p.bias ? __dadd_rn(acc[j], be) : acc[j];
                    p.labs[(size_t)t * p.E + e] = (float)sqrt(xn2[j]) * (1.0f + 1e-6f) * wn;
                }
            }
        }
    }
    if (warp == 2 || warp == 3) asm volatile("bar.sync 1, 192;" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 64;" ::"r"(tmem) : "memory");
    }
}

// ------------------------------------------------------------------ helpers around it
// Tile list of one GEMM: every active expert's pair rows in tiles of N tokens x 128 weight
// rows, then the shared expert's token rows (when Is > 0).  One CTA.
__global__ void pf_build_tiles_kernel(const int *offsets, const int *active, const int *n_active, int T, int P,
                                      int n_tile, int m_rows_routed, int k_routed, int m_rows_shared, int k_shared,
                                      PfTile *tiles, int *n_tiles, int max_tiles) {
    __shared__ int start[MAX_EXPERTS + 2];
    const int n_act = *n_active;
    const int mt_r = m_rows_routed / PF_M, mt_s = m_rows_shared / PF_M;
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int a = 0; a < n_act; ++a) {
            start[a] = acc;
            const int e = active[a];
            const int cnt = offsets[e + 1] - offsets[e];
            acc += (cnt + n_tile - 1) / n_tile * mt_r;
        }
        start[n_act] = acc;
        if (mt_s > 0) acc += (T + n_tile - 1) / n_tile * mt_s;
        start[n_act + 1] = acc;
        *n_tiles = acc < max_tiles ? acc : max_tiles;
    }
    __syncthreads();
    for (int a = 0; a <= n_act; ++a) {
        const bool shared = a == n_act;
        if (shared && mt_s == 0) break;
        const int e = shared ? -1 : active[a];
        const int row0 = shared ? P : offsets[e];
        const int cnt = shared ? T : offsets[e + 1] - offsets[e];
        const int mt = shared ? mt_s : mt_r;
        const int n_tiles_e = (cnt + n_tile - 1) / n_tile * mt;
        for (int i = threadIdx.x; i < n_tiles_e; i += blockDim.x) {
            const int idx = start[a] + i;
            if (idx >= max_tiles) break;
            const int nt = i / mt, m = i % mt;
            PfTile tl;
            tl.expert = e;
            tl.m0 = m * PF_M;
            tl.b_row = row0 + nt * n_tile;
            tl.n = min(n_tile, cnt - nt * n_tile);
            tl.quant = shared ? 0 : 1;
            tl.K = shared ? k_shared : k_routed;
            tl.pad0 = tl.pad1 = 0;
            tiles[idx] = tl;
        }
    }
}

// Rows of X (fp16) in pair order, then the tokens in order for the shared expert; the
// routing weight of each row (1 for the shared rows).  One CTA per row.  An activation
// beyond the fp16 range (|x| > 65504, or not finite) sets the EDEVICE status: the grouped
// path computes in fp16 and does not silently turn it into an infinity.
__global__ void pf_gather_kernel(const __nv_bfloat16 *__restrict__ x, int T, int H, int k, const int *sorted_token,
                                 const int *sorted_slot, const float *topk_w, int P, __half *xall, float *row_w,
                                 int *status) {
    const int r = blockIdx.x;
    int tok;
    float w = 1.0f;
    if (r < P) {
        tok = sorted_token[r];
        w = topk_w[(size_t)tok * k + sorted_slot[r]];
    } else {
        tok = r - P;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(x + (size_t)tok * H);
    uint2 *dst = reinterpret_cast<uint2 *>(xall + (size_t)r * H);
    float amax = 0.0f;
    for (int i = threadIdx.x; i < H / 8; i += blockDim.x) {
        const uint4 v = __ldg(src + i);
        const uint32_t vs[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float lo = bf16lo(vs[q]), hi = bf16hi(vs[q]);
            amax = fmaxf(amax, fmaxf(fabsf(lo), fabsf(hi)));
            if (lo != lo || hi != hi) amax = INFINITY;
            const __half2 h = __floats2half2_rn(lo, hi);
            o[q] = *reinterpret_cast<const uint32_t *>(&h);
        }
        dst[2 * i] = make_uint2(o[0], o[1]);
        dst[2 * i + 1] = make_uint2(o[2], o[3]);
    }
    if (amax > 65504.0f) set_status(status, ST_EDEVICE);
    if (threadIdx.x == 0) row_w[r] = w;
}

// y[t] = sum_j O[inv_pos[t, j]] + O[P + t] (the shared row, when present), 4 columns a thread.
__global__ void pf_combine_kernel(const float *__restrict__ oall, int T, int H, int k, const int *inv_pos, int P,
                                  int has_shared, float *__restrict__ y) {
    const int t = blockIdx.x;
    for (int c = threadIdx.x * 4; c < H; c += blockDim.x * 4) {
        float4 acc = has_shared ? *reinterpret_cast<const float4 *>(oall + (size_t)(P + t) * H + c)
                                : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < k; ++j) {
            const int p = inv_pos[(size_t)t * k + j];
            const float4 v = *reinterpret_cast<const float4 *>(oall + (size_t)p * H + c);
            acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
        }
        *reinterpret_cast<float4 *>(y + (size_t)t * H + c) = acc;
    }
}

// bf16 -> fp16 (shared-expert weights, once at load).
__global__ void bf16_to_f16_kernel(const __nv_bfloat16 *__restrict__ src, __half *__restrict__ dst, size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        dst[i] = __float2half_rn(__bfloat162float(src[i]));
}

struct PrefillWork {
    __half *xall = nullptr;   // [Pm + Tm][H]
    __half *hall = nullptr;   // [Pm + Tm][ldH]
    float *oall = nullptr;    // [Pm + Tm][H]
    float *row_w = nullptr;   // [Pm + Tm]
    PfTile *tiles1 = nullptr, *tiles2 = nullptr;
    int *n_tiles = nullptr;   // [2]
    int max_tiles1 = 0, max_tiles2 = 0;
    int ldH = 0;
};

template <class Carver>
void prefill_layout(PrefillWork &w, Carver &c, int Tm, int k, int E, int H, int I, int Is) {
    const size_t rows = (size_t)Tm * k + Tm;
    w.ldH = I > Is ? I : Is;
    w.xall = c.template take<__half>(rows * H);
    w.hall = c.template take<__half>(rows * w.ldH);
    w.oall = c.template take<float>(rows * H);
    w.row_w = c.template take<float>(rows);
    const int n_groups1 = (int)((size_t)Tm * k / PF_N1) + E + Tm / PF_N1 + 2;
    const int n_groups2 = (int)((size_t)Tm * k / PF_N2) + E + Tm / PF_N2 + 2;
    const int mt1 = (I > Is ? I : Is) / PF_M, mt2 = H / PF_M;
    w.max_tiles1 = n_groups1 * mt1;
    w.max_tiles2 = n_groups2 * mt2;
    w.tiles1 = c.template take<PfTile>(w.max_tiles1);
    w.tiles2 = c.template take<PfTile>(w.max_tiles2);
    w.n_tiles = c.template take<int>(2);
}
inline void prefill_init(PrefillWork &) {}

}  // namespace ds4
