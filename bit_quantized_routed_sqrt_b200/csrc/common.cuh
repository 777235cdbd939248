// common.cuh -- shared device helpers of the ds4moe library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace ds4 {

// Device status words (mirror the public ds4moe_status values).
enum : int { ST_OK = 0, ST_ETIMEOUT = 5, ST_EDEVICE = 6 };

// Q2_K super-block: 256 weights in 84 bytes (16 scale bytes, 64 quant bytes, fp16 d, fp16 dmin).
constexpr int QK = 256;
constexpr int BLOCK_BYTES = 84;

// Device tile layout of a Q2_K matrix [R rows x K inputs]: 32 consecutive rows x one
// 256-input block form one 2688-byte tile, tiles ordered (row group, block):
//   bytes [0, 2048):    quant chunk c (0..3) of row r at c*512 + r*16 (16 quant bytes each:
//                       chunk c holds quant bytes 16c .. 16c+15 of the row's block)
//   bytes [2048, 2560): 16 scale bytes of row r at 2048 + r*16
//   bytes [2560, 2688): d | dmin << 16 (fp16 pair) of row r at 2560 + r*4
// A warp whose lane r reads row r touches 512 contiguous bytes per quant chunk.
constexpr int TILE_ROWS = 32;
constexpr int TILE_BYTES = TILE_ROWS * BLOCK_BYTES;   // 2688
constexpr int TILE_QS = 0;
constexpr int TILE_SC = 2048;
constexpr int TILE_DM = 2560;

__host__ __device__ constexpr size_t tiled_bytes(int rows, int K) { return (size_t)rows / TILE_ROWS * (K / QK) * TILE_BYTES; }

__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float h2f(uint32_t bits16) {
    return __half2float(__ushort_as_half((unsigned short)(bits16 & 0xFFFF)));
}

// Streaming 16-byte load that bypasses L1 allocation (weights are read once per call).
__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ uint32_t ld_stream_u32(const void *p) {
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

// Asynchronous prefetch of [p, p + bytes) into L2 (p 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Prefetch a byte range into L2 in 32 KiB pieces, piece i issued by worker i of n.
__device__ __forceinline__ void prefetch_range_l2(const void *base, size_t bytes, int worker, int n_workers) {
    const size_t piece = 32768;
    const size_t n = (bytes + piece - 1) / piece;
    for (size_t i = worker; i < n; i += n_workers) {
        const size_t off = i * piece;
        const size_t len = bytes - off < piece ? bytes - off : piece;
        prefetch_l2(reinterpret_cast<const char *>(base) + off, (uint32_t)(len & ~(size_t)15));
    }
}

// Two-way dot of a pair of signed 16-bit values with two unsigned bytes (bytes 0,1 or 2,3 of b).
__device__ __forceinline__ int dp2a_lo(int a, uint32_t b, int c) {
    int d;
    asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp2a_hi(int a, uint32_t b, int c) {
    int d;
    asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + expf(-g)); }

// Router score sqrt(softplus(l)) in fp32, accurate for very negative logits: with
// t = exp(-|l|), softplus(l) = max(l, 0) + log1p(t), and for t < 1/32 log1p(t) is taken
// from the 4-term series t - t^2/2 + t^3/3 - t^4/4 on t clamped to [0, 1/32]
// (truncation error below t^5/5, i.e. relative 1.9e-7), which avoids the cancellation
// of log(1 + exp(l)) in fp32.  Source: opensource-hub.com "antirez/ds4" FAQ,
// router-precision entry.
__device__ __forceinline__ float softplus_accurate(float l) {
    float t = expf(-fabsf(l));
    float lp;
    if (t < 0.03125f) {
        float c = fminf(fmaxf(t, 0.0f), 0.03125f);
        lp = c * (1.0f + c * (-0.5f + c * (0.333333343f + c * -0.25f)));
    } else {
        lp = log1pf(t);
    }
    return fmaxf(l, 0.0f) + lp;
}
__device__ __forceinline__ float router_score(float l) { return sqrtf(softplus_accurate(l)); }

// The naive fp32 form log(1 + exp(l)) (diagnostic only; never used by the router).
__device__ __forceinline__ float router_score_naive(float l) { return sqrtf(logf(1.0f + expf(l))); }

__device__ __forceinline__ void set_status(int *st, int code) {
    if (st) atomicCAS(st, ST_OK, code);
}

}  // namespace ds4
