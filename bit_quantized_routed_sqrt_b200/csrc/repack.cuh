// repack.cuh -- Q2_K AoS super-blocks <-> the device tile layout (see common.cuh).
#pragma once
#include "common.cuh"

namespace ds4 {

// One thread per (matrix, row, block).  Threads are numbered with the row-in-group
// fastest so that the 16-byte stores of a warp are contiguous.
//   aos:   [n_mats][rows][nb][84] bytes (4-byte aligned base)
//   tiled: [n_mats][rows/32][nb][2688]
__global__ void repack_q2k_kernel(const uint8_t *__restrict__ aos, uint8_t *__restrict__ tiled, int n_mats,
                                  int rows, int nb) {
    const long long per_mat = (long long)rows * nb;
    const long long total = per_mat * n_mats;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long m = i / per_mat;
        long long rem = i - m * per_mat;
        const int rr = (int)(rem % TILE_ROWS);
        rem /= TILE_ROWS;
        const int b = (int)(rem % nb);
        const int rg = (int)(rem / nb);
        const int r = rg * TILE_ROWS + rr;
        const uint32_t *src = reinterpret_cast<const uint32_t *>(aos + ((m * rows + r) * nb + b) * BLOCK_BYTES);
        uint32_t v[21];
#pragma unroll
        for (int w = 0; w < 21; ++w) v[w] = __ldg(src + w);
        uint8_t *tile = tiled + (m * per_mat / TILE_ROWS + (long long)rg * nb + b) * TILE_BYTES;
#pragma unroll
        for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4 *>(tile + TILE_QS + c * 512 + rr * 16) =
                make_uint4(v[4 + 4 * c], v[5 + 4 * c], v[6 + 4 * c], v[7 + 4 * c]);
        *reinterpret_cast<uint4 *>(tile + TILE_SC + rr * 16) = make_uint4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<uint32_t *>(tile + TILE_DM + rr * 4) = v[20];
    }
}

// Inverse of repack_q2k_kernel for one matrix (round-trip checks).
__global__ void export_q2k_kernel(const uint8_t *__restrict__ tiled, uint8_t *__restrict__ aos, int rows, int nb) {
    const long long total = (long long)rows * nb;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int r = (int)(i / nb), b = (int)(i % nb);
        const int rg = r / TILE_ROWS, rr = r % TILE_ROWS;
        const uint8_t *tile = tiled + ((long long)rg * nb + b) * TILE_BYTES;
        uint32_t v[21];
        const uint4 sc = *reinterpret_cast<const uint4 *>(tile + TILE_SC + rr * 16);
        v[0] = sc.x; v[1] = sc.y; v[2] = sc.z; v[3] = sc.w;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint4 q = *reinterpret_cast<const uint4 *>(tile + TILE_QS + c * 512 + rr * 16);
            v[4 + 4 * c] = q.x; v[5 + 4 * c] = q.y; v[6 + 4 * c] = q.z; v[7 + 4 * c] = q.w;
        }
        v[20] = *reinterpret_cast<const uint32_t *>(tile + TILE_DM + rr * 4);
        uint32_t *dst = reinterpret_cast<uint32_t *>(aos + i * BLOCK_BYTES);
#pragma unroll
        for (int w = 0; w < 21; ++w) dst[w] = v[w];
    }
}

}  // namespace ds4
