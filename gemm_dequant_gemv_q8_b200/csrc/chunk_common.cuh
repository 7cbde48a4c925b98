// chunk_common.cuh -- operand layouts of the NVFP4 prefill-chunk GEMM (tcgen05 block-scaled MMA).
//
// Both operands are stored in global memory exactly as the tensor core reads them from shared
// memory, so each pipeline stage is filled by plain bulk copies:
//   codes : rows of 128 bytes (256 E2M1 values of one k-group), 16-byte chunk c of row r stored at
//           chunk position c ^ (r % 8) -- the 128-byte-swizzled K-major canonical layout; 8-row
//           groups are 1024 bytes apart.
//   scales: per 64-value k-block and per 128 rows, a 512-byte atom; the E4M3 scale of row r
//           (0..127) and 16-value block j (0..3) is at byte (r % 32) * 16 + (r / 32) * 4 + j, the
//           layout the 32x128b scale-factor copy into tensor memory expects.
// Weights (QLIN_PACK_MMA): units of 256 rows x 256 values = 32768 B codes + 8 atoms (4 k-blocks x
// 2 row halves) = 36864 B, in [row tile][k-group] order after the 256-byte header.
// Activations (quantized by the chunk path): units of 128 rows x 256 values = 16384 B codes +
// 4 atoms = 18432 B, in [row tile][k-group] order.
#pragma once
#include "qlin_common.cuh"

namespace qlin {

constexpr int kMmaWRows = 256;   // weight rows per tile (the MMA N dimension)
constexpr int kMmaARows = 128;   // activation rows per tile (the MMA M dimension)
constexpr int kMmaWUnit = 256 * 128 + 8 * 512;  // 36864
constexpr int kMmaAUnit = 128 * 128 + 4 * 512;  // 18432

__host__ __device__ inline int64_t mma_code_off(int r, int chunk) {
    return (int64_t)r * 128 + ((chunk ^ (r & 7)) << 4);
}
// scale atom byte offset inside a unit's scale region: kb = 64-value block, r = row in the tile
__host__ __device__ inline int64_t mma_scale_off(int kb, int r, int j, int halves) {
    const int h = r >> 7, rr = r & 127;
    return (int64_t)(kb * halves + h) * 512 + (rr & 31) * 16 + (rr >> 5) * 4 + j;
}

}  // namespace qlin
