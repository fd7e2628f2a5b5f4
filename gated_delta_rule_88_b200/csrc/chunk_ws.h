// chunk_ws.h -- layout of the per-(chunk, head) records that the bf16
// chunk-prep kernel writes and the chain kernel reads (dk = dv = 128, chunk
// C = 64).  One record per (chunk, head), chunk-major:
//     record index = global_chunk * H + head
// where global_chunk enumerates the chunks of sequence 0, then sequence 1, ...
//
// The matrix regions are stored as shared-memory images, so the consumer
// copies them verbatim into 1024-byte-aligned shared memory and hands them to
// the tensor cores: "K-major, 128-byte swizzle" means rows of 64 bf16
// (128 bytes), and within each 8-row group the 16-byte chunk j of row r sits
// at chunk position j ^ (r % 8).  A matrix with K = 128 is two such blocks of
// 64 columns, one after the other.
#pragma once

#include <stddef.h>

namespace kda {
namespace ws {

constexpr int C = 64;          // chunk length
constexpr int D = 128;         // dk = dv

// [W; Qg]: 128 rows (rows 0-63: W = T (beta K e^G), rows 64-127: Qg = Q e^G)
// x 128 channels, K-major SW128, two 64-channel blocks of 128 rows x 128 B.
constexpr size_t OFF_AW = 0;
// Kt^T: 128 channel rows x 64 tokens, Kt = K e^{G_C - G}; K-major SW128.
constexpr size_t OFF_KTT = 32768;
// P: 64 x 64, P_ij = sum_c q_ic k_jc e^{G_ic - G_jc} (j <= i, else 0);
// K-major SW128.
constexpr size_t OFF_P = 49152;
// U = T (beta V): 64 tokens x 128, as four plain row-major tiles of 32
// columns ([tile][64][32] bf16, 4 KiB per tile).
constexpr size_t OFF_U = 57344;
constexpr size_t U_TILE = 4096;
// e^{G_C}: 128 fp32.
constexpr size_t OFF_EGC = 73728;
constexpr size_t RECORD = 74240;     // bytes per record

// byte offset of element (r, c), c in 0..63, in a K-major SW128 image with
// 128-byte rows
__host__ __device__ constexpr size_t sw128(int r, int c) {
    return (size_t)r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1);
}
// [W; Qg] element (r in 0..127, channel c in 0..127)
__host__ __device__ constexpr size_t aw_off(int r, int c) {
    return OFF_AW + (size_t)(c >> 6) * 16384 + sw128(r, c & 63);
}

}  // namespace ws
}  // namespace kda
