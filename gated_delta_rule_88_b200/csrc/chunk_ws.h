// chunk_ws.h -- layout of the per-(chunk, head) scratch records that the
// bf16 chunk-prep kernel writes and the chain kernel reads (dk = dv = 128,
// chunk C = 64).  One record per (chunk, head), chunk-major:
//     record index = global_chunk * H + head
// where global_chunk enumerates the chunks of sequence 0, then sequence 1,
// ...  All matrices are row-major bf16 with 128-element (256-byte) rows.
#pragma once

#include <stddef.h>

namespace kda {
namespace ws {

constexpr int C = 64;          // chunk length
constexpr int D = 128;         // dk = dv
constexpr size_t OFF_W = 0;          // W   = T (beta K e^G)          [64][128]
constexpr size_t OFF_QG = 16384;     // Qg  = Q e^G                   [64][128]
constexpr size_t OFF_KT = 32768;     // Kt  = K e^{G_C - G}           [64][128]
constexpr size_t OFF_U = 49152;      // U   = T (beta V)              [64][128]
constexpr size_t OFF_P = 65536;      // P   = tril(Q K^T with decay)  [64][64]
constexpr size_t OFF_EGC = 73728;    // e^{G_C}                       [128] fp32
constexpr size_t RECORD = 74240;     // bytes per record (multiple of 256)

}  // namespace ws
}  // namespace kda
