// Layout of the tensor-core prefill's per-(chunk, head) workspace image, shared
// by the kernels that write it (tc_intra), read it (tc_recur) and reuse it in the
// backward pass (kb_chain_tc).  The scratch starts with an error word.
#pragma once

#include <stdint.h>

namespace kda {
namespace tcimg {

constexpr uint32_t kOffWkQh = 0;         // [128 rows][128 k] bf16 SW128 K-major: rows 0-63 Wk, 64-127 Q exp(g) (hi)
constexpr uint32_t kOffWkQl = 32768;     // lo parts
constexpr uint32_t kOffKdTh = 65536;     // [128 rows (channel)][64 k (token)] bf16 SW128 K-major (hi)
constexpr uint32_t kOffKdTl = 81920;     // lo parts
constexpr uint32_t kOffU = 98304;        // U : fp32, see u_index()
constexpr uint32_t kOffPh = 131072;      // P [64 rows][64 k] bf16 SW128 K-major (hi)
constexpr uint32_t kOffPl = 139264;      // lo parts
constexpr uint32_t kOffGam = 147456;     // Gamma_C fp32 [128]
constexpr uint32_t kChunkBytes = 147968;
constexpr uint32_t kErrHeader = 256;     // first bytes of the TC scratch: error word

// U tiles: [4 column blocks of 32][64 rows][8 chunks of 4 floats], chunk
// permuted by row % 8 so that row-per-thread float4 reads hit distinct banks.
__host__ __device__ __forceinline__ int u_index(int r, int j) {   // j % 4 == 0
    return (j >> 5) * 2048 + r * 32 + (((((j & 31) >> 2)) ^ (r & 7)) << 2);
}

}  // namespace tcimg
}  // namespace kda
