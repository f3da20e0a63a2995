// Start states of the consecutive segments of a sequence from the segments'
// affine maps.  The state carried across a chunk boundary is affine in the
// state it starts from ("From GPT-2 to Kimi K3" essay, pwwt.cn/news/3716252,
// chunkwise paragraph: a fixed-size state carried from chunk to chunk), so a
// segment of tokens maps its start state S to M S + F, with M (d_k x d_k) and
// F (d_k x d_v) from kda_chunk_segment_map.  Chaining them gives every
// segment's start state:
//     S_0 = init (or 0),   S_{r+1} = M_r S_r + F_r.
#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kCols = 32;   // state columns per block

// grid (N H, dv / 32), block dk threads: thread c forms row c of each S_{r+1}
// (fp32), with the current column tile of S_r in shared memory.
__global__ void __launch_bounds__(128) compose_states(const float* __restrict__ M, const float* __restrict__ F,
                                                      const float* __restrict__ init, int R, int NH, int dk, int dv,
                                                      float* __restrict__ out) {
    __shared__ float St[128][kCols + 1];
    const int nh = blockIdx.x, j0 = blockIdx.y * kCols, c = threadIdx.x;
    const size_t srow = ((size_t)nh * dk + c) * dv + j0;     // row c of a state, this tile
    float s[kCols];
#pragma unroll
    for (int j = 0; j < kCols; ++j) s[j] = init ? init[srow + j] : 0.f;
#pragma unroll
    for (int j = 0; j < kCols; ++j) out[srow + j] = s[j];
    for (int r = 0; r < R; ++r) {
#pragma unroll
        for (int j = 0; j < kCols; ++j) St[c][j] = s[j];
        __syncthreads();
        const size_t fo = (size_t)r * NH * dk * dv + srow;
        const float* mrow = M + ((size_t)r * NH * dk + (size_t)nh * dk + c) * dk;
#pragma unroll
        for (int j = 0; j < kCols; ++j) s[j] = F[fo + j];
        for (int kk = 0; kk < dk; kk += 4) {
            const float4 m = *reinterpret_cast<const float4*>(mrow + kk);
#pragma unroll
            for (int j = 0; j < kCols; ++j) {
                s[j] = fmaf(m.x, St[kk][j], s[j]);
                s[j] = fmaf(m.y, St[kk + 1][j], s[j]);
                s[j] = fmaf(m.z, St[kk + 2][j], s[j]);
                s[j] = fmaf(m.w, St[kk + 3][j], s[j]);
            }
        }
        __syncthreads();
        const size_t oo = (size_t)(r + 1) * NH * dk * dv + srow;
#pragma unroll
        for (int j = 0; j < kCols; ++j) out[oo + j] = s[j];
    }
}

}  // namespace

cudaError_t launch_compose_states(const float* M, const float* F, const float* init, int R, int N, int H, int dk,
                                  int dv, float* out, cudaStream_t stream) {
    const int NH = N * H;
    if (NH == 0) return cudaSuccess;
    compose_states<<<dim3(NH, dv / kCols), dk, 0, stream>>>(M, F, init, R, NH, dk, dv, out);
    return cudaGetLastError();
}

}  // namespace kda
