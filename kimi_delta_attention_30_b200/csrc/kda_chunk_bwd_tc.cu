// Tensor-core (tcgen05) chunk-local products of the KDA backward pass, for
// bf16 inputs with d_k = d_v = 128 and 64-token chunks.
//
// Per (chunk, head), with the chunk's start state S and the gradient dS' of its
// end state (both 128 x 128 fp32), W and dW (64 x 128 fp32, per-token
// corrections and their gradient) and dO (64 x 128 bf16):
//     dQg = dO S^T,   dWk = -dW S^T,   dKd = W dS'^T,   dP = dO W^T (i <= r),
//     dGam_c = sum_j dS'_cj S_cj.
// These are the chain rule through O = Qg S + P W and S' = Diag(Gam) S + Kd^T W
// (the chunk form the forward computes; derivation as in the CUDA-core kernels:
// "From GPT-2 to Kimi K3" essay, pwwt.cn/news/3716252, chunkwise paragraph, for
// the form; the pages give no backward pass).
//
// One CTA of 256 threads per (chunk, head).  Operands are staged in shared
// memory as bf16 images, K-major with the 128-byte swizzle, each fp32 value as
// hi = RN(x) and lo = RN(x - hi) and every product formed as hi*hi + hi*lo +
// lo*hi (dO is a bf16 input, exact in hi alone, so its products take two terms):
//     D1 = [dO ; dW] S^T   (M = 128, N = 128)  -> dQg (rows 0-63), -dWk (rows 64-127)
//     D2 = W dS'^T         (M =  64, N = 128)  -> dKd
//     D3 = dO W^T          (M =  64, N =  64)  -> dP
// with fp32 accumulators in tensor memory, read back by the threads that store
// the results.  dGam is summed while S and dS' pass through registers.
#include "kda_internal.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int kAThreads = 256;
constexpr int kD = 128;
constexpr int kC = 64;

// shared-memory images (byte offsets from the 1024-aligned dynamic base)
constexpr uint32_t kA1h = 0;          // [dO ; dW] hi, 128 rows x 128 k
constexpr uint32_t kA1l = 32768;      // lo (rows 0-63, dO, are zero)
constexpr uint32_t kA2h = 65536;      // W hi, 64 rows x 128 k (A of D2 and B of D3)
constexpr uint32_t kA2l = 81920;
constexpr uint32_t kB1h = 98304;      // S hi, 128 rows (channel) x 128 k (state column)
constexpr uint32_t kB1l = 131072;
constexpr uint32_t kB2h = 163840;     // dS' hi
constexpr uint32_t kB2l = 196608;
constexpr uint32_t kBarOff = 229376;  // mbarrier, tensor-memory base
constexpr uint32_t kASmem = kBarOff + 16;
constexpr uint32_t kATmemCols = 512;  // D1 0-127, D2 128-255, D3 256-319

__device__ __forceinline__ size_t toff(int t, int H, int h) { return ((size_t)t * H + h) * kD; }

// four fp32 values -> hi and lo bf16 quadruples, stored at byte offset `off` of each image
__device__ __forceinline__ void store4_split(uint8_t* hi, uint8_t* lo, uint32_t off, float4 x) {
    uint32_t h0, l0, h1, l1;
    split2(x.x, x.y, h0, l0);
    split2(x.z, x.w, h1, l1);
    *reinterpret_cast<uint2*>(hi + off) = make_uint2(h0, h1);
    *reinterpret_cast<uint2*>(lo + off) = make_uint2(l0, l1);
}

__global__ void __launch_bounds__(kAThreads, 1)
kb_a_tc(const __nv_bfloat16* __restrict__ d_o, const float* __restrict__ W, const float* __restrict__ dW,
        const float* __restrict__ S_chunk, const float* __restrict__ dS_chunk, float* __restrict__ dQg,
        float* __restrict__ dKd, float* __restrict__ dWk, float* __restrict__ dGam, float* __restrict__ dP,
        int* __restrict__ err, ChunkMap cmap, int H) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // no static shared memory: the dynamic region starts at the CTA's shared window
    if (smem_u32(smem_raw) & 1023u) {
        if (threadIdx.x == 0) atomicCAS(err, 0, (int)KDA_ERR_DEVICE);
        return;
    }
    uint8_t* sm = smem_raw;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kBarOff);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kBarOff + 8);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int seq, tok0, len, idx;
    cmap.locate((int)blockIdx.x, seq, tok0, len, idx);
    const int h = (int)blockIdx.y;
    const size_t chunk = blockIdx.x;
    const size_t sbase = (chunk * H + h) * kD * kD;

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init_fence();
    }
    if (warp == 0) {
        tmem_alloc(tslot, kATmemCols);
        tmem_relinquish();
    }

    // ---- S and dS' (B operands, row = channel c, K = state column j) and dGam ----------
    // float4 index e = tid + 256 i: row c = e / 32 (warp w: rows w + 8 i), 4 columns of it
    float gsum[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int e = tid + 256 * i, c = e >> 5, j4 = (e & 31) * 4;
        const float4 s4 = *reinterpret_cast<const float4*>(S_chunk + sbase + (size_t)c * kD + j4);
        const float4 d4 = *reinterpret_cast<const float4*>(dS_chunk + sbase + (size_t)c * kD + j4);
        const uint32_t off = sw128_offset(c, j4, 128);
        store4_split(sm + kB1h, sm + kB1l, off, s4);
        store4_split(sm + kB2h, sm + kB2l, off, d4);
        gsum[i] = fmaf(s4.x, d4.x, fmaf(s4.y, d4.y, fmaf(s4.z, d4.z, s4.w * d4.w)));
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float v = gsum[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) dGam[(chunk * H + h) * kD + warp + 8 * i] = v;
    }
    // ---- dO (rows 0-63 of A1, exact in bf16: hi only, lo zero) ----------------------
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = tid + 256 * i, r = e >> 4, k8 = (e & 15) * 8;
        uint4 x = make_uint4(0u, 0u, 0u, 0u);
        if (r < len) x = *reinterpret_cast<const uint4*>(d_o + toff(tok0 + r, H, h) + k8);
        *reinterpret_cast<uint4*>(sm + kA1h + sw128_chunk(r, k8, 128)) = x;
        *reinterpret_cast<uint4*>(sm + kA1l + sw128_chunk(r, k8, 128)) = make_uint4(0u, 0u, 0u, 0u);
    }
    // ---- W (A2) and dW (rows 64-127 of A1) ---------------------------------------------
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = tid + 256 * i, r = e >> 5, j4 = (e & 31) * 4;
        float4 w4 = make_float4(0.f, 0.f, 0.f, 0.f), dw4 = w4;
        if (r < len) {
            w4 = *reinterpret_cast<const float4*>(W + toff(tok0 + r, H, h) + j4);
            dw4 = *reinterpret_cast<const float4*>(dW + toff(tok0 + r, H, h) + j4);
        }
        store4_split(sm + kA2h, sm + kA2l, sw128_offset(r, j4, 64), w4);
        store4_split(sm + kA1h, sm + kA1l, sw128_offset(64 + r, j4, 128), dw4);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;

    if (tid == 0) {
        const uint32_t a1h = smem_u32(sm + kA1h), a1l = smem_u32(sm + kA1l);
        const uint32_t a2h = smem_u32(sm + kA2h), a2l = smem_u32(sm + kA2l);
        const uint32_t b1h = smem_u32(sm + kB1h), b1l = smem_u32(sm + kB1l);
        const uint32_t b2h = smem_u32(sm + kB2h), b2l = smem_u32(sm + kB2l);
        for (int s = 0; s < kD / 16; ++s) {
            const uint32_t acc = s > 0 ? 1u : 0u;
            // D1 = [dO ; dW] S^T
            mma_bf16(tbase, sw128_desc_k(a1h, 128, s), sw128_desc_k(b1h, 128, s), idesc_bf16_f32(128, 128), acc);
            mma_bf16(tbase, sw128_desc_k(a1h, 128, s), sw128_desc_k(b1l, 128, s), idesc_bf16_f32(128, 128), 1u);
            mma_bf16(tbase, sw128_desc_k(a1l, 128, s), sw128_desc_k(b1h, 128, s), idesc_bf16_f32(128, 128), 1u);
            // D2 = W dS'^T
            mma_bf16(tbase + 128, sw128_desc_k(a2h, 64, s), sw128_desc_k(b2h, 128, s), idesc_bf16_f32(64, 128), acc);
            mma_bf16(tbase + 128, sw128_desc_k(a2h, 64, s), sw128_desc_k(b2l, 128, s), idesc_bf16_f32(64, 128), 1u);
            mma_bf16(tbase + 128, sw128_desc_k(a2l, 64, s), sw128_desc_k(b2h, 128, s), idesc_bf16_f32(64, 128), 1u);
            // D3 = dO W^T (dO: rows 0-63 of A1)
            mma_bf16(tbase + 256, sw128_desc_k(a1h, 128, s), sw128_desc_k(a2h, 64, s), idesc_bf16_f32(64, 64), acc);
            mma_bf16(tbase + 256, sw128_desc_k(a1h, 128, s), sw128_desc_k(a2l, 64, s), idesc_bf16_f32(64, 64), 1u);
        }
        mma_commit(bar);
    }
    // the warp-collective tensor-memory reads below need one answer for the whole CTA
    const bool ok = __syncthreads_and(mbar_wait(bar, 0) ? 1 : 0) != 0;
    if (!ok && tid == 0) atomicCAS(err, 0, (int)KDA_ERR_TIMEOUT);
    tc_fence_after();

    if (ok) {
        const int sp = warp & 3, half = warp >> 2;
        // D1: lane 32 sp + lane = row R (R < 64: dQg row R; R >= 64: -dWk row R - 64),
        // columns 64 half .. + 63
        {
            const int R = 32 * sp + lane;
            const int r = R & 63;
            float v[4][16];
#pragma unroll
            for (int g = 0; g < 4; ++g) tmem_ld16(tmem_addr(tbase, 32 * sp, 64 * half + 16 * g), v[g]);
            tmem_ld_wait();
            if (r < len) {
                float* dst = (R < 64 ? dQg : dWk) + toff(tok0 + r, H, h) + 64 * half;
                const float sg = R < 64 ? 1.f : -1.f;
#pragma unroll
                for (int g = 0; g < 4; ++g)
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4*>(dst + 16 * g + e) =
                            make_float4(sg * v[g][e], sg * v[g][e + 1], sg * v[g][e + 2], sg * v[g][e + 3]);
            }
        }
        // D2 and D3 (M = 64): row r = 16 sp + lane sits in lane 32 sp + lane for lanes 0-15
        {
            const int r = 16 * sp + (lane & 15);
            float v[4][16];
#pragma unroll
            for (int g = 0; g < 4; ++g) tmem_ld16(tmem_addr(tbase, 32 * sp, 128 + 64 * half + 16 * g), v[g]);
            tmem_ld_wait();
            if (lane < 16 && r < len) {
                float* dst = dKd + toff(tok0 + r, H, h) + 64 * half;
#pragma unroll
                for (int g = 0; g < 4; ++g)
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4*>(dst + 16 * g + e) =
                            make_float4(v[g][e], v[g][e + 1], v[g][e + 2], v[g][e + 3]);
            }
            float p[2][16];
#pragma unroll
            for (int g = 0; g < 2; ++g) tmem_ld16(tmem_addr(tbase, 32 * sp, 256 + 32 * half + 16 * g), p[g]);
            tmem_ld_wait();
            if (lane < 16) {
                float* dst = dP + (chunk * H + h) * kC * kC + (size_t)r * kC + 32 * half;
#pragma unroll
                for (int g = 0; g < 2; ++g)
#pragma unroll
                    for (int e = 0; e < 16; e += 4) {
                        float4 x;
                        const int i0 = 32 * half + 16 * g + e;
                        x.x = (r < len && i0 <= r) ? p[g][e] : 0.f;
                        x.y = (r < len && i0 + 1 <= r) ? p[g][e + 1] : 0.f;
                        x.z = (r < len && i0 + 2 <= r) ? p[g][e + 2] : 0.f;
                        x.w = (r < len && i0 + 3 <= r) ? p[g][e + 3] : 0.f;
                        *reinterpret_cast<float4*>(dst + 16 * g + e) = x;
                    }
            }
        }
    } else {
        // a wait gave up: let the products drain before the tensor memory is freed
        if (tid == 0) {
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < 100000000ull) {
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, kATmemCols);
}

}  // namespace

cudaError_t launch_kb_a_tc(const void* d_o, const float* W, const float* dW, const float* S_chunk,
                           const float* dS_chunk, float* dQg, float* dKd, float* dWk, float* dGam, float* dP, int* err,
                           const ChunkMap& cmap, int n_chunks, int H, cudaStream_t stream) {
    if (n_chunks == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kb_a_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kASmem);
    if (e != cudaSuccess) return e;
    kb_a_tc<<<dim3(n_chunks, H), kAThreads, kASmem, stream>>>((const __nv_bfloat16*)d_o, W, dW, S_chunk, dS_chunk,
                                                              dQg, dKd, dWk, dGam, dP, err, cmap, H);
    return cudaGetLastError();
}

}  // namespace kda
