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
//
// kb_chain_tc, the reverse chain (described with the kernel below), and
// kb_b_tc, the back substitution through the WY/UT transform, per (chunk, head),
// with T = (I + A)^{-1} stored by the recompute:
//     [Y | Z] = T^T [dW | dWk]          (M =  64, N = 256, K =  64)
//     dA = -[Y | Z] [U | Wk]^T, i < r   (M =  64, N =  64, K = 256)
// then dv = beta Y, dKg = beta Z, dbeta_r = v_r.Y_r + Kg_r.Z_r + sum_i dA_ri At_ri
// and dAt = Diag(beta) dA on CUDA cores.  U and Wk come straight from the
// recompute's per-chunk image (U fp32, Wk as its hi/lo bf16 rows).  T's row-major image is the MN-major A
// operand of the first product, [dW | dWk] its MN-major B operand; the second
// reads [Y | Z] (from tensor memory, split into bf16 hi/lo) as its K-major A
// operand and [U | Wk] as its K-major B operand.
#include "kda_internal.cuh"
#include "kda_tc.cuh"
#include "kda_tc_image.cuh"

namespace kda {
namespace {

using namespace tc;
using namespace tcimg;

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

__device__ __forceinline__ void record_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// multiprocessors of the current device, looked up once per device
int sm_count_bwd() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

// eight consecutive values (one 16-byte chunk) split into hi and lo images
__device__ __forceinline__ void store8_split_tc(uint8_t* hi, uint8_t* lo, uint32_t off, const float* x) {
    uint4 hv, lv;
    split2(x[0], x[1], hv.x, lv.x);
    split2(x[2], x[3], hv.y, lv.y);
    split2(x[4], x[5], hv.z, lv.z);
    split2(x[6], x[7], hv.w, lv.w);
    *reinterpret_cast<uint4*>(hi + off) = hv;
    *reinterpret_cast<uint4*>(lo + off) = lv;
}

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

// ---------------------------------------------------------------------------- kb_b_tc
constexpr uint32_t kBTh = 0;          // T, row-major 64 x 64 (MN-major A of the first product)
constexpr uint32_t kBTl = 8192;
constexpr uint32_t kBXh = 16384;      // [dW | dWk] row-major 64 x 256, then [Y | Z] (K-major A)
constexpr uint32_t kBXl = 49152;
constexpr uint32_t kBUh = 81920;      // [U | Wk] row-major 64 x 256 (K-major B of the second)
constexpr uint32_t kBUl = 114688;
constexpr uint32_t kBBar = 147456;    // mbarrier, tensor-memory base, dbeta sums [64]
constexpr uint32_t kBSmem = kBBar + 16 + kC * 4;

__host__ __device__ constexpr uint32_t idesc_amn_bmn(int M, int N) {
    return idesc_bf16_f32(M, N) | (1u << 15) | (1u << 16);
}

// one 64 x 256 row-major image from two 64 x 128 fp32 arrays (rows past len zero)
__device__ __forceinline__ void stage_pair(uint8_t* hi, uint8_t* lo, const float* a, const float* b, int tok0,
                                           int len, int H, int h, int tid) {
#pragma unroll 4
    for (int u = 0; u < 16; ++u) {
        const int e = tid + kAThreads * u, i = e >> 6, j4 = (e & 63) * 4;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < len) x = *reinterpret_cast<const float4*>((j4 < kD ? a : b) + toff(tok0 + i, H, h) + (j4 & 127));
        store4_split(hi, lo, sw128_offset(i, j4, 64), x);
    }
}

// [U | Wk] (64 token rows x 256, K-major) straight from the recompute's image of
// this (chunk, head): U from its fp32 tile, split as above; Wk's hi and lo bf16
// chunks copied as they are (rows 0-63 of the [Wk ; Q exp(g)] image); rows past
// the chunk's end zero.
__device__ __forceinline__ void stage_u_wk_image(uint8_t* hi, uint8_t* lo, const uint8_t* img, int len, int tid) {
    const float* u = reinterpret_cast<const float*>(img + kOffU);
#pragma unroll 4
    for (int it = 0; it < 8; ++it) {
        const int e = tid + kAThreads * it, i = e >> 5, j4 = (e & 31) * 4;
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (i < len) x = *reinterpret_cast<const float4*>(u + u_index(i, j4));
        store4_split(hi, lo, sw128_offset(i, j4, 64), x);
    }
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int e = tid + kAThreads * it, i = e >> 4, j8 = (e & 15) * 8;
        uint4 xh = make_uint4(0u, 0u, 0u, 0u), xl = xh;
        if (i < len) {
            xh = *reinterpret_cast<const uint4*>(img + kOffWkQh + sw128_chunk(i, j8, 128));
            xl = *reinterpret_cast<const uint4*>(img + kOffWkQl + sw128_chunk(i, j8, 128));
        }
        *reinterpret_cast<uint4*>(hi + sw128_chunk(i, kD + j8, 64)) = xh;
        *reinterpret_cast<uint4*>(lo + sw128_chunk(i, kD + j8, 64)) = xl;
    }
}

__global__ void __launch_bounds__(kAThreads, 1)
kb_b_tc(const float* __restrict__ T, const float* __restrict__ At, const uint8_t* __restrict__ images,
        const float* __restrict__ dW, const float* __restrict__ dWk,
        const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
        const __nv_bfloat16* __restrict__ beta, const float* __restrict__ g, const float* __restrict__ gl,
        __nv_bfloat16* __restrict__ dv_out, __nv_bfloat16* __restrict__ dbeta_out, float* __restrict__ dKg,
        float* __restrict__ dAt, int* __restrict__ err, ChunkMap cmap, int H) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    if (smem_u32(smem_raw) & 1023u) {
        if (threadIdx.x == 0) atomicCAS(err, 0, (int)KDA_ERR_DEVICE);
        return;
    }
    uint8_t* sm = smem_raw;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kBBar);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kBBar + 8);
    float* dbs = reinterpret_cast<float*>(sm + kBBar + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int seq, tok0, len, idx;
    cmap.locate((int)blockIdx.x, seq, tok0, len, idx);
    const int h = (int)blockIdx.y;
    const size_t chunk = blockIdx.x;
    const size_t cbase = (chunk * H + h) * (size_t)(kC * kC);

    if (tid == 0) {
        mbar_init(bar, 1);
        mbar_init_fence();
    }
    if (tid < kC) dbs[tid] = 0.f;
    if (warp == 0) {
        tmem_alloc(tslot, kATmemCols);
        tmem_relinquish();
    }
    // ---- operands ------------------------------------------------------------------------
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int e = tid + kAThreads * u, i = e >> 4, c4 = (e & 15) * 4;
        const float4 x = *reinterpret_cast<const float4*>(T + cbase + (size_t)i * kC + c4);
        store4_split(sm + kBTh, sm + kBTl, sw128_offset(i, c4, 64), x);
    }
    stage_pair(sm + kBXh, sm + kBXl, dW, dWk, tok0, len, H, h, tid);
    stage_u_wk_image(sm + kBUh, sm + kBUl, images + (chunk * H + h) * (size_t)kChunkBytes, len, tid);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;
    // ---- [Y | Z] = T^T [dW | dWk] ------------------------------------------------------------
    if (tid == 0) {
        const uint32_t th = smem_u32(sm + kBTh), tl = smem_u32(sm + kBTl);
        const uint32_t xh = smem_u32(sm + kBXh), xl = smem_u32(sm + kBXl);
        for (int s = 0; s < kC / 16; ++s) {
            const uint32_t acc = s > 0 ? 1u : 0u;
            mma_bf16(tbase, mn_desc_k(th, kC, s), mn_desc_k(xh, kC, s), idesc_amn_bmn(64, 256), acc);
            mma_bf16(tbase, mn_desc_k(th, kC, s), mn_desc_k(xl, kC, s), idesc_amn_bmn(64, 256), 1u);
            mma_bf16(tbase, mn_desc_k(tl, kC, s), mn_desc_k(xh, kC, s), idesc_amn_bmn(64, 256), 1u);
        }
        mma_commit(bar);
    }
    bool ok = __syncthreads_and(mbar_wait(bar, 0) ? 1 : 0) != 0;
    tc_fence_after();
    const int sp = warp & 3, half = warp >> 2;
    const int r = 16 * sp + (lane & 15);
    const bool row_lane = lane < 16;
    const bool valid = row_lane && r < len;
    const float br = valid ? __bfloat162float(beta[(size_t)(tok0 + r) * H + h]) : 0.f;
    float part = 0.f;   // this lane's share of dbeta_r
    if (ok) {
        // half 0: Y (columns 0-127), half 1: Z (128-255), 32 columns at a time
        for (int qq = 0; qq < 4; ++qq) {
            const int jb = 128 * half + 32 * qq;
            float y[32];
            {
                float a[16], b[16];
                tmem_ld16(tmem_addr(tbase, 32 * sp, jb), a);
                tmem_ld16(tmem_addr(tbase, 32 * sp, jb + 16), b);
                tmem_ld_wait();
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    y[x] = a[x];
                    y[16 + x] = b[x];
                }
            }
            if (row_lane) {
#pragma unroll
                for (int x = 0; x < 4; ++x) store8_split_tc(sm + kBXh, sm + kBXl, sw128_chunk(r, jb + 8 * x, 64), y + 8 * x);
            }
            if (valid) {
                const size_t ro = toff(tok0 + r, H, h);
                if (half == 0) {
#pragma unroll
                    for (int x = 0; x < 32; x += 8) {
                        const uint4 vv = *reinterpret_cast<const uint4*>(v + ro + jb + x);
                        const uint32_t w4[4] = {vv.x, vv.y, vv.z, vv.w};
                        uint4 o;
                        uint32_t* o4 = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            const float2 vf = unpack_bf16x2(w4[m]);
                            part = fmaf(vf.x, y[x + 2 * m], fmaf(vf.y, y[x + 2 * m + 1], part));
                            o4[m] = pack_bf16(br * y[x + 2 * m], br * y[x + 2 * m + 1]);
                        }
                        *reinterpret_cast<uint4*>(dv_out + ro + jb + x) = o;
                    }
                } else {
                    const int cb = jb - 128;
#pragma unroll
                    for (int x = 0; x < 32; x += 8) {
                        const uint4 kk = *reinterpret_cast<const uint4*>(k + ro + cb + x);
                        const uint32_t w4[4] = {kk.x, kk.y, kk.z, kk.w};
                        float gv[8], lv[8];
                        *reinterpret_cast<float4*>(gv) = *reinterpret_cast<const float4*>(g + ro + cb + x);
                        *reinterpret_cast<float4*>(gv + 4) = *reinterpret_cast<const float4*>(g + ro + cb + x + 4);
                        *reinterpret_cast<float4*>(lv) = *reinterpret_cast<const float4*>(gl + ro + cb + x);
                        *reinterpret_cast<float4*>(lv + 4) = *reinterpret_cast<const float4*>(gl + ro + cb + x + 4);
#pragma unroll
                        for (int m = 0; m < 4; ++m) {
                            const float2 kf = unpack_bf16x2(w4[m]);
                            part = fmaf(kf.x * exp_g(gv[2 * m], lv[2 * m]), y[x + 2 * m], part);
                            part = fmaf(kf.y * exp_g(gv[2 * m + 1], lv[2 * m + 1]), y[x + 2 * m + 1], part);
                        }
                        *reinterpret_cast<float4*>(dKg + ro + cb + x) =
                            make_float4(br * y[x], br * y[x + 1], br * y[x + 2], br * y[x + 3]);
                        *reinterpret_cast<float4*>(dKg + ro + cb + x + 4) =
                            make_float4(br * y[x + 4], br * y[x + 5], br * y[x + 6], br * y[x + 7]);
                    }
                }
            }
        }
    }
    // ---- dA = -[Y | Z] [U | Wk]^T ------------------------------------------------------------
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0 && ok) {
        const uint32_t ah = smem_u32(sm + kBXh), al = smem_u32(sm + kBXl);
        const uint32_t bh = smem_u32(sm + kBUh), bl = smem_u32(sm + kBUl);
        for (int s = 0; s < 256 / 16; ++s) {
            const uint32_t acc = s > 0 ? 1u : 0u;
            mma_bf16(tbase + 256, sw128_desc_k(ah, 64, s), sw128_desc_k(bh, 64, s), idesc_bf16_f32(64, 64), acc);
            mma_bf16(tbase + 256, sw128_desc_k(ah, 64, s), sw128_desc_k(bl, 64, s), idesc_bf16_f32(64, 64), 1u);
            mma_bf16(tbase + 256, sw128_desc_k(al, 64, s), sw128_desc_k(bh, 64, s), idesc_bf16_f32(64, 64), 1u);
        }
        mma_commit(bar);
    }
    if (ok) ok = __syncthreads_and(mbar_wait(bar, 1) ? 1 : 0) != 0;
    else __syncthreads();
    tc_fence_after();
    if (!ok && tid == 0) atomicCAS(err, 0, (int)KDA_ERR_TIMEOUT);
    if (ok) {
        const int ib = 32 * half;
        float d[32];
        {
            float a[16], b[16];
            tmem_ld16(tmem_addr(tbase, 32 * sp, 256 + ib), a);
            tmem_ld16(tmem_addr(tbase, 32 * sp, 256 + ib + 16), b);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                d[x] = a[x];
                d[16 + x] = b[x];
            }
        }
        if (row_lane) {
            const float* atr = At + cbase + (size_t)r * kC + ib;
            float* dst = dAt + cbase + (size_t)r * kC + ib;
#pragma unroll
            for (int x = 0; x < 32; x += 4) {
                float da[4];
#pragma unroll
                for (int m = 0; m < 4; ++m) da[m] = (valid && ib + x + m < r) ? -d[x + m] : 0.f;
                const float4 a4 = *reinterpret_cast<const float4*>(atr + x);
                part = fmaf(da[0], a4.x, fmaf(da[1], a4.y, fmaf(da[2], a4.z, fmaf(da[3], a4.w, part))));
                *reinterpret_cast<float4*>(dst + x) = make_float4(br * da[0], br * da[1], br * da[2], br * da[3]);
            }
            atomicAdd(&dbs[r], part);
        }
    } else {
        if (tid == 0) {
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < 100000000ull) {
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (ok && tid < len) dbeta_out[(size_t)(tok0 + tid) * H + h] = __float2bfloat16_rn(dbs[tid]);
    if (warp == 0) tmem_dealloc(tbase, kATmemCols);
}

// ---------------------------------------------------------------------------- kb_chain_tc
// The mirror of tc_recur, for the gradients (bf16, d = 128).  Per chunk, walking
// each sequence backwards with the gradient dS' of the chunk's end state (fp32,
// 128 x BV columns) in tensor memory:
//     dW  = Kd dS' + P^T dO                    (M =  64, N = BV)
//     dS  = Diag(Gamma_C) dS' + Qg^T dO - Wk^T dW   (M = 128, N = BV)
// (the chain rule through W = U - Wk S, O = Qg S + P W and S' = Diag(Gamma_C) S +
// Kd^T W).  The operands are the forward's per-chunk images, which the recompute
// left in the workspace: Kd^T (rows = channels) serves as the MN-major A operand
// of Kd dS', P as that of P^T dO, and the two halves of [Wk ; Q exp(g)] as those of
// Wk^T dW and Qg^T dO.  dO (bf16, exact in one term) is staged as an MN-major B
// image by the CUDA cores.  Stores each chunk's dS' (dS_chunk) and dW (fp32), and
// the initial-state gradient at the end.
constexpr int kChainThreads = 256;

template <int BV>
struct ChainLayout {
    static constexpr uint32_t kWkQ = 0;                 // hi 32 KB + lo 32 KB
    static constexpr uint32_t kKdT = 65536;             // hi 16 KB + lo 16 KB
    static constexpr uint32_t kP = 98304;               // hi 8 KB + lo 8 KB
    static constexpr uint32_t kDO = 114688;             // dO, 64 rows x 128 B (first BV columns used)
    static constexpr uint32_t kDS = 122880;             // dS' hi/lo, 128 rows x 128 B each
    static constexpr uint32_t kDW = kDS + 32768;        // -dW hi/lo, 64 rows x 128 B each
    static constexpr uint32_t kGam = kDW + 16384;       // Gamma_C fp32 [128]
    static constexpr uint32_t kBars = kGam + 512;
    static constexpr uint32_t kSmem = kBars + 128;
    static constexpr uint32_t kAlloc = kSmem + 1024;
    static constexpr uint32_t kTmemCols = (2 * BV <= 64) ? 64 : 128;   // dS' (128 lanes) | dW (M = 64)
};

// descriptor of the K-slice [16 s, 16 s + 16) of an MN-major operand whose
// 64-wide M (or N) blocks lie `block_stride` bytes apart (K rows of 128 bytes)
__device__ __forceinline__ uint64_t mn_desc_ks(uint32_t addr, uint32_t block_stride, int s) {
    const uint32_t a = addr + (uint32_t)s * 2048u;
    uint64_t d = (uint64_t)((a >> 4) & 0x3FFFu);
    d |= (uint64_t)((block_stride >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

template <int BV>
__global__ void __launch_bounds__(kChainThreads, 1)
kb_chain_tc(const uint8_t* __restrict__ ws, const __nv_bfloat16* __restrict__ d_o, const float* __restrict__ d_final,
            float* __restrict__ dS_chunk, float* __restrict__ dW_out, float* __restrict__ d_init,
            int* __restrict__ err, SeqMap smap, int H) {
    using Lay = ChainLayout<BV>;
    constexpr int HB = BV / 2;          // state columns per thread
    constexpr int NG = HB / 16;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::kBars);
    uint64_t* wkq_full = bars + 0;
    uint64_t* kdp_full = bars + 1;      // Kd^T, P and Gamma_C landed
    uint64_t* bar_w = bars + 2;         // dW products done
    uint64_t* bar_s = bars + 3;         // dS products done
    uint32_t* sflags = reinterpret_cast<uint32_t*>(bars + 4);   // [0] tmem base, [1] abort
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = warp & 3, cq = (warp >> 2) * HB;
    constexpr int kTiles = kD / BV;
    const int z = (int)(blockIdx.x % kTiles);
    const int h = (int)((blockIdx.x / kTiles) % (unsigned)H);
    const SeqInfo sq = smap.get((int)(blockIdx.x / (kTiles * (unsigned)H)));
    const int j0 = z * BV;
    const int nch = (sq.len + kC - 1) / kC;
    const float* gam_s = reinterpret_cast<const float*>(sm + Lay::kGam);

    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bars[i], 1);
        sflags[1] = 0;
        mbar_init_fence();
    }
    if (warp == 0) {
        tmem_alloc(&sflags[0], Lay::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sflags[0];
    const uint32_t t_s = tbase, t_w = tbase + BV;   // dS' (all 128 lanes), dW (M = 64 layout)

    auto chunk_src = [&](int n) { return ws + (size_t)((size_t)(sq.chunk0 + n) * H + h) * kChunkBytes; };
    auto load_wkq = [&](int n) {
        const uint8_t* src = chunk_src(n);
        mbar_arrive_expect_tx(wkq_full, 65536);
        bulk_g2s(sm + Lay::kWkQ, src + kOffWkQh, 32768, wkq_full);
        bulk_g2s(sm + Lay::kWkQ + 32768, src + kOffWkQl, 32768, wkq_full);
    };
    auto load_kdp = [&](int n) {
        const uint8_t* src = chunk_src(n);
        mbar_arrive_expect_tx(kdp_full, 32768 + 16384 + 512);
        bulk_g2s(sm + Lay::kKdT, src + kOffKdTh, 16384, kdp_full);
        bulk_g2s(sm + Lay::kKdT + 16384, src + kOffKdTl, 16384, kdp_full);
        bulk_g2s(sm + Lay::kP, src + kOffPh, 8192, kdp_full);
        bulk_g2s(sm + Lay::kP + 8192, src + kOffPl, 8192, kdp_full);
        bulk_g2s(sm + Lay::kGam, src + kOffGam, 512, kdp_full);
    };
    // dO of chunk n (rows r < L, columns j0 .. j0 + BV) as the MN-major B image; zero rows past L
    auto stage_do = [&](int n) {
        const int L = min(kC, sq.len - n * kC);
        for (int e = tid; e < kC * (BV / 8); e += kChainThreads) {
            const int r = e / (BV / 8), c8 = (e - r * (BV / 8)) * 8;
            uint4 x = make_uint4(0u, 0u, 0u, 0u);
            if (r < L) x = *reinterpret_cast<const uint4*>(d_o + ((size_t)(sq.tok0 + n * kC + r) * H + h) * kD + j0 + c8);
            *reinterpret_cast<uint4*>(sm + Lay::kDO + mn_chunk(r, c8, kC)) = x;
        }
    };
    auto fail = [&]() {
        record_error(err, KDA_ERR_TIMEOUT);
        atomicExch(&sflags[1], 1u);
    };
    if (tid == 0 && nch > 0) {
        load_wkq(nch - 1);
        load_kdp(nch - 1);
    }
    if (nch > 0) stage_do(nch - 1);

    // this thread's row c of dS', columns j0 + cq + [0, HB)
    const int c = 32 * sp + lane;
    float s[HB];
    {
        const size_t base = (((size_t)sq.seq * H + h) * kD + c) * kD + j0 + cq;
#pragma unroll
        for (int j = 0; j < HB; j += 4) {
            const float4 x = d_final ? *reinterpret_cast<const float4*>(d_final + base + j)
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
            s[j] = x.x; s[j + 1] = x.y; s[j + 2] = x.z; s[j + 3] = x.w;
        }
    }
    const uint32_t a_wk = smem_u32(sm + Lay::kWkQ), a_kd = smem_u32(sm + Lay::kKdT), a_p = smem_u32(sm + Lay::kP);
    const uint32_t b_do = smem_u32(sm + Lay::kDO), b_ds = smem_u32(sm + Lay::kDS), b_dw = smem_u32(sm + Lay::kDW);
    uint32_t par = 0;
    for (int n = nch - 1; n >= 0; --n, par ^= 1u) {
        const int L = min(kC, sq.len - n * kC);
        // dS' of this chunk: to the workspace, as the B image, and Gamma_C dS' into tensor memory
        {
            float* dst = dS_chunk + ((((size_t)sq.chunk0 + n) * H + h) * kD + c) * kD + j0 + cq;
#pragma unroll
            for (int j = 0; j < HB; j += 4)
                *reinterpret_cast<float4*>(dst + j) = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
        }
#pragma unroll
        for (int j = 0; j < HB; j += 8) store8_split_tc(sm + Lay::kDS, sm + Lay::kDS + 16384, mn_chunk(c, cq + j, 128), s + j);
        if (!mbar_wait(kdp_full, par)) fail();
        const float gam = gam_s[c];
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            float t[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) t[e] = gam * s[16 * g + e];
            tmem_st16(tmem_addr(t_s, 32 * sp, cq + 16 * g), t);
        }
        tmem_st_wait();
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (sflags[1]) break;
        tc_fence_after();
        if (tid == 0) {
            // dW = Kd dS' + P^T dO
            for (int k = 0; k < kD / 16; ++k) {
                const uint64_t ah = mn_desc_ks(a_kd, 16384, k), al = mn_desc_ks(a_kd + 16384, 16384, k);
                const uint64_t bh = mn_desc_ks(b_ds, 16384, k), bl = mn_desc_ks(b_ds + 16384, 16384, k);
                const uint32_t id = idesc_amn_bmn(64, BV);
                mma_bf16(t_w, ah, bh, id, k > 0 ? 1u : 0u);
                mma_bf16(t_w, ah, bl, id, 1u);
                mma_bf16(t_w, al, bh, id, 1u);
            }
            for (int k = 0; k < kC / 16; ++k) {
                const uint64_t ah = mn_desc_ks(a_p, 8192, k), al = mn_desc_ks(a_p + 8192, 8192, k);
                const uint64_t bd = mn_desc_ks(b_do, 8192, k);
                const uint32_t id = idesc_amn_bmn(64, BV);
                mma_bf16(t_w, ah, bd, id, 1u);
                mma_bf16(t_w, al, bd, id, 1u);
            }
            mma_commit(bar_w);
            // dS += Qg^T dO (independent of the chain: runs while dW is read back)
            if (!mbar_wait(wkq_full, par)) {
                fail();
            } else {
                for (int k = 0; k < kC / 16; ++k) {
                    const uint64_t ah = mn_desc_ks(a_wk + 8192, 16384, k), al = mn_desc_ks(a_wk + 32768 + 8192, 16384, k);
                    const uint64_t bd = mn_desc_ks(b_do, 8192, k);
                    const uint32_t id = idesc_amn_bmn(128, BV);
                    mma_bf16(t_s, ah, bd, id, 1u);
                    mma_bf16(t_s, al, bd, id, 1u);
                }
            }
        }
        if (!mbar_wait(bar_w, par)) fail();
        tc_fence_after();
        if (tid == 0 && n > 0) load_kdp(n - 1);   // Kd^T, P (and Gamma_C) have been read
        // dW (M = 64 layout: row r in lanes 0-15 of sub-partition r / 16): to the workspace
        // and, negated, as the B image of Wk^T dW
        {
            const int r = 16 * sp + (lane & 15);
            float d[NG][16];
#pragma unroll
            for (int g = 0; g < NG; ++g) tmem_ld16(tmem_addr(t_w, 32 * sp, cq + 16 * g), d[g]);
            tmem_ld_wait();
            if (lane < 16) {
#pragma unroll
                for (int g = 0; g < NG; ++g) {
                    if (r < L) {
                        float* dst = dW_out + ((size_t)(sq.tok0 + n * kC + r) * H + h) * kD + j0 + cq + 16 * g;
#pragma unroll
                        for (int e = 0; e < 16; e += 4)
                            *reinterpret_cast<float4*>(dst + e) = make_float4(d[g][e], d[g][e + 1], d[g][e + 2], d[g][e + 3]);
                    }
                    float nd[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) nd[e] = (r < L) ? -d[g][e] : 0.f;
                    store8_split_tc(sm + Lay::kDW, sm + Lay::kDW + 8192, mn_chunk(r, cq + 16 * g, kC), nd);
                    store8_split_tc(sm + Lay::kDW, sm + Lay::kDW + 8192, mn_chunk(r, cq + 16 * g + 8, kC), nd + 8);
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            // dS += Wk^T (-dW)
            for (int k = 0; k < kC / 16; ++k) {
                const uint64_t ah = mn_desc_ks(a_wk, 16384, k), al = mn_desc_ks(a_wk + 32768, 16384, k);
                const uint64_t bh = mn_desc_ks(b_dw, 8192, k), bl = mn_desc_ks(b_dw + 8192, 8192, k);
                const uint32_t id = idesc_amn_bmn(128, BV);
                mma_bf16(t_s, ah, bh, id, 1u);
                mma_bf16(t_s, ah, bl, id, 1u);
                mma_bf16(t_s, al, bh, id, 1u);
            }
            mma_commit(bar_s);
        }
        if (!mbar_wait(bar_s, par)) fail();
        tc_fence_after();
        __syncthreads();   // every MMA of this chunk is done: the [Wk ; Qg] and dO buffers are free
        if (tid == 0 && n > 0) load_wkq(n - 1);
        if (n > 0) stage_do(n - 1);
        {
            float t[NG][16];
#pragma unroll
            for (int g = 0; g < NG; ++g) tmem_ld16(tmem_addr(t_s, 32 * sp, cq + 16 * g), t[g]);
            tmem_ld_wait();
#pragma unroll
            for (int g = 0; g < NG; ++g)
#pragma unroll
                for (int e = 0; e < 16; ++e) s[16 * g + e] = t[g][e];
        }
    }
    __syncthreads();
    const bool failed = sflags[1] != 0;
    if (!failed && d_init) {
        const size_t base = (((size_t)sq.seq * H + h) * kD + c) * kD + j0 + cq;
#pragma unroll
        for (int j = 0; j < HB; j += 4)
            *reinterpret_cast<float4*>(d_init + base + j) = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
    }
    if (failed && tid == 0) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 100000000ull) {
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, Lay::kTmemCols);
}

template <int BV>
cudaError_t launch_chain(const uint8_t* ws, const void* d_o, const float* d_final, float* dS_chunk, float* dW,
                         float* d_init, int* err, const SeqMap& smap, int n_seqs, int H, cudaStream_t stream) {
    using Lay = ChainLayout<BV>;
    cudaError_t e = cudaFuncSetAttribute(kb_chain_tc<BV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::kAlloc);
    if (e != cudaSuccess) return e;
    kb_chain_tc<BV><<<dim3((unsigned)(n_seqs * H * (kD / BV))), kChainThreads, Lay::kAlloc, stream>>>(
        ws, (const __nv_bfloat16*)d_o, d_final, dS_chunk, dW, d_init, err, smap, H);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_kb_b_tc(const float* T, const float* At, const void* tc_ws, const float* dW,
                           const float* dWk, const void* k, const void* v, const void* beta, const float* g,
                           const float* gl, void* dv_out, void* dbeta_out, float* dKg, float* dAt, int* err,
                           const ChunkMap& cmap, int n_chunks, int H, cudaStream_t stream) {
    if (n_chunks == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kb_b_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kBSmem);
    if (e != cudaSuccess) return e;
    const uint8_t* images = reinterpret_cast<const uint8_t*>(tc_ws) + kErrHeader;
    kb_b_tc<<<dim3(n_chunks, H), kAThreads, kBSmem, stream>>>(
        T, At, images, dW, dWk, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, (const __nv_bfloat16*)beta, g, gl,
        (__nv_bfloat16*)dv_out, (__nv_bfloat16*)dbeta_out, dKg, dAt, err, cmap, H);
    return cudaGetLastError();
}

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

// The backward pass's reverse chain on the tensor cores, from the per-chunk
// images the recompute (launch_tc_states) left in tc_ws.
cudaError_t launch_tc_chain(void* tc_ws, const void* d_o, const float* d_final, float* dS_chunk, float* dW,
                            float* d_init, const SeqMap& smap, int n_seqs, int H, cudaStream_t stream) {
    if (n_seqs == 0) return cudaSuccess;
    int* err = reinterpret_cast<int*>(tc_ws);
    const uint8_t* ws = reinterpret_cast<const uint8_t*>(tc_ws) + kErrHeader;
    if ((long)n_seqs * H * 4 <= sm_count_bwd())
        return launch_chain<32>(ws, d_o, d_final, dS_chunk, dW, d_init, err, smap, n_seqs, H, stream);
    return launch_chain<64>(ws, d_o, d_final, dS_chunk, dW, d_init, err, smap, n_seqs, H, stream);
}

}  // namespace kda
