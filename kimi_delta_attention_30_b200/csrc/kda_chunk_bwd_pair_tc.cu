// Tensor-core (tcgen05) pairwise gradient terms of the KDA backward pass, for
// bf16 inputs with d_k = 128 and 64-token chunks (kb_c_tc).
//
// Per (chunk, head) the chunk form has the decayed key products
// At_ri = sum_c k_rc k_ic E_ric (i < r) and scores P_ri = sum_c q_rc k_ic E_ric
// (i <= r), E_ric = exp(g_rc - g_ic) with g the chunk's cumulative log decay
// ("From GPT-2 to Kimi K3" essay, pwwt.cn/news/3716252, chunkwise paragraph, for
// the form; the pages give no backward pass, so this is the chain rule through
// it).  Given their gradients dAt and dP (from the back substitution and the
// chunk-local products) and the gradients of the elementwise factors
// (dQg, dKg, dKd, dGam), per channel c:
//     X1_r = sum_{i<r}  dAt_ri k_i E_ri          X2_r = sum_{i<r} dP_ri k_i E_ri
//     Y_i  = sum_{r>i} (dAt_ri k_r + dP_ri q_r) E_ri
//     dq_r = X2_r + dP_rr k_r + dQg_r e^{g_r}
//     dk_r = X1_r + Y_r + dP_rr q_r + dKg_r e^{g_r} + dKd_r e^{g_last - g_r}
// and dlog alpha_j collects every term whose decay spans token j: the pairwise
// terms T_ri = (dAt_ri k_r + dP_ri q_r) k_i E_ri with i < j <= r sum to
//     F(j) = sum_{r >= j} D_r,   D_r = k_r X1_r + q_r X2_r - k_r Y_r
// (row sums minus column sums; the pairs with both ends at or after j cancel),
// so  dlog alpha_j = F(j) + sum_{r<j} dKd_r Kd_r + sum_{r>=j} (dQg_r Qg_r +
// dKg_r Kg_r) + dGam Gam, zero where the forward's floor on log alpha was active.
// The diagonal of dP enters X2 and Y only elementwise: in D_r its two
// appearances cancel exactly, and in a strongly decaying head F(j) is far
// smaller than that term, so its rounding in the products would dominate.
//
// X and Y are products with the channels as the MMA's M (128 rows of tensor
// memory: the thread that reads lane c owns channel c, so the per-channel
// cumulative sums stay in one thread) and the rows/keys as N, in block-
// referenced form as in the forward's first product.  For row block I
// (16 rows) the keys are scaled by e^{gb_I - g_i}, gb_I = g at the row before the
// block, and the result by e^{g_r - gb_I}; for key block J the rows are scaled by
// e^{g_r - ge_J}, ge_J = g at the block's last row, and the result by
// e^{ge_J - g_i}.  Every factor is <= 1 except on the diagonal blocks, where it is
// at most e^{range of the block}; a block whose decay range exceeds 80 nats is
// left out of the products and its pairs are summed exactly on CUDA cores by the
// threads that own the channels.  Operands are bf16 hi/lo images with every
// product formed as hi*hi + hi*lo + lo*hi, fp32 accumulation in tensor memory:
//     X  (cols   0-127): for block I, A = key version I (K = 16 (I + 1) keys,
//                        M-major), B = [dAt ; dP] rows of block I (N = 32, K-major)
//     Y  (cols 128-191): for block J, A = row versions of k, then of q (K = rows
//                        16 J .. 63, M-major), B = dAt^T, then dP^T, keys of J
// The versions of k and q are built in two 80 KB buffers while the previous
// product runs; the CTA holds 229.5 KB of shared memory (one per SM).
#include "kda_internal.cuh"
#include "kda_tc.cuh"

namespace kda {
namespace {

using namespace tc;

constexpr int kQT = 256;   // threads
constexpr int kQC = 64;    // tokens per chunk
constexpr int kQD = 128;   // channels (d_k)
// shared memory, byte offsets from the 1024-aligned dynamic base
constexpr uint32_t kV0 = 0;           // key versions; later the row versions of q
constexpr uint32_t kV1 = 81920;       // row versions of k (at first: dAt, dP in fp32)
constexpr uint32_t kVLo = 40960;      // lo image, from the start of a version buffer
constexpr uint32_t kImX = 163840;     // [dAt ; dP] rows per block: row 32 I + x dAt, 32 I + 16 + x dP (128 rows)
constexpr uint32_t kImXLo = 16384;
constexpr uint32_t kImAT = 196608;    // dAt^T, rows = keys, K = rows r
constexpr uint32_t kImPT = 204800;    // dP^T (no diagonal)
constexpr uint32_t kImTLo = 16384;    // lo images of dAt^T and dP^T
constexpr uint32_t kBarOff = 229376;  // two mbarriers, the tensor-memory base
constexpr uint32_t kQSmem = kBarOff + 64;
constexpr uint32_t kQTmemCols = 256;
constexpr float kRangeMax = 80.f;     // nats: the largest decay range a diagonal block may span in the products
// epilogue arrays (fp32 [64][128]) and the diagonal blocks, once every product is done
constexpr uint32_t kEX1 = 0, kEX2 = 32768, kEY = 65536, kEDiag = 98304, kETab = 106496;

static_assert(kImAT + 2 * 8192 == kImPT + 8192 && kImPT + kImTLo == 221184, "transposed image layout");
static_assert(kQSmem <= 232448, "shared memory per block");

// byte offset of key version I (K = 16 (I + 1) rows) and of row version J (K = 64 - 16 J rows)
__host__ __device__ constexpr uint32_t kv_off(int I) { return 2048u * (uint32_t)(I * (I + 1)); }
__host__ __device__ constexpr uint32_t rv_off(int J) { return 4096u * (uint32_t)(4 * J - J * (J - 1) / 2); }

__device__ __forceinline__ size_t toff(int t, int H, int h) { return ((size_t)t * H + h) * kQD; }

// instruction descriptor: bf16 operands, fp32 accumulator, A M-major, B K-major
__host__ __device__ constexpr uint32_t idesc_amn(int M, int N) { return idesc_bf16_f32(M, N) | (1u << 15); }

__device__ __forceinline__ void store8_split(uint8_t* hi, uint8_t* lo, uint32_t off, const float* x) {
    uint4 hv, lv;
    split2(x[0], x[1], hv.x, lv.x);
    split2(x[2], x[3], hv.y, lv.y);
    split2(x[4], x[5], hv.z, lv.z);
    split2(x[6], x[7], hv.w, lv.w);
    *reinterpret_cast<uint4*>(hi + off) = hv;
    *reinterpret_cast<uint4*>(lo + off) = lv;
}

__device__ __forceinline__ void bf16x8_to_f32(uint4 u, float* x) {
    const float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y), c = unpack_bf16x2(u.z), d = unpack_bf16x2(u.w);
    x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y; x[4] = c.x; x[5] = c.y; x[6] = d.x; x[7] = d.y;
}

__device__ __forceinline__ void load8f(const float* p, float* x) {
    const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w; x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

// One row of this thread's 8 channels: k or q (bf16), g as (hi, lo); rows past the
// chunk's end give zero k and q and the last row's g.
struct Row8 {
    float k[8], q[8], gh[8], gl[8];
};

__device__ __forceinline__ void load_row8(Row8& R, const __nv_bfloat16* k, const __nv_bfloat16* q, const float* g,
                                          const float* gl, int tok0, int len, int r, int H, int h, int c8,
                                          bool want_q) {
    const int rr = r < len ? r : len - 1;
    const size_t off = toff(tok0 + rr, H, h) + c8;
    load8f(g + off, R.gh);
    load8f(gl + off, R.gl);
    if (r < len) {
        bf16x8_to_f32(*reinterpret_cast<const uint4*>(k + off), R.k);
        if (want_q) bf16x8_to_f32(*reinterpret_cast<const uint4*>(q + off), R.q);
    } else {
#pragma unroll
        for (int u = 0; u < 8; ++u) R.k[u] = R.q[u] = 0.f;
    }
}

// One row of 8 channels for the elementwise epilogue (rows past the end: the last row's g,
// everything else zero).
struct E2Row {
    float gh[8], gl[8], dqg[8], dkg[8], dkd[8];
    uint4 k, q, la;
};

__device__ __forceinline__ void load_e2row(E2Row& R, const __nv_bfloat16* k, const __nv_bfloat16* q,
                                           const __nv_bfloat16* la, const float* g, const float* gl,
                                           const float* dQg, const float* dKg, const float* dKd, int tok0, int len,
                                           int r, int H, int h, int c8) {
    const bool live = r < len;
    const size_t off = toff(tok0 + (live ? r : len - 1), H, h) + c8;
    load8f(g + off, R.gh);
    load8f(gl + off, R.gl);
    if (live) {
        R.k = *reinterpret_cast<const uint4*>(k + off);
        R.q = *reinterpret_cast<const uint4*>(q + off);
        R.la = *reinterpret_cast<const uint4*>(la + off);
        load8f(dQg + off, R.dqg);
        load8f(dKg + off, R.dkg);
        load8f(dKd + off, R.dkd);
    } else {
        R.k = R.q = R.la = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int u = 0; u < 8; ++u) R.dqg[u] = R.dkg[u] = R.dkd[u] = 0.f;
    }
}

__device__ __forceinline__ uint4 pack8_bf16(const float* x) {
    return make_uint4(pack_bf16(x[0], x[1]), pack_bf16(x[2], x[3]), pack_bf16(x[4], x[5]), pack_bf16(x[6], x[7]));
}

__global__ void __launch_bounds__(kQT, 1)
kb_c_tc(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
        const __nv_bfloat16* __restrict__ la, const float* __restrict__ g, const float* __restrict__ gl,
        const float* __restrict__ dAt, const float* __restrict__ dP, const float* __restrict__ dQg,
        const float* __restrict__ dKd, const float* __restrict__ dKg, const float* __restrict__ dGam,
        __nv_bfloat16* __restrict__ dq_out, __nv_bfloat16* __restrict__ dk_out, __nv_bfloat16* __restrict__ dla_out,
        int* __restrict__ err, ChunkMap cmap, int H) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // no static shared memory: the dynamic region starts at the CTA's shared window
    if (smem_u32(smem_raw) & 1023u) {
        if (threadIdx.x == 0) atomicCAS(err, 0, (int)KDA_ERR_DEVICE);
        return;
    }
    uint8_t* sm = smem_raw;
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + kBarOff);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(sm + kBarOff + 16);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    int seq, tok0, len, idx;
    cmap.locate((int)blockIdx.x, seq, tok0, len, idx);
    const int h = (int)blockIdx.y;
    const size_t unit = (size_t)blockIdx.x * H + h;
    const size_t pbase = unit * kQC * kQC;

    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        mbar_init_fence();
    }
    if (warp == 0) {
        tmem_alloc(tslot, kQTmemCols);
        tmem_relinquish();
    }

    // Every global load of a phase is issued before the phase's first wait, and the
    // next phase's loads before the previous product's wait: with one CTA per SM the
    // round trips to memory are what the kernel's time is made of otherwise.
    // ---- this thread's 8 channels, its rows r0 + 16 j, and the block references ----
    const int c8 = (tid & 15) * 8, r0 = tid >> 4;
    float ref[4][8];   // g at rows 15, 31, 47, 63 (hi part; any consistent reference serves)
#pragma unroll
    for (int j = 0; j < 4; ++j) load8f(g + toff(tok0 + min(16 * j + 15, len - 1), H, h) + c8, ref[j]);
    float sa[2][8] = {}, sq[2][8] = {};   // dAt and dP rows for the staging
#pragma unroll
    for (int it = 0; it < 2; ++it) {
        const int qi = tid + kQT * it, r = qi >> 3, i8 = (qi & 7) * 8;
        if (r < len) {
            load8f(dAt + pbase + (size_t)r * kQC + i8, sa[it]);
            load8f(dP + pbase + (size_t)r * kQC + i8, sq[it]);
        }
    }
    Row8 R[4];   // k, g of this thread's rows: kept for all three version builds
#pragma unroll
    for (int j = 0; j < 4; ++j) load_row8(R[j], k, q, g, gl, tok0, len, r0 + 16 * j, H, h, c8, false);
    const int sp = warp & 3, half = warp >> 2, c = 32 * sp + lane;   // the epilogue's channel and rows
    // bit b: diagonal block b is summed pairwise.  A warp's 32 threads hold all 128
    // channels of the references, so a warp-wide OR gives every warp the CTA's flags.
    unsigned flags = 0;
#pragma unroll
    for (int I = 0; I < 4; ++I) {
        float rg = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) rg = fmaxf(rg, (I > 0 ? ref[I - 1][u] : 0.f) - ref[I][u]);
        if (rg > kRangeMax) flags |= 1u << I;
    }
    flags = __reduce_or_sync(0xffffffffu, flags);

    // ---- dAt (i < r) and dP (i < r): fp32 staging and the [dAt ; dP] image ----
    float* stA = reinterpret_cast<float*>(sm + kV1);
    float* stP = stA + kQC * kQC;
#pragma unroll
    for (int it = 0; it < 2; ++it) {
        const int qi = tid + kQT * it, r = qi >> 3, i8 = (qi & 7) * 8;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const bool live = r < len && i8 + u < r;
            sa[it][u] = live ? sa[it][u] : 0.f;
            sq[it][u] = live ? sq[it][u] : 0.f;
        }
        *reinterpret_cast<float4*>(stA + r * kQC + i8) = make_float4(sa[it][0], sa[it][1], sa[it][2], sa[it][3]);
        *reinterpret_cast<float4*>(stA + r * kQC + i8 + 4) = make_float4(sa[it][4], sa[it][5], sa[it][6], sa[it][7]);
        *reinterpret_cast<float4*>(stP + r * kQC + i8) = make_float4(sq[it][0], sq[it][1], sq[it][2], sq[it][3]);
        *reinterpret_cast<float4*>(stP + r * kQC + i8 + 4) = make_float4(sq[it][4], sq[it][5], sq[it][6], sq[it][7]);
        const int I = r >> 4, x = r & 15;
        store8_split(sm + kImX, sm + kImX + kImXLo, sw128_chunk(32 * I + x, i8, 128), sa[it]);
        store8_split(sm + kImX, sm + kImX + kImXLo, sw128_chunk(32 * I + 16 + x, i8, 128), sq[it]);
    }
    // ---- key versions: KV_I[i] = k_i e^{gb_I - g_i} for keys i < 16 (I + 1) ----
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int r = r0 + 16 * j;
#pragma unroll
        for (int I = j; I < 4; ++I) {
            float x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                x[u] = (I == j && ((flags >> j) & 1u))
                           ? 0.f
                           : R[j].k[u] * exp_gdiff(I > 0 ? ref[I - 1][u] : 0.f, 0.f, R[j].gh[u], R[j].gl[u]);
            store8_split(sm + kV0 + kv_off(I), sm + kV0 + kVLo + kv_off(I), mn_chunk(r, c8, 16 * (I + 1)), x);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;
    const uint32_t v0 = smem_u32(sm + kV0), v1 = smem_u32(sm + kV1);
    const uint32_t imx = smem_u32(sm + kImX), imat = smem_u32(sm + kImAT), impt = smem_u32(sm + kImPT);

    // X: D[c][32 I + n] = sum_i KV_I[i][c] [dAt ; dP]_{block I row n, i}
    if (tid == 0) {
#pragma unroll
        for (int I = 0; I < 4; ++I) {
            const uint32_t ah = v0 + kv_off(I), al = ah + kVLo;
            const int K = 16 * (I + 1);
            for (int s = 0; s <= I; ++s) {
                const uint64_t adh = mn_desc_k(ah, K, s), adl = mn_desc_k(al, K, s);
                const uint64_t bdh = sw128_desc(imx + 4096u * I + 32u * s);
                const uint64_t bdl = sw128_desc(imx + kImXLo + 4096u * I + 32u * s);
                const uint32_t id = idesc_amn(128, 32);
                mma_bf16(tbase + 32 * I, adh, bdh, id, s > 0 ? 1u : 0u);
                mma_bf16(tbase + 32 * I, adh, bdl, id, 1u);
                mma_bf16(tbase + 32 * I, adl, bdh, id, 1u);
            }
        }
        mma_commit(&bar[0]);
    }
    // q of this thread's rows, for the row versions of q: kept packed, so that nothing waits
    // for it before those are built
    uint4 qp[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int r = r0 + 16 * j;
        qp[j] = r < len ? *reinterpret_cast<const uint4*>(q + toff(tok0 + r, H, h) + c8) : make_uint4(0u, 0u, 0u, 0u);
    }
    // ---- dAt^T and dP^T images (rows = keys i, K = rows r) from the staging, by warps 1-7
    // (warp 0 issues the products) ----
    for (int qi = tid - 32; qi >= 0 && qi < 512; qi += kQT - 32) {
        const int i = qi & 63, r8 = (qi >> 6) * 8;
        float a[8], p[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            a[u] = stA[(r8 + u) * kQC + i];
            p[u] = stP[(r8 + u) * kQC + i];
        }
        store8_split(sm + kImAT, sm + kImAT + kImTLo, sw128_chunk(i, r8, 64), a);
        store8_split(sm + kImPT, sm + kImPT + kImTLo, sw128_chunk(i, r8, 64), p);
    }
    __syncthreads();   // the staging is read; its buffer takes the row versions of k
    // ---- row versions of k: RV_J[r] = k_r e^{g_r - ge_J} for rows r >= 16 J ----
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int r = r0 + 16 * j;
#pragma unroll
        for (int J = 0; J <= j; ++J) {
            float x[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                x[u] = (J == j && ((flags >> j) & 1u)) ? 0.f
                                                         : R[j].k[u] * exp_gdiff(R[j].gh[u], R[j].gl[u], ref[J][u], 0.f);
            store8_split(sm + kV1 + rv_off(J), sm + kV1 + kVLo + rv_off(J), mn_chunk(r - 16 * J, c8, 64 - 16 * J), x);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // Y (k part): D[c][128 + 16 J + n] = sum_{r >= 16 J} RV_J[r][c] dAt[r][16 J + n]
    if (tid == 0) {
#pragma unroll
        for (int J = 0; J < 4; ++J) {
            const uint32_t ah = v1 + rv_off(J), al = ah + kVLo;
            const int K = 64 - 16 * J;
            for (int s = J; s < 4; ++s) {
                const uint64_t adh = mn_desc_k(ah, K, s - J), adl = mn_desc_k(al, K, s - J);
                const uint64_t bdh = sw128_desc(imat + 2048u * J + 32u * s);
                const uint64_t bdl = sw128_desc(imat + kImTLo + 2048u * J + 32u * s);
                const uint32_t id = idesc_amn(128, 16);
                mma_bf16(tbase + 128 + 16 * J, adh, bdh, id, s > J ? 1u : 0u);
                mma_bf16(tbase + 128 + 16 * J, adh, bdl, id, 1u);
                mma_bf16(tbase + 128 + 16 * J, adl, bdh, id, 1u);
            }
        }
    }
    // the key versions are free once X is done
    bool ok = __syncthreads_and(mbar_wait(&bar[0], 0) ? 1 : 0) != 0;
    float dgv[8];
    if (ok) {
        // ---- row versions of q into the first buffer ----
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int r = r0 + 16 * j;
            float qv[8];
            bf16x8_to_f32(qp[j], qv);
#pragma unroll
            for (int J = 0; J <= j; ++J) {
                float x[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    x[u] = (J == j && ((flags >> j) & 1u))
                               ? 0.f
                               : qv[u] * exp_gdiff(R[j].gh[u], R[j].gl[u], ref[J][u], 0.f);
                store8_split(sm + kV0 + rv_off(J), sm + kV0 + kVLo + rv_off(J), mn_chunk(r - 16 * J, c8, 64 - 16 * J),
                             x);
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // Y (q part), accumulated onto the k part
        if (tid == 0) {
#pragma unroll
            for (int J = 0; J < 4; ++J) {
                const uint32_t ah = v0 + rv_off(J), al = ah + kVLo;
                const int K = 64 - 16 * J;
                for (int s = J; s < 4; ++s) {
                    const uint64_t adh = mn_desc_k(ah, K, s - J), adl = mn_desc_k(al, K, s - J);
                    const uint64_t bdh = sw128_desc(impt + 2048u * J + 32u * s);
                    const uint64_t bdl = sw128_desc(impt + kImTLo + 2048u * J + 32u * s);
                    const uint32_t id = idesc_amn(128, 16);
                    mma_bf16(tbase + 128 + 16 * J, adh, bdh, id, 1u);
                    mma_bf16(tbase + 128 + 16 * J, adh, bdl, id, 1u);
                    mma_bf16(tbase + 128 + 16 * J, adl, bdh, id, 1u);
                }
            }
            mma_commit(&bar[1]);
        }
        // in flight while the last product runs: the diagonal blocks of dAt and dP (element
        // e = tid + 256 it: dAt at 2 it, dP at 2 it + 1)
#pragma unroll
        for (int it = 0; it < 4; ++it) {
            const int e = tid + kQT * it, bk = e >> 8, x = (e >> 4) & 15, y = e & 15, r = 16 * bk + x;
            const bool live = r < len;
            const size_t o = pbase + (size_t)r * kQC + 16 * bk + y;
            dgv[2 * it] = (live && y < x) ? dAt[o] : 0.f;
            dgv[2 * it + 1] = (live && y <= x) ? dP[o] : 0.f;
        }
        ok = __syncthreads_and(mbar_wait(&bar[1], 0) ? 1 : 0) != 0;
    }
    if (!ok) {
        if (tid == 0) {
            atomicCAS(err, 0, (int)KDA_ERR_TIMEOUT);
            // a wait gave up: let the products drain before the tensor memory is freed
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < 100000000ull) {
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == 0) tmem_dealloc(tbase, kQTmemCols);
        return;
    }
    tc_fence_after();

    // ---- epilogue ----
    float* Xs1 = reinterpret_cast<float*>(sm + kEX1);   // [64][128] X1, X2, Y: scaled for flagged blocks, raw otherwise
    float* Xs2 = reinterpret_cast<float*>(sm + kEX2);
    float* Ys = reinterpret_cast<float*>(sm + kEY);
    float* dg = reinterpret_cast<float*>(sm + kEDiag);  // diagonal blocks: dAt [b][16][16] at 512 b, dP at 512 b + 256
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int e = tid + kQT * it, bk = e >> 8, xy = e & 255;
        dg[512 * bk + xy] = dgv[2 * it];
        dg[512 * bk + 256 + xy] = dgv[2 * it + 1];
    }
    __syncthreads();
    // E1: the owner of channel c (rows 32 half ..) moves X1, X2, Y out of tensor memory; a
    // flagged block is scaled here and gets its exact pairs
#pragma unroll 1
    for (int bb = 0; bb < 2; ++bb) {
        const int b = 2 * half + bb;
        float X1[16], X2[16], Y[16];
        tmem_ld16(tmem_addr(tbase, 32 * sp, 32 * b), X1);
        tmem_ld16(tmem_addr(tbase, 32 * sp, 32 * b + 16), X2);
        tmem_ld16(tmem_addr(tbase, 32 * sp, 128 + 16 * b), Y);
        tmem_ld_wait();
        if ((flags >> b) & 1u) {
            float kx[16], qx[16], gh[16], glo[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                const int r = 16 * b + x;
                const bool live = r < len;
                const size_t off = toff(tok0 + (live ? r : len - 1), H, h) + c;
                gh[x] = g[off];
                glo[x] = gl[off];
                kx[x] = live ? __bfloat162float(k[off]) : 0.f;
                qx[x] = live ? __bfloat162float(q[off]) : 0.f;
            }
            // the references the versions were built with (g at rows 16 b - 1 and 16 b + 15)
            const float gb = b > 0 ? g[toff(tok0 + min(16 * b - 1, len - 1), H, h) + c] : 0.f;
            const float ge = g[toff(tok0 + min(16 * b + 15, len - 1), H, h) + c];
#pragma unroll
            for (int x = 0; x < 16; ++x) {
                const float sr = exp_gdiff(gh[x], glo[x], gb, 0.f);
                X1[x] *= sr;
                X2[x] *= sr;
                Y[x] *= exp_gdiff(ge, 0.f, gh[x], glo[x]);
            }
            // the block's pairs, exactly: every factor exp of a non-positive difference
            const float* da = dg + 512 * b;
            const float* dp = da + 256;
#pragma unroll
            for (int x = 1; x < 16; ++x)
#pragma unroll
                for (int y = 0; y < x; ++y) {
                    const float e = exp_gdiff(gh[x], glo[x], gh[y], glo[y]);
                    const float a = da[16 * x + y], p = dp[16 * x + y];
                    const float ke = kx[y] * e;
                    X1[x] = fmaf(a, ke, X1[x]);
                    X2[x] = fmaf(p, ke, X2[x]);
                    Y[y] = fmaf(fmaf(a, kx[x], p * qx[x]), e, Y[y]);
                }
        }
#pragma unroll
        for (int x = 0; x < 16; ++x) {
            const int r = 16 * b + x;
            Xs1[r * kQD + c] = X1[x];
            Xs2[r * kQD + c] = X2[x];
            Ys[r * kQD + c] = Y[x];
        }
    }
    __syncthreads();
    // E2: warp w takes rows 8 w .. 8 w + 7; lane (8 channels c2 = 8 (lane & 15), row group
    // gi = 2 w + lane / 16 = rows 4 gi .. 4 gi + 3), so that a load covers two whole rows.  The
    // elementwise terms, dq and dk; the row groups' sums go through a small table for the scans.
    float* Tdq = reinterpret_cast<float*>(sm + kETab);          // [16][128]: sum over the group of DQ_r
    float* Tp = Tdq + 16 * kQD;                                  // [16][128]: sum over the group of P_r
    {
        const int gi = 2 * warp + (lane >> 4), c2 = 8 * (lane & 15), b = gi >> 2;
        float gC8[8], gCl8[8], gb8[8] = {}, ge8[8];
        load8f(g + toff(tok0 + len - 1, H, h) + c2, gC8);
        load8f(gl + toff(tok0 + len - 1, H, h) + c2, gCl8);
        if (b > 0) load8f(g + toff(tok0 + min(16 * b - 1, len - 1), H, h) + c2, gb8);
        load8f(g + toff(tok0 + min(16 * b + 15, len - 1), H, h) + c2, ge8);
        const bool raw = !((flags >> b) & 1u);
        float dqv[4][8], pv[4][8];   // per row: D_r + dQg Qg + dKg Kg, and dKd Kd
        unsigned lok = 0;            // bit 8 x + u: row 4 gi + x exists, log alpha above the floor
        E2Row e2a, e2b;
        load_e2row(e2a, k, q, la, g, gl, dQg, dKg, dKd, tok0, len, 4 * gi, H, h, c2);
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            // one row ahead: row x + 1's loads are in flight while row x is worked on
            E2Row& cur = (x & 1) ? e2b : e2a;
            E2Row& nxt = (x & 1) ? e2a : e2b;
            if (x < 3) load_e2row(nxt, k, q, la, g, gl, dQg, dKg, dKd, tok0, len, 4 * gi + x + 1, H, h, c2);
            const int r = 4 * gi + x;
            const bool live = r < len;
            float kx[8], qx[8], lav[8], x1[8], x2[8], y[8];
            bf16x8_to_f32(cur.k, kx);
            bf16x8_to_f32(cur.q, qx);
            bf16x8_to_f32(cur.la, lav);
            load8f(Xs1 + r * kQD + c2, x1);
            load8f(Xs2 + r * kQD + c2, x2);
            load8f(Ys + r * kQD + c2, y);
            const float dpd = dg[512 * b + 256 + 17 * (r & 15)];
            float dq8[8], dk8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                if (raw) {
                    const float sr = exp_gdiff(cur.gh[u], cur.gl[u], gb8[u], 0.f);
                    x1[u] *= sr;
                    x2[u] *= sr;
                    y[u] *= exp_gdiff(ge8[u], 0.f, cur.gh[u], cur.gl[u]);
                }
                const float eg = exp_g(cur.gh[u], cur.gl[u]);
                const float ed = exp_gdiff(gC8[u], gCl8[u], cur.gh[u], cur.gl[u]);
                dq8[u] = fmaf(dpd, kx[u], x2[u]) + cur.dqg[u] * eg;
                dk8[u] = (x1[u] + fmaf(dpd, qx[u], y[u])) + fmaf(cur.dkg[u], eg, cur.dkd[u] * ed);
                // rows past the end have k = q = 0 and zero gradients: both terms vanish
                const float D = fmaf(kx[u], x1[u] - y[u], qx[u] * x2[u]);
                dqv[x][u] = D + fmaf(cur.dqg[u], qx[u], cur.dkg[u] * kx[u]) * eg;
                pv[x][u] = cur.dkd[u] * kx[u] * ed;
                if (live && lav[u] >= kLogAlphaFloor) lok |= 1u << (8 * x + u);
            }
            if (live) {
                *reinterpret_cast<uint4*>(dq_out + toff(tok0 + r, H, h) + c2) = pack8_bf16(dq8);
                *reinterpret_cast<uint4*>(dk_out + toff(tok0 + r, H, h) + c2) = pack8_bf16(dk8);
            }
        }
        float td[8], tp[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            td[u] = (dqv[0][u] + dqv[1][u]) + (dqv[2][u] + dqv[3][u]);
            tp[u] = (pv[0][u] + pv[1][u]) + (pv[2][u] + pv[3][u]);
        }
        *reinterpret_cast<float4*>(Tdq + gi * kQD + c2) = make_float4(td[0], td[1], td[2], td[3]);
        *reinterpret_cast<float4*>(Tdq + gi * kQD + c2 + 4) = make_float4(td[4], td[5], td[6], td[7]);
        *reinterpret_cast<float4*>(Tp + gi * kQD + c2) = make_float4(tp[0], tp[1], tp[2], tp[3]);
        *reinterpret_cast<float4*>(Tp + gi * kQD + c2 + 4) = make_float4(tp[4], tp[5], tp[6], tp[7]);
        __syncthreads();
        // the table in place: thread (channel, which) turns its 16 group sums into the sums over
        // the groups after (DQ) or before (P) each one
        {
            const int cc = tid & (kQD - 1);
            float* col = (tid < kQD ? Tdq : Tp) + cc;
            float v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = col[i * kQD];
            float acc = 0.f;
            if (tid < kQD) {
#pragma unroll
                for (int i = 15; i >= 0; --i) {
                    const float t = v[i];
                    v[i] = acc;
                    acc += t;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float t = v[i];
                    v[i] = acc;
                    acc += t;
                }
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) col[i * kQD] = v[i];
        }
        __syncthreads();
        float suf[8], pre[8], dgm[8];
        load8f(Tdq + gi * kQD + c2, suf);
        load8f(Tp + gi * kQD + c2, pre);
        load8f(dGam + unit * kQD + c2, dgm);
        float F[4][8];
#pragma unroll
        for (int x = 3; x >= 0; --x)
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                suf[u] += dqv[x][u];
                F[x][u] = suf[u];
            }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int r = 4 * gi + x;
            float o[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                o[u] = ((lok >> (8 * x + u)) & 1u) ? F[x][u] + pre[u] + dgm[u] * exp_g(gC8[u], gCl8[u]) : 0.f;
                pre[u] += pv[x][u];
            }
            if (r < len) *reinterpret_cast<uint4*>(dla_out + toff(tok0 + r, H, h) + c2) = pack8_bf16(o);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, kQTmemCols);
}

}  // namespace

cudaError_t launch_kb_c_tc(const void* q, const void* k, const void* la, const float* g, const float* gl,
                           const float* dAt, const float* dP, const float* dQg, const float* dKd, const float* dKg,
                           const float* dGam, void* dq, void* dk, void* dla, int* err, const ChunkMap& cmap,
                           int n_chunks, int H, cudaStream_t stream) {
    if (n_chunks == 0) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(kb_c_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kQSmem);
    if (e != cudaSuccess) return e;
    using bf = __nv_bfloat16;
    kb_c_tc<<<dim3(n_chunks, H), kQT, kQSmem, stream>>>(
        (const bf*)q, (const bf*)k, (const bf*)la, g, gl, dAt, dP, dQg, dKd, dKg, dGam, (bf*)dq, (bf*)dk, (bf*)dla, err,
        cmap, H);
    return cudaGetLastError();
}

}  // namespace kda
