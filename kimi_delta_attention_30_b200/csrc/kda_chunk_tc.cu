// Tensor-core (tcgen05) chunkwise KDA prefill: bf16 inputs, d_k = d_v = 128,
// chunk C = 64, fp32 state and accumulation.
//
// Two kernels:
//
//   tc_intra  (one CTA per (chunk, head), all chunks in parallel)
//     cumulative log decay g (row a1), then on the tensor cores the
//     decay-weighted strictly-lower A = Diag(beta) (K K^T . exp(g_r - g_i)) and
//     the inclusive score matrix P = (Q K^T . exp(g_r - g_i)); T = (I + A)^{-1}
//     by blocked forward substitution on CUDA cores; then (tensor cores)
//       U  = T Diag(beta) V,        Wk = T Diag(beta) (K . exp(g))       (row a2)
//       U' = P U,                   Q' = Q . exp(g) - P Wk
//       Kd = K . exp(g_C - g),      Gamma_C = exp(g_C)
//     written to the workspace in the exact shared-memory layout the second
//     kernel's MMAs consume (so its loads are plain 1-D bulk copies).
//
//   tc_recur  (one CTA per (sequence, head, d_v tile), sequential over chunks)
//     with the fp32 state tile S (d_k x BV) in TMEM:
//       D   = [Wk ; Q'] S                         M = 128 MMA
//       W   = U - D[0:64]                         per-token corrections
//       O   = D[64:128] + U'                      outputs (row a4)
//       S  <- Diag(Gamma_C) S + Kd^T W            M = 128 MMA accumulating in TMEM (row a3)
//     The next chunk's operands stream in by bulk copies (TMA engine, no
//     multicast) while the current chunk is processed.
//
// Derivation (ours; the oracle's chunk form checks it against the token
// recurrence): with Gamma_r = exp(g_r) the per-token corrections W solve
// (I + A) W = Diag(beta)(V - (K . Gamma) S_0), so W = U - Wk S_0; the outputs
// are O = (Q . Gamma) S_0 + P W = Q' S_0 + U'; the next state is
// Diag(Gamma_C) S_0 + Kd^T W.  Chunkwise form: "From GPT-2 to Kimi K3" essay
// (pwwt.cn/news/3716252), chunkwise and Gated DeltaNet paragraphs; WY / DPLR
// restructuring: "我终于看懂了 KDA" explainer (pwwt.cn/news/3787313),
// sections 16-17.
//
// Precision.  Every tensor-core product is formed in three bf16 terms,
// a_hi b_hi + a_hi b_lo + a_lo b_hi (hi = RN_bf16(x), lo = RN_bf16(x - hi)),
// with fp32 accumulation: about 16 significant bits per operand.  Heavy decay
// makes single tokens dominate many of the sums, so a single bf16 rounding of
// an operand would show up at ~2^-9 times the (heavy) tail of o; three terms
// keep the whole path within the fp32 regime.  U and U' are kept in fp32.
//
// Decay factors.  Rows form 16-row blocks; gb[b] is g at the row before block
// b (gb[0] = 0), gb[4] = g_C.  Every factor handed to the tensor cores is exp of
// a non-positive difference, except exp(gb[I] - gb[I+1]) (<= exp(decay range
// of block I)) on the diagonal blocks; a block whose range exceeds kDiagRange
// nats has its diagonal A / P entries recomputed pairwise on CUDA cores.
#include "kda_internal.cuh"
#include "kda_tc.cuh"

namespace kda {

extern const char* const kTcKernelNames[] = {"tc_intra", "tc_recur"};
extern const int kTcKernelCount = 2;

namespace {

using namespace tc;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr float kDiagRange = 80.0f;

// ---- workspace image of one (chunk, head) --------------------------------------
constexpr uint32_t kOffWkQh = 0;         // [128 rows][128 k] bf16 SW128: rows 0-63 Wk, 64-127 Q' (hi)
constexpr uint32_t kOffWkQl = 32768;     // lo parts
constexpr uint32_t kOffKdTh = 65536;     // [128 rows (channel)][64 k (token)] bf16 SW128 (hi)
constexpr uint32_t kOffKdTl = 81920;     // lo parts
constexpr uint32_t kOffU = 98304;        // U : [4 column blocks][64 rows][32] fp32
constexpr uint32_t kOffU2 = 131072;      // U': same layout
constexpr uint32_t kOffGam = 163840;     // Gamma_C fp32 [128]
constexpr uint32_t kChunkBytes = 164352;
constexpr uint32_t kErrHeader = 256;     // first bytes of the TC scratch: error word

// ---- tc_intra shared memory (byte offsets from a 1024-aligned base) -----------
constexpr int kIntraThreads = 256;
// phase 1: MMA-1 operands
constexpr uint32_t kAKQh = 0;            // [K.E ; Q.E]  128 x 128
constexpr uint32_t kAKQl = 32768;
constexpr uint32_t kKFh = 65536;         // decayed key versions 160 x 128
constexpr uint32_t kKFl = 106496;
constexpr uint32_t kXVh = 147456;        // (beta V)^T 128 x 64
constexpr uint32_t kXVl = 163840;
// phase 2 (after MMA 1, inside [0, 147456))
constexpr uint32_t kXKh = 0;             // (beta K exp(g))^T 128 x 64
constexpr uint32_t kXKl = 16384;
constexpr uint32_t kAs = 32768;          // A fp32 [64][64]
constexpr uint32_t kPh = 49152;          // P 64 x 64
constexpr uint32_t kPl = 57344;
constexpr uint32_t kTs = 65536;          // T fp32 [64][64]
constexpr uint32_t kScr = 81920;         // 8 KB scratch
constexpr uint32_t kTh = 90112;          // T 64 x 64
constexpr uint32_t kTl = 98304;
// phase 3 (after MMA 2): U^T and Wk^T operands in the dead X regions
constexpr uint32_t kUTh = 0, kUTl = 16384, kWTh = kXVh, kWTl = kXVl;
constexpr uint32_t kTab = 180224;        // tables
constexpr int kNumTab = 18;              // tau[4], sigma[6], exp(gb)[4], exp(g_C - gb[b+1])[4]
constexpr uint32_t kIntraSmem = kTab + kNumTab * 128 * 4 + 5 * 128 * 4 + 64 * 4 + 64;
constexpr uint32_t kIntraAlloc = kIntraSmem + 1024;

// rows of the decayed-key versions: version R covers keys [0, 16 R + 16)
__device__ __forceinline__ int kf_off(int R) { return (R * (R + 1)) * 8; }   // 0, 16, 48, 96

__device__ __forceinline__ int tab_tau(int R) { return R; }                                  // exp(gb[R] - gb[R+1])
__device__ __forceinline__ int tab_sigma(int R, int I) { return 4 + (R * (R - 1)) / 2 + I; } // exp(gb[R] - gb[I+1]), I < R
__device__ __forceinline__ int tab_e0(int I) { return 10 + I; }                              // exp(gb[I])
__device__ __forceinline__ int tab_ec(int I) { return 14 + I; }                              // exp(g_C - gb[I+1])

__device__ __forceinline__ void unpack4(uint2 v, float (&f)[4]) {
    f[0] = bf16_lo(v.x);
    f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y);
    f[3] = bf16_hi(v.y);
}

// four consecutive k values of one row, split into the hi and lo tiles
__device__ __forceinline__ void store4_split(uint8_t* hi_tile, uint8_t* lo_tile, uint32_t off, float a, float b,
                                             float c, float d) {
    uint2 hv, lv;
    split2(a, b, hv.x, lv.x);
    split2(c, d, hv.y, lv.y);
    *reinterpret_cast<uint2*>(hi_tile + off) = hv;
    *reinterpret_cast<uint2*>(lo_tile + off) = lv;
}

__device__ __forceinline__ void store1_split(uint8_t* hi_tile, uint8_t* lo_tile, uint32_t off, float x) {
    __nv_bfloat16 hv, lv;
    split1(x, hv, lv);
    *reinterpret_cast<__nv_bfloat16*>(hi_tile + off) = hv;
    *reinterpret_cast<__nv_bfloat16*>(lo_tile + off) = lv;
}

// eight consecutive k values (one 16-byte chunk) split into hi and lo tiles
__device__ __forceinline__ void store8_split(uint8_t* hi_tile, uint8_t* lo_tile, uint32_t off, const float* x) {
    uint4 hv, lv;
    split2(x[0], x[1], hv.x, lv.x);
    split2(x[2], x[3], hv.y, lv.y);
    split2(x[4], x[5], hv.z, lv.z);
    split2(x[6], x[7], hv.w, lv.w);
    *reinterpret_cast<uint4*>(hi_tile + off) = hv;
    *reinterpret_cast<uint4*>(lo_tile + off) = lv;
}

__device__ __forceinline__ void record_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// D (+)= A B^T in three bf16 terms over `ksteps` K-slices of 16.
__device__ __forceinline__ void mma3(uint32_t d, uint32_t ah, uint32_t al, int arows, uint32_t bh, uint32_t bl,
                                     int brows, int ksteps, uint32_t idesc, bool accumulate) {
    for (int s = 0; s < ksteps; ++s) {
        const uint32_t acc0 = (accumulate || s > 0) ? 1u : 0u;
        mma_bf16(d, sw128_desc_k(ah, arows, s), sw128_desc_k(bh, brows, s), idesc, acc0);
        mma_bf16(d, sw128_desc_k(ah, arows, s), sw128_desc_k(bl, brows, s), idesc, 1u);
        mma_bf16(d, sw128_desc_k(al, arows, s), sw128_desc_k(bh, brows, s), idesc, 1u);
    }
}

// ============================================================================
// tc_intra
// ============================================================================
__global__ void __launch_bounds__(kIntraThreads, 1)
tc_intra(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
         const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ la,
         const __nv_bfloat16* __restrict__ beta, uint8_t* __restrict__ ws, int* __restrict__ err, ChunkMap cmap,
         int H) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float* tab = reinterpret_cast<float*>(sm + kTab);                 // [18][128]
    float* gb = tab + kNumTab * 128;                                  // [5][128]
    float* sbeta = gb + 5 * 128;                                      // [64]
    uint32_t* sflags = reinterpret_cast<uint32_t*>(sbeta + 64);       // [0] fallback mask, [1] abort, [2] tmem base
    __shared__ uint64_t mbar;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int c0 = 4 * lane, r0 = 8 * warp;    // this thread: channels [c0, c0+4), rows [r0, r0+8)
    const int I = warp >> 1;                   // 16-row block of this thread's rows
    int seq, tok0, len, cidx;
    cmap.locate(blockIdx.x, seq, tok0, len, cidx);
    const int h = blockIdx.y;
    uint8_t* out = ws + (size_t)((size_t)blockIdx.x * H + h) * kChunkBytes;

    if (tid == 0) {
        sflags[0] = 0;
        sflags[1] = 0;
        mbar_init(&mbar, 1);
        mbar_init_fence();
    }
    if (warp == 0) {
        tmem_alloc(&sflags[2], 256);
        tmem_relinquish();
    }
    if (tid < 64) sbeta[tid] = (tid < len) ? __bfloat162float(beta[(size_t)(tok0 + tid) * H + h]) : 0.f;

    // ---- this thread's 8 rows x 4 channels of k, q, v, log alpha ----------
    uint2 kr[8], qr[8], vr[8];
    float g[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int r = r0 + j;
        if (r < len) {
            const size_t off = ((size_t)(tok0 + r) * H + h) * kD + c0;
            kr[j] = *reinterpret_cast<const uint2*>(k + off);
            qr[j] = *reinterpret_cast<const uint2*>(q + off);
            vr[j] = *reinterpret_cast<const uint2*>(v + off);
            float a[4];
            unpack4(*reinterpret_cast<const uint2*>(la + off), a);
#pragma unroll
            for (int x = 0; x < 4; ++x) g[j][x] = fmaxf(a[x], kLogAlphaFloor);
        } else {
            kr[j] = make_uint2(0, 0);
            qr[j] = kr[j];
            vr[j] = kr[j];
#pragma unroll
            for (int x = 0; x < 4; ++x) g[j][x] = 0.f;
        }
    }
    // ---- cumulative log decay (row a1): local prefix, then carries --------
#pragma unroll
    for (int j = 1; j < 8; ++j)
#pragma unroll
        for (int x = 0; x < 4; ++x) g[j][x] += g[j - 1][x];
    float* tot = tab;   // [8][128] partial totals (the table space is free until the tables are built)
#pragma unroll
    for (int x = 0; x < 4; ++x) tot[warp * 128 + c0 + x] = g[7][x];
    __syncthreads();
    {
        float carry[4] = {0.f, 0.f, 0.f, 0.f};
        for (int p = 0; p < warp; ++p)
#pragma unroll
            for (int x = 0; x < 4; ++x) carry[x] += tot[p * 128 + c0 + x];
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int x = 0; x < 4; ++x) g[j][x] += carry[x];
    }
    if (tid < 128) gb[tid] = 0.f;
    if (warp & 1) {
#pragma unroll
        for (int x = 0; x < 4; ++x) gb[(I + 1) * 128 + c0 + x] = g[7][x];
    }
    __syncthreads();

    // ---- factor tables and the per-block range check -----------------------
    if (tid < 128) {
        const int c = tid;
        float gbv[5];
#pragma unroll
        for (int b = 0; b < 5; ++b) gbv[b] = gb[b * 128 + c];
        uint32_t fb = 0;
#pragma unroll
        for (int R = 0; R < 4; ++R) {
            const float range = gbv[R] - gbv[R + 1];
            if (range > kDiagRange) fb |= 1u << R;
            tab[tab_tau(R) * 128 + c] = __expf(fminf(range, kDiagRange));
#pragma unroll
            for (int J = 0; J < R; ++J) tab[tab_sigma(R, J) * 128 + c] = __expf(gbv[R] - gbv[J + 1]);
            tab[tab_e0(R) * 128 + c] = __expf(gbv[R]);
            tab[tab_ec(R) * 128 + c] = __expf(gbv[4] - gbv[R + 1]);
        }
        if (fb) atomicOr(&sflags[0], fb);
    }
    __syncthreads();
    const uint32_t fbmask = sflags[0];
    if (tid < 128) {
        // a block recomputed pairwise contributes nothing through the MMA
#pragma unroll
        for (int R = 0; R < 4; ++R)
            if (fbmask & (1u << R)) tab[tab_tau(R) * 128 + tid] = 0.f;
    }
    __syncthreads();

    // ---- MMA-1 operands, Q exp(g) and Kd into the workspace, (beta V)^T ------
    {
        float e0[4], ec[4], gref[4], glast[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            e0[x] = tab[tab_e0(I) * 128 + c0 + x];
            ec[x] = tab[tab_ec(I) * 128 + c0 + x];
            gref[x] = gb[I * 128 + c0 + x];
            glast[x] = gb[(I + 1) * 128 + c0 + x];
        }
        float kd[4][8], bv[4][8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = r0 + j;
            float kk[4], qq[4], vv[4], E[4], F[4];
            unpack4(kr[j], kk);
            unpack4(qr[j], qq);
            unpack4(vr[j], vv);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                E[x] = __expf(g[j][x] - gref[x]);
                F[x] = __expf(glast[x] - g[j][x]);
            }
            store4_split(sm + kAKQh, sm + kAKQl, sw128_offset(r, c0, 128), kk[0] * E[0], kk[1] * E[1],
                         kk[2] * E[2], kk[3] * E[3]);
            store4_split(sm + kAKQh, sm + kAKQl, sw128_offset(64 + r, c0, 128), qq[0] * E[0], qq[1] * E[1],
                         qq[2] * E[2], qq[3] * E[3]);
            // Q exp(g) into the Q' rows of the workspace image (completed at the end)
            store4_split(out + kOffWkQh, out + kOffWkQl, sw128_offset(64 + r, c0, 128), qq[0] * E[0] * e0[0],
                         qq[1] * E[1] * e0[1], qq[2] * E[2] * e0[2], qq[3] * E[3] * e0[3]);
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                if (R < I) continue;
                float f[4];
#pragma unroll
                for (int x = 0; x < 4; ++x)
                    f[x] = kk[x] * F[x] * tab[((R == I) ? tab_tau(R) : tab_sigma(R, I)) * 128 + c0 + x];
                store4_split(sm + kKFh, sm + kKFl, sw128_offset(kf_off(R) + r, c0, 160), f[0], f[1], f[2], f[3]);
            }
            const float b = sbeta[r];
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                kd[x][j] = kk[x] * F[x] * ec[x];
                bv[x][j] = b * vv[x];
            }
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            store8_split(out + kOffKdTh, out + kOffKdTl, sw128_chunk(c0 + x, r0, 128), kd[x]);
            store8_split(sm + kXVh, sm + kXVl, sw128_chunk(c0 + x, r0, 128), bv[x]);
        }
        if (tid < 128) reinterpret_cast<float*>(out + kOffGam)[tid] = __expf(gb[4 * 128 + tid]);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sflags[2];

    // ---- MMA 1: [K.E ; Q.E] (128 x 128) x versions^T (160 x 128), three terms --
    if (tid == 0) {
        mma3(tbase, smem_u32(sm + kAKQh), smem_u32(sm + kAKQl), 128, smem_u32(sm + kKFh), smem_u32(sm + kKFl), 160,
             kD / 16, idesc_bf16_f32(128, 160), false);
        mma_commit(&mbar);
    }
    uint32_t phase = 0;
    if (!mbar_wait(&mbar, phase)) {
        record_error(err, KDA_ERR_TIMEOUT);
        atomicExch(&sflags[1], 1u);
    }
    phase ^= 1;
    tc_fence_after();
    __syncthreads();
    const bool abort1 = sflags[1] != 0;

    float* As = reinterpret_cast<float*>(sm + kAs);
    float* Ts = reinterpret_cast<float*>(sm + kTs);
    float* scr = reinterpret_cast<float*>(sm + kScr);
    if (!abort1) {
        // ---- A and P out of TMEM ---------------------------------------------------
        // lane L < 64: row L of the key products; L >= 64: row L-64 of the query
        // products.  Warps w and w+4 share sub-partition w % 4 and split its columns.
        const int sp = warp & 3, L = 32 * sp + lane;
        const int r = L & 63;
        const bool is_p = L >= 64;
        const int R = r >> 4;
        const int cbeg = (sp & 1) ? 48 : 0, cend = (sp & 1) ? 160 : 48;
        const int ngrp = (cend - cbeg) / 16;
        const int half = (ngrp + 1) / 2;
        const int gbeg = (warp < 4) ? 0 : half, gend = (warp < 4) ? half : ngrp;
        const float br = sbeta[r];
        for (int gi = gbeg; gi < gend; ++gi) {
            float vals[16];
            tmem_ld16(tmem_addr(tbase, 32 * sp, cbeg + 16 * gi), vals);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int col = cbeg + 16 * gi + e;
                const int i = col - kf_off(R);
                if (i < 0 || i >= 16 * R + 16) continue;   // another block's version
                if (!is_p) As[r * 64 + i] = (i < r) ? br * vals[e] : 0.f;
                else store1_split(sm + kPh, sm + kPl, sw128_offset(r, i, 64), (i <= r) ? vals[e] : 0.f);
            }
        }
        if (warp < 4) {
            for (int i = 16 * R + 16; i < 64; ++i) {
                if (!is_p) As[r * 64 + i] = 0.f;
                else store1_split(sm + kPh, sm + kPl, sw128_offset(r, i, 64), 0.f);
            }
        }
        // (beta K exp(g))^T, three-term operand (MMA 1 no longer reads this region)
        float bk[4][8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float kk[4];
            unpack4(kr[j], kk);
            const float b = sbeta[r0 + j];
#pragma unroll
            for (int x = 0; x < 4; ++x) bk[x][j] = b * kk[x] * __expf(g[j][x]);
        }
#pragma unroll
        for (int x = 0; x < 4; ++x) store8_split(sm + kXKh, sm + kXKl, sw128_chunk(c0 + x, r0, 128), bk[x]);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- diagonal blocks with a large decay range: pairwise on CUDA cores ----------
    if (!abort1 && fbmask) {
        for (int R = 0; R < 4; ++R) {
            if (!(fbmask & (1u << R))) continue;
            float* sh = scr;   // [16][128] block-local cumulative log decay
            for (int e = tid; e < 16 * 128; e += kIntraThreads) {
                const int rr = e >> 7, c = e & 127, row = 16 * R + rr;
                sh[e] = (row < len) ? fmaxf(__bfloat162float(la[((size_t)(tok0 + row) * H + h) * kD + c]),
                                            kLogAlphaFloor)
                                    : 0.f;
            }
            __syncthreads();
            if (tid < 128)
                for (int rr = 1; rr < 16; ++rr) sh[rr * 128 + tid] += sh[(rr - 1) * 128 + tid];
            __syncthreads();
            for (int p = warp; p < 136; p += kIntraThreads / 32) {
                int rr = 0;
                while ((rr + 1) * (rr + 2) / 2 <= p) ++rr;
                const int ii = p - rr * (rr + 1) / 2;
                const int row = 16 * R + rr, col = 16 * R + ii;
                float sa = 0.f, spq = 0.f;
                if (row < len) {
                    const size_t ro = ((size_t)(tok0 + row) * H + h) * kD, io = ((size_t)(tok0 + col) * H + h) * kD;
                    for (int c = lane; c < 128; c += 32) {
                        const float kdv = __bfloat162float(k[io + c]) * __expf(sh[rr * 128 + c] - sh[ii * 128 + c]);
                        sa += __bfloat162float(k[ro + c]) * kdv;
                        spq += __bfloat162float(q[ro + c]) * kdv;
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    sa += __shfl_xor_sync(0xffffffffu, sa, o);
                    spq += __shfl_xor_sync(0xffffffffu, spq, o);
                }
                if (lane == 0) {
                    As[row * 64 + col] = (ii < rr) ? sbeta[row] * sa : 0.f;
                    store1_split(sm + kPh, sm + kPl, sw128_offset(row, col, 64), spq);
                }
            }
            __syncthreads();
        }
    }

    // ---- T = (I + A)^{-1}: diagonal 16 x 16 blocks, then by block distance -----------
    if (!abort1) {
        if (warp < 4 && lane < 16) {
            const int base = 16 * warp, j = lane;
            for (int rr = 0; rr < 16; ++rr) Ts[(base + rr) * 64 + base + j] = (rr == j) ? 1.f : 0.f;
            for (int rr = j + 1; rr < 16; ++rr) {
                float s = 0.f;
                for (int i = j; i < rr; ++i) s += As[(base + rr) * 64 + base + i] * Ts[(base + i) * 64 + base + j];
                Ts[(base + rr) * 64 + base + j] = -s;
            }
        }
        for (int e = tid; e < 64 * 64; e += kIntraThreads) {
            const int rr = e >> 6, cc = e & 63;
            if ((cc >> 4) > (rr >> 4)) Ts[e] = 0.f;
        }
        __syncthreads();
        float* Y = scr;   // [3][16][16]
        for (int d = 1; d < 4; ++d) {
            const int nb = 4 - d;
            for (int e = tid; e < nb * 256; e += kIntraThreads) {
                const int bi = e >> 8, rr = (e >> 4) & 15, ii = e & 15;
                const int R = bi + d, I2 = bi;
                float s = 0.f;
                for (int J = I2; J < R; ++J)
                    for (int m = 0; m < 16; ++m)
                        s += As[(16 * R + rr) * 64 + 16 * J + m] * Ts[(16 * J + m) * 64 + 16 * I2 + ii];
                Y[e] = s;
            }
            __syncthreads();
            for (int e = tid; e < nb * 256; e += kIntraThreads) {
                const int bi = e >> 8, rr = (e >> 4) & 15, ii = e & 15;
                const int R = bi + d, I2 = bi;
                float s = 0.f;
                for (int m = 0; m < 16; ++m) s += Ts[(16 * R + rr) * 64 + 16 * R + m] * Y[bi * 256 + m * 16 + ii];
                Ts[(16 * R + rr) * 64 + 16 * I2 + ii] = -s;
            }
            __syncthreads();
        }
        for (int e = tid; e < 64 * 8; e += kIntraThreads) {
            const int rr = e >> 3, k8 = (e & 7) * 8;
            store8_split(sm + kTh, sm + kTl, sw128_chunk(rr, k8, 64), Ts + rr * 64 + k8);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- MMA 2: [U | Wk] = T [beta V | beta K exp(g)] ------------------------------------
    if (tid == 0 && !abort1) {
        const uint32_t th = smem_u32(sm + kTh), tl = smem_u32(sm + kTl);
        mma3(tmem_addr(tbase, 0, 0), th, tl, 64, smem_u32(sm + kXVh), smem_u32(sm + kXVl), 128, kC / 16,
             idesc_bf16_f32(64, 128), false);
        mma3(tmem_addr(tbase, 0, 128), th, tl, 64, smem_u32(sm + kXKh), smem_u32(sm + kXKl), 128, kC / 16,
             idesc_bf16_f32(64, 128), false);
        mma_commit(&mbar);
    }
    if (!abort1 && !mbar_wait(&mbar, phase)) {
        record_error(err, KDA_ERR_TIMEOUT);
        atomicExch(&sflags[1], 1u);
    }
    phase ^= 1;
    tc_fence_after();
    __syncthreads();
    const bool abort2 = sflags[1] != 0;

    // ---- epilogue 2: U (fp32) and Wk (hi/lo image) to the workspace; U^T, Wk^T operands --
    // M = 64 layout: sub-partition sp, lanes 0-15 hold rows 16 sp + lane.
    if (!abort2) {
        const int sp = warp & 3;
        const int r = 16 * sp + (lane & 15);
        const bool second = warp >= 4;     // warps 4-7: the Wk half
        const bool active = lane < 16;
        for (int gi = 0; gi < 8; ++gi) {
            float vals[16];
            tmem_ld16(tmem_addr(tbase, 32 * sp, (second ? 128 : 0) + 16 * gi), vals);
            tmem_ld_wait();
            if (!active) continue;
            if (!second) {
                const int cb = (16 * gi) >> 5, cc = (16 * gi) & 31;
                float4* dst = reinterpret_cast<float4*>(out + kOffU + cb * 8192 + r * 128 + cc * 4);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[e] = make_float4(vals[4 * e], vals[4 * e + 1], vals[4 * e + 2], vals[4 * e + 3]);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    store1_split(sm + kUTh, sm + kUTl, sw128_offset(16 * gi + e, r, 128), vals[e]);
            } else {
                store8_split(out + kOffWkQh, out + kOffWkQl, sw128_chunk(r, 16 * gi, 128), vals);
                store8_split(out + kOffWkQh, out + kOffWkQl, sw128_chunk(r, 16 * gi + 8, 128), vals + 8);
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    store1_split(sm + kWTh, sm + kWTl, sw128_offset(16 * gi + e, r, 128), vals[e]);
            }
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- MMA 3: [U' | P Wk] = P [U | Wk] -------------------------------------------------
    if (tid == 0 && !abort2) {
        const uint32_t ph = smem_u32(sm + kPh), pl = smem_u32(sm + kPl);
        mma3(tmem_addr(tbase, 0, 0), ph, pl, 64, smem_u32(sm + kUTh), smem_u32(sm + kUTl), 128, kC / 16,
             idesc_bf16_f32(64, 128), false);
        mma3(tmem_addr(tbase, 0, 128), ph, pl, 64, smem_u32(sm + kWTh), smem_u32(sm + kWTl), 128, kC / 16,
             idesc_bf16_f32(64, 128), false);
        mma_commit(&mbar);
    }
    if (!abort2 && !mbar_wait(&mbar, phase)) {
        record_error(err, KDA_ERR_TIMEOUT);
        atomicExch(&sflags[1], 1u);
    }
    tc_fence_after();
    __syncthreads();
    const bool abort3 = sflags[1] != 0;

    // ---- epilogue 3: U' (fp32); Q' = Q exp(g) - P Wk (hi/lo image) -------------------------
    if (!abort3) {
        const int sp = warp & 3;
        const int r = 16 * sp + (lane & 15);
        const bool second = warp >= 4;
        const bool active = lane < 16;
        for (int gi = 0; gi < 8; ++gi) {
            float vals[16];
            tmem_ld16(tmem_addr(tbase, 32 * sp, (second ? 128 : 0) + 16 * gi), vals);
            tmem_ld_wait();
            if (!active) continue;
            if (!second) {
                const int cb = (16 * gi) >> 5, cc = (16 * gi) & 31;
                float4* dst = reinterpret_cast<float4*>(out + kOffU2 + cb * 8192 + r * 128 + cc * 4);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    dst[e] = make_float4(vals[4 * e], vals[4 * e + 1], vals[4 * e + 2], vals[4 * e + 3]);
            } else {
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const uint32_t off = sw128_chunk(64 + r, 16 * gi + 8 * hh, 128);
                    const uint4 qh = *reinterpret_cast<const uint4*>(out + kOffWkQh + off);
                    const uint4 ql = *reinterpret_cast<const uint4*>(out + kOffWkQl + off);
                    const float* pv = vals + 8 * hh;
                    float qv[8] = {bf16_lo(qh.x) + bf16_lo(ql.x), bf16_hi(qh.x) + bf16_hi(ql.x),
                                   bf16_lo(qh.y) + bf16_lo(ql.y), bf16_hi(qh.y) + bf16_hi(ql.y),
                                   bf16_lo(qh.z) + bf16_lo(ql.z), bf16_hi(qh.z) + bf16_hi(ql.z),
                                   bf16_lo(qh.w) + bf16_lo(ql.w), bf16_hi(qh.w) + bf16_hi(ql.w)};
#pragma unroll
                    for (int e = 0; e < 8; ++e) qv[e] -= pv[e];
                    store8_split(out + kOffWkQh, out + kOffWkQl, off, qv);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, 256);
}

// ============================================================================
// tc_recur
// ============================================================================
constexpr int kRecurThreads = 128;

template <int BV>
struct RecurLayout {
    static constexpr uint32_t kWkQ = 0;                                        // hi 32 KB + lo 32 KB
    static constexpr uint32_t kKdT = 65536;                                    // hi 16 KB + lo 16 KB
    static constexpr uint32_t kUtile = (uint32_t)BV * 64 * 4;                  // U (or U') tile, fp32
    static constexpr uint32_t kUStage = 2 * kUtile + 512;                      // U, U', Gamma_C
    static constexpr uint32_t kUU = 98304;                                     // two U stages
    static constexpr uint32_t kST = (kUU + 2 * kUStage + 1023) / 1024 * 1024;  // S^T hi/lo [BV][128 k]
    static constexpr uint32_t kWT = kST + 2 * (uint32_t)BV * 256;              // W^T hi/lo [BV][64 k]
    static constexpr uint32_t kBars = kWT + 2 * (uint32_t)BV * 128;
    static constexpr uint32_t kSmem = kBars + 128;
    static constexpr uint32_t kAlloc = kSmem + 1024;
    static constexpr uint32_t kTmemCols = (2 * BV < 32) ? 32 : 2 * BV;
};

template <int BV>
__global__ void __launch_bounds__(kRecurThreads, 1)
tc_recur(const uint8_t* __restrict__ ws, const float* __restrict__ init_state, float* __restrict__ final_state,
         __nv_bfloat16* __restrict__ o, int* __restrict__ err, SeqMap smap, int H) {
    using Lay = RecurLayout<BV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::kBars);
    uint64_t* wkq_full = bars + 0;
    uint64_t* kdt_full = bars + 1;
    uint64_t* uu_full = bars + 2;     // [2]
    uint64_t* bar1 = bars + 4;
    uint64_t* bar2 = bars + 5;
    uint32_t* sflags = reinterpret_cast<uint32_t*>(bars + 6);        // [0] tmem base, [1] abort
    uint8_t* sth = sm + Lay::kST;
    uint8_t* stl = sth + BV * 256;
    uint8_t* wth = sm + Lay::kWT;
    uint8_t* wtl = wth + BV * 128;

    const int tid = threadIdx.x, warp = tid >> 5;
    const SeqInfo sq = smap.get(blockIdx.x);
    const int h = blockIdx.y;
    const int j0 = blockIdx.z * BV;
    const int nch = (sq.len + kC - 1) / kC;
    const int cb0 = j0 / 32;   // first 32-column block of U / U'

    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
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
    const uint32_t t_d = tbase;              // D = [Wk ; Q'] S   (columns [0, BV))
    const uint32_t t_s = tbase + BV;         // S                 (columns [BV, 2 BV))

    auto chunk_src = [&](int n) {
        return ws + (size_t)((size_t)(sq.chunk0 + n) * H + h) * kChunkBytes;
    };
    auto load_wkq = [&](int n) {
        const uint8_t* src = chunk_src(n);
        mbar_arrive_expect_tx(wkq_full, 65536);
        bulk_g2s(sm + Lay::kWkQ, src + kOffWkQh, 32768, wkq_full);
        bulk_g2s(sm + Lay::kWkQ + 32768, src + kOffWkQl, 32768, wkq_full);
    };
    auto load_kdt = [&](int n) {
        const uint8_t* src = chunk_src(n);
        mbar_arrive_expect_tx(kdt_full, 32768);
        bulk_g2s(sm + Lay::kKdT, src + kOffKdTh, 16384, kdt_full);
        bulk_g2s(sm + Lay::kKdT + 16384, src + kOffKdTl, 16384, kdt_full);
    };
    auto load_uu = [&](int n, int stage) {
        const uint8_t* src = chunk_src(n);
        uint8_t* dst = sm + Lay::kUU + stage * Lay::kUStage;
        mbar_arrive_expect_tx(&uu_full[stage], Lay::kUStage);
        bulk_g2s(dst, src + kOffU + cb0 * 8192, Lay::kUtile, &uu_full[stage]);
        bulk_g2s(dst + Lay::kUtile, src + kOffU2 + cb0 * 8192, Lay::kUtile, &uu_full[stage]);
        bulk_g2s(dst + 2 * Lay::kUtile, src + kOffGam, 512, &uu_full[stage]);
    };
    if (tid == 0 && nch > 0) {
        load_wkq(0);
        load_kdt(0);
        load_uu(0, 0);
        if (nch > 1) load_uu(1, 1);
    }

    // this thread's state row c = tid, columns [j0, j0 + BV)
    const int c = tid;
    float s[BV];
    {
        const size_t base = (((size_t)sq.seq * H + h) * kD + c) * kD + j0;
#pragma unroll
        for (int j = 0; j < BV; j += 4) {
            float4 x = init_state ? *reinterpret_cast<const float4*>(init_state + base + j)
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
            s[j] = x.x; s[j + 1] = x.y; s[j + 2] = x.z; s[j + 3] = x.w;
        }
    }

    for (int n = 0; n < nch; ++n) {
        const int stage = n & 1;
        const uint8_t* uu = sm + Lay::kUU + stage * Lay::kUStage;
        // S_n as the B operand of MMA 1 (three-term): element (row j, k = c)
#pragma unroll
        for (int j = 0; j < BV; ++j) store1_split(sth, stl, sw128_offset(j, c, BV), s[j]);
        if (!mbar_wait(&uu_full[stage], (uint32_t)(n >> 1) & 1u)) {
            record_error(err, KDA_ERR_TIMEOUT);
            atomicExch(&sflags[1], 1u);
        }
        // Diag(Gamma_C) S_n into TMEM; MMA 2 accumulates on top of it
        const float gam = reinterpret_cast<const float*>(uu + 2 * Lay::kUtile)[c];
#pragma unroll
        for (int jb = 0; jb < BV; jb += 16) {
            float t[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) t[e] = gam * s[jb + e];
            tmem_st16(tmem_addr(t_s, 32 * warp, jb), t);
        }
        tmem_st_wait();
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (sflags[1]) break;
        tc_fence_after();
        if (tid == 0) {
            if (!mbar_wait(wkq_full, (uint32_t)n & 1u)) {
                record_error(err, KDA_ERR_TIMEOUT);
                atomicExch(&sflags[1], 1u);
            } else {
                const uint32_t a = smem_u32(sm + Lay::kWkQ);
                mma3(t_d, a, a + 32768, 128, smem_u32(sth), smem_u32(stl), BV, kD / 16, idesc_bf16_f32(128, BV),
                     false);
            }
            mma_commit(bar1);
        }
        if (!mbar_wait(bar1, (uint32_t)n & 1u)) {
            record_error(err, KDA_ERR_TIMEOUT);
            atomicExch(&sflags[1], 1u);
        }
        tc_fence_after();
        if (tid == 0 && n + 1 < nch) load_wkq(n + 1);   // MMA 1 is done with the buffer
        // lanes 0-63: W = U - Wk S (rows are tokens); lanes 64-127: O = Q' S + U'
        {
            const int r = tid & 63;
            const float* ut = reinterpret_cast<const float*>(uu + ((tid < 64) ? 0 : Lay::kUtile));
            const int rows_here = min(kC, sq.len - n * kC);
#pragma unroll
            for (int jb = 0; jb < BV; jb += 16) {
                float d[16];
                tmem_ld16(tmem_addr(t_d, 32 * warp, jb), d);
                tmem_ld_wait();
                float u[16];
#pragma unroll
                for (int e = 0; e < 16; e += 4) {
                    const int j = jb + e;
                    const float4 w = *reinterpret_cast<const float4*>(ut + (j >> 5) * 2048 + r * 32 + (j & 31));
                    u[e] = w.x; u[e + 1] = w.y; u[e + 2] = w.z; u[e + 3] = w.w;
                }
                if (tid < 64) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) store1_split(wth, wtl, sw128_offset(jb + e, r, BV), u[e] - d[e]);
                } else if (r < rows_here) {
                    __nv_bfloat16* dst = o + ((size_t)(sq.tok0 + n * kC + r) * H + h) * kD + j0 + jb;
                    uint4 w0, w1;
                    w0.x = pack_bf16(d[0] + u[0], d[1] + u[1]); w0.y = pack_bf16(d[2] + u[2], d[3] + u[3]);
                    w0.z = pack_bf16(d[4] + u[4], d[5] + u[5]); w0.w = pack_bf16(d[6] + u[6], d[7] + u[7]);
                    w1.x = pack_bf16(d[8] + u[8], d[9] + u[9]); w1.y = pack_bf16(d[10] + u[10], d[11] + u[11]);
                    w1.z = pack_bf16(d[12] + u[12], d[13] + u[13]); w1.w = pack_bf16(d[14] + u[14], d[15] + u[15]);
                    reinterpret_cast<uint4*>(dst)[0] = w0;
                    reinterpret_cast<uint4*>(dst)[1] = w1;
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (sflags[1]) break;
        tc_fence_after();
        if (tid == 0) {
            if (!mbar_wait(kdt_full, (uint32_t)n & 1u)) {
                record_error(err, KDA_ERR_TIMEOUT);
                atomicExch(&sflags[1], 1u);
            } else {
                const uint32_t a = smem_u32(sm + Lay::kKdT);
                mma3(t_s, a, a + 16384, 128, smem_u32(wth), smem_u32(wtl), BV, kC / 16, idesc_bf16_f32(128, BV),
                     true);
            }
            mma_commit(bar2);
        }
        if (!mbar_wait(bar2, (uint32_t)n & 1u)) {
            record_error(err, KDA_ERR_TIMEOUT);
            atomicExch(&sflags[1], 1u);
        }
        tc_fence_after();
        if (tid == 0) {
            if (n + 1 < nch) load_kdt(n + 1);          // MMA 2 is done with the buffer
            if (n + 2 < nch) load_uu(n + 2, stage);    // every thread is past its reads of this stage
        }
#pragma unroll
        for (int jb = 0; jb < BV; jb += 16) {
            float t[16];
            tmem_ld16(tmem_addr(t_s, 32 * warp, jb), t);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 16; ++e) s[jb + e] = t[e];
        }
    }
    __syncthreads();
    const bool failed = sflags[1] != 0;
    if (!failed && final_state) {
        const size_t base = (((size_t)sq.seq * H + h) * kD + c) * kD + j0;
#pragma unroll
        for (int j = 0; j < BV; j += 4)
            *reinterpret_cast<float4*>(final_state + base + j) = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
    }
    if (failed && tid == 0) {
        // a wait gave up: give in-flight copies and MMAs a bounded time to land before freeing TMEM
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
cudaError_t launch_recur(const uint8_t* ws, const float* init_state, float* final_state, __nv_bfloat16* o, int* err,
                         const SeqMap& smap, int n_seqs, int H, cudaStream_t stream) {
    using Lay = RecurLayout<BV>;
    cudaError_t e = cudaFuncSetAttribute(tc_recur<BV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::kAlloc);
    if (e != cudaSuccess) return e;
    tc_recur<BV><<<dim3(n_seqs, H, kD / BV), kRecurThreads, Lay::kAlloc, stream>>>(ws, init_state, final_state, o,
                                                                                   err, smap, H);
    return cudaGetLastError();
}

}  // namespace

bool tc_available() { return true; }

bool tc_supports(int C) { return C == kC; }

size_t tc_workspace_bytes(int n_chunks, int H, int C) {
    if (C != kC) return 0;
    return kErrHeader + (size_t)n_chunks * H * kChunkBytes;
}

cudaError_t launch_tc_prefill(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                              const float* init_state, void* o, float* final_state, const ChunkMap& cmap,
                              const SeqMap& smap, int n_chunks, int n_seqs, int H, int C, void* tc_ws,
                              cudaStream_t stream) {
    if (C != kC) return cudaErrorNotSupported;
    int* err = reinterpret_cast<int*>(tc_ws);
    uint8_t* ws = reinterpret_cast<uint8_t*>(tc_ws) + kErrHeader;
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
    if (n_chunks > 0) {
        e = cudaFuncSetAttribute(tc_intra, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kIntraAlloc);
        if (e != cudaSuccess) return e;
        tc_intra<<<dim3(n_chunks, H), kIntraThreads, kIntraAlloc, stream>>>(
            (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
            (const __nv_bfloat16*)log_alpha, (const __nv_bfloat16*)beta, ws, err, cmap, H);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    timing_mark(stream, 1);
    if (n_seqs > 0) {
        const long units = (long)n_seqs * H;
        if (units * 4 <= 148)
            e = launch_recur<32>(ws, init_state, final_state, (__nv_bfloat16*)o, err, smap, n_seqs, H, stream);
        else
            e = launch_recur<64>(ws, init_state, final_state, (__nv_bfloat16*)o, err, smap, n_seqs, H, stream);
        if (e != cudaSuccess) return e;
    }
    timing_mark(stream, 2);
    return cudaSuccess;
}

}  // namespace kda
