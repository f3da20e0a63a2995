// Tensor-core (tcgen05) chunkwise KDA prefill: bf16 inputs, d_k = d_v = 128,
// chunk C = 64, fp32 state and accumulation.
//
// Two kernels:
//
//   tc_intra  (one CTA per (chunk, head), all chunks in parallel, 2 CTAs/SM)
//     cumulative log decay g (row a1); on the tensor cores the decay-weighted
//     strictly-lower A = Diag(beta) (K K^T . exp(g_r - g_i)) and the inclusive
//     score matrix P = (Q K^T . exp(g_r - g_i)); T = (I + A)^{-1} by blocked
//     substitution on CUDA cores; then on the tensor cores
//       T [beta V | beta K exp(g)] = [U | Wk]                                  (row a2)
//     i.e. U = T Diag(beta) V, Wk = T Diag(beta)(K . exp(g)), plus Q . exp(g),
//     P, Kd = K . exp(g_C - g) and Gamma_C = exp(g_C).  Results go to the
//     workspace in the layout the second kernel consumes.
//
//   tc_recur  (one CTA per (sequence, head, d_v tile), sequential over chunks)
//     with the fp32 state tile S (d_k x BV) in TMEM:
//       D   = [Wk ; Q . exp(g)] S                 M = 128 MMA
//       W   = U - D[0:64]                         per-token corrections
//       S  <- Diag(Gamma_C) S + Kd^T W            M = 128 MMA accumulating in TMEM (row a3)
//       D  += [0 ; P] W,  O = D[64:128]           outputs (row a4), read during the next chunk
//     The next chunk's operands stream in by 1-D bulk copies (TMA engine, each
//     into this CTA's own shared memory) while the current chunk is processed.
//
// Derivation (ours; the oracle's chunk form checks it against the token
// recurrence): with Gamma_r = exp(g_r) the per-token corrections W solve
// (I + A) W = Diag(beta)(V - (K . Gamma) S_0), so W = U - Wk S_0; the outputs
// are O = (Q . Gamma) S_0 + P W; the next state is Diag(Gamma_C) S_0 + Kd^T W.  Chunkwise form: "From GPT-2 to Kimi K3" essay
// (pwwt.cn/news/3716252), chunkwise and Gated DeltaNet paragraphs; WY / DPLR
// restructuring: "我终于看懂了 KDA" explainer (pwwt.cn/news/3787313),
// sections 16-17.
//
// Precision.  Every tensor-core product is formed in three bf16 terms,
// a_hi b_hi + a_hi b_lo + a_lo b_hi (hi = RN_bf16(x), lo = RN_bf16(x - hi)),
// with fp32 accumulation: about 16 significant bits per operand.  Heavy decay
// lets single tokens dominate many of the sums, so one bf16 rounding of an
// operand would show up at ~2^-9 times the heavy tail of o; three terms keep
// the path in the fp32 regime.  U is stored in fp32.
//
// Decay factors.  Rows form 16-row blocks; gb[b] is g at the row before block
// b (gb[0] = 0), gb[4] = g_C.  Every factor handed to the tensor cores is exp of
// a non-positive difference, except exp(gb[I] - gb[I+1]) (<= exp(decay range
// of block I)) on the diagonal blocks; a block whose range exceeds kDiagRange
// nats has its diagonal A / P entries recomputed pairwise on CUDA cores.
#include "kda_internal.cuh"
#include "kda_tc.cuh"
#include "kda_tc_image.cuh"

namespace kda {

extern const char* const kTcKernelNames[] = {"tc_intra", "tc_recur"};
extern const int kTcKernelCount = 2;

namespace {

using namespace tc;
using namespace tcimg;

constexpr int kC = 64;
constexpr int kD = 128;
constexpr float kDiagRange = 80.0f;

// ---- tc_intra shared memory (byte offsets from a 1024-aligned base) -----------
constexpr int kIntraThreads = 256;
// first MMA, one half of the channels at a time
constexpr uint32_t kAKQh = 0;            // [K.E ; Q.E]  128 rows x 64 k
constexpr uint32_t kAKQl = 16384;
constexpr uint32_t kKFh = 32768;         // decayed key versions 160 rows x 64 k
constexpr uint32_t kKFl = 53248;
constexpr uint32_t kKdStage = 73728;     // Kd^T rows of one channel half, hi 8 KB + lo 8 KB (bulk-copied out)
constexpr uint32_t kLaStage = 73728;     // at the start: the chunk's log alpha rows (64 x 256 B, bulk-copied in)
// after the first MMA
constexpr uint32_t kAs = 0;              // A fp32 [64][65]
constexpr uint32_t kPh = 17408;          // P 64 x 64 (K-major)
constexpr uint32_t kPl = 25600;
constexpr uint32_t kScr = 33792;         // 8 KB scratch
constexpr uint32_t kTs = 41984;          // T fp32 [64][68]
constexpr uint32_t kFbStage = 41984;     // before T: rows of a large-range diagonal block (3 x 8 KB)
// T (64 rows x 64 k, K-major), the A operand of the last product
constexpr uint32_t kTPh = 65536;
constexpr uint32_t kTPl = 81920;
// [beta V | beta K exp(g)] (MN-major, 64 token rows x 256 columns)
constexpr uint32_t kXh = 0;
constexpr uint32_t kXl = 32768;
constexpr uint32_t kTab = 98304;         // tables
constexpr int kNumTab = 18;              // tau[4], sigma[6], exp(gb)[4], exp(g_C - gb[b+1])[4]
constexpr uint32_t kIntraBars = kTab + kNumTab * 128 * 4 + 5 * 128 * 4 + 3 * 64 * 4 + 64;   // 3 mbarriers
constexpr uint32_t kIntraSmem = kIntraBars + 32;
// no static shared memory: the dynamic region starts at the CTA's (1024-aligned)
// shared window, so the kernel addresses it without a runtime offset
constexpr uint32_t kIntraAlloc = kIntraSmem;
constexpr int kGCol = 192;               // TMEM columns 192-255 hold g until the last product
constexpr int kAS = 65;                  // row stride of As (floats)
constexpr int kTS = 68;                  // row stride of Ts (floats; rows 16-byte aligned)

// rows of the decayed-key versions: version R covers keys [0, 16 R + 16)
__host__ __device__ __forceinline__ int kf_off(int R) { return (R * (R + 1)) * 8; }   // 0, 16, 48, 96

__device__ __forceinline__ int tab_tau(int R) { return R; }                                  // exp(gb[R] - gb[R+1])
__device__ __forceinline__ int tab_sigma(int R, int I) { return 4 + (R * (R - 1)) / 2 + I; } // exp(gb[R] - gb[I+1]), I < R
__device__ __forceinline__ int tab_e0(int I) { return 10 + I; }                              // exp(gb[I])
__device__ __forceinline__ int tab_ec(int I) { return 14 + I; }                              // exp(g_C - gb[I+1])

// two values of one row -> 4-byte stores into the hi and lo tiles
__device__ __forceinline__ void store2_split(uint8_t* hi_tile, uint8_t* lo_tile, uint32_t off, float a, float b) {
    uint32_t hv, lv;
    split2(a, b, hv, lv);
    *reinterpret_cast<uint32_t*>(hi_tile + off) = hv;
    *reinterpret_cast<uint32_t*>(lo_tile + off) = lv;
}

// eight consecutive values (one 16-byte chunk) split into hi and lo tiles
__device__ __forceinline__ void store8_split(uint8_t* hi_tile, uint8_t* lo_tile, uint32_t off, const float* x) {
    uint4 hv, lv;
    split2(x[0], x[1], hv.x, lv.x);
    split2(x[2], x[3], hv.y, lv.y);
    split2(x[4], x[5], hv.z, lv.z);
    split2(x[6], x[7], hv.w, lv.w);
    *reinterpret_cast<uint4*>(hi_tile + off) = hv;
    *reinterpret_cast<uint4*>(lo_tile + off) = lv;
}

// The same with the hi and lo values at different offsets of their tiles.
__device__ __forceinline__ void store8_split2(uint8_t* hi, uint32_t ohi, uint8_t* lo, uint32_t olo, const float* x) {
    uint4 hv, lv;
    split2(x[0], x[1], hv.x, lv.x);
    split2(x[2], x[3], hv.y, lv.y);
    split2(x[4], x[5], hv.z, lv.z);
    split2(x[6], x[7], hv.w, lv.w);
    *reinterpret_cast<uint4*>(hi + ohi) = hv;
    *reinterpret_cast<uint4*>(lo + olo) = lv;
}

__device__ __forceinline__ void record_error(int* err, int code) {
    if (err) atomicCAS(err, 0, code);
}

// D (+)= A B^T over `ksteps` K-slices of 16, in three bf16 terms; A K-major,
// B K-major (b_mn = false) or MN-major (b_mn = true, `brows` = K rows).
__device__ __forceinline__ void mma3(uint32_t d, uint32_t ah, uint32_t al, int arows, uint32_t bh, uint32_t bl,
                                     int brows, bool b_mn, int ksteps, uint32_t idesc, bool accumulate) {
    for (int s = 0; s < ksteps; ++s) {
        const uint32_t acc0 = (accumulate || s > 0) ? 1u : 0u;
        const uint64_t dah = sw128_desc_k(ah, arows, s), dal = sw128_desc_k(al, arows, s);
        const uint64_t dbh = b_mn ? mn_desc_k(bh, brows, s) : sw128_desc_k(bh, brows, s);
        const uint64_t dbl = b_mn ? mn_desc_k(bl, brows, s) : sw128_desc_k(bl, brows, s);
        mma_bf16(d, dah, dbh, idesc, acc0);
        mma_bf16(d, dah, dbl, idesc, 1u);
        mma_bf16(d, dal, dbh, idesc, 1u);
    }
}

// The same three terms with B MN-major and its hi and lo tiles side by side as one
// operand [B_hi | B_lo] of width 2N (the lo tile one 64-wide block after the hi
// tile): D[0, N) (+)= A_hi B_hi + A_lo B_hi and D[N, 2N) (+)= A_hi B_lo, two MMAs
// per K-slice instead of three (each A tile read once); the caller adds the two
// halves of D.
__device__ __forceinline__ void mma2w(uint32_t d, uint32_t ah, uint32_t al, int arows, uint32_t bh, int brows,
                                      int ksteps, uint32_t idesc_wide, uint32_t idesc_narrow, bool accumulate) {
    for (int s = 0; s < ksteps; ++s) {
        const uint32_t acc0 = (accumulate || s > 0) ? 1u : 0u;
        const uint64_t dah = sw128_desc_k(ah, arows, s), dal = sw128_desc_k(al, arows, s);
        const uint64_t db = mn_desc_k(bh, brows, s);
        mma_bf16(d, dah, db, idesc_wide, acc0);
        mma_bf16(d, dal, db, idesc_narrow, 1u);
    }
}

// Columns [c0, c0 + 2 NC) of the block column I of T = (I + A)^{-1}, below the
// diagonal, given the diagonal inverses T_JJ in Ts: for R = I+1 .. 3,
// Y = sum_{I <= J < R} A_RJ T_JI and T_RI = -T_RR Y.  One warp: lane = (row r of
// the block, column group lane / 16 of NC columns).
template <int NC>
__device__ __forceinline__ void tsolve_cols(const float* As, float* Ts, float* Yw, int I, int c0, int lane) {
    const int r = lane & 15;
    const int cl = (lane >> 4) * NC;        // first column of this lane inside the slice
    const int col = c0 + cl;
    for (int R = I + 1; R < 4; ++R) {
        float2 acc[NC / 2];
#pragma unroll
        for (int x = 0; x < NC / 2; ++x) acc[x] = make_float2(0.f, 0.f);
        for (int J = I; J < R; ++J) {
            const float* arow = As + (16 * R + r) * kAS + 16 * J;
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const float2 av = make_float2(arow[m], arow[m]);
                const float* trow = Ts + (16 * J + m) * kTS + col;
#pragma unroll
                for (int x = 0; x < NC / 2; ++x)
                    acc[x] = fma2(av, *reinterpret_cast<const float2*>(trow + 2 * x), acc[x]);
            }
        }
#pragma unroll
        for (int x = 0; x < NC / 2; ++x) *reinterpret_cast<float2*>(Yw + r * 8 + cl + 2 * x) = acc[x];
        __syncwarp();
        float2 t[NC / 2];
#pragma unroll
        for (int x = 0; x < NC / 2; ++x) t[x] = make_float2(0.f, 0.f);
        const float* drow = Ts + (16 * R + r) * kTS + 16 * R;
#pragma unroll
        for (int m = 0; m < 16; ++m) {
            const float2 dv = make_float2(drow[m], drow[m]);
#pragma unroll
            for (int x = 0; x < NC / 2; ++x)
                t[x] = fma2(dv, *reinterpret_cast<const float2*>(Yw + m * 8 + cl + 2 * x), t[x]);
        }
#pragma unroll
        for (int x = 0; x < NC / 2; ++x)
            *reinterpret_cast<float2*>(Ts + (16 * R + r) * kTS + col + 2 * x) = make_float2(-t[x].x, -t[x].y);
        __syncwarp();   // T_RI is read at the next level; Yw is reused
    }
}

// ============================================================================
// tc_intra
// ============================================================================
template <bool PREP>
__global__ void __launch_bounds__(kIntraThreads, 2)
tc_intra(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
         const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ la,
         const __nv_bfloat16* __restrict__ beta, uint8_t* __restrict__ ws, int* __restrict__ err, ChunkMap cmap,
         int H, unsigned prep_flags, unsigned long long stall_ns, float* __restrict__ t_store,
         float* __restrict__ at_store) {
    // PREP = false is the plain operator: no preprocessing code is compiled in
    const unsigned prep = PREP ? prep_flags : 0u;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // The swizzled operand tiles need a 1024-byte aligned base.  This kernel has no
    // static shared memory, so its dynamic region starts at the CTA's shared window;
    // should that ever not be 1024-aligned, the kernel records an error and stops.
    if (smem_u32(smem_raw) & 1023u) {
        if (threadIdx.x == 0) atomicCAS(err, 0, (int)KDA_ERR_DEVICE);
        return;
    }
    uint8_t* sm = smem_raw;
    float* tab = reinterpret_cast<float*>(sm + kTab);                 // [18][128]
    float* gb = tab + kNumTab * 128;                                  // [5][128]
    float* sbeta = gb + 5 * 128;                                      // [64]
    float* inv_nk = sbeta + 64;                                       // [64] 1 / ||k_r|| (1 without normalisation)
    float* inv_nq = inv_nk + 64;                                      // [64] 1 / ||q_r||
    uint32_t* sflags = reinterpret_cast<uint32_t*>(inv_nq + 64);      // [0] fallback mask, [1] abort, [2] tmem base
    uint64_t& mbar = reinterpret_cast<uint64_t*>(sm + kIntraBars)[0];      // tensor-core products, in issue order
    uint64_t& mbar_k = reinterpret_cast<uint64_t*>(sm + kIntraBars)[1];    // the second half of the last product
    uint64_t& mbar_never = reinterpret_cast<uint64_t*>(sm + kIntraBars)[3];  // completed by nothing (failure test)

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // this thread: rows [8 w, 8 w + 8) of 16-row block I = w / 2, and channels
    // 2 lane, 2 lane + 1 of each 64-channel half (index x = 2 half + e)
    const int I = warp >> 1;
    const int kc = 2 * lane;                  // channel inside a half
    const int r0 = 8 * warp;
    int seq, tok0, len, cidx;
    // heads vary fastest over the grid: CTAs that run together read neighbouring
    // 256-byte pieces of the same token rows and write neighbouring workspace images
    const int chunk = (int)(blockIdx.x / (unsigned)H);
    const int h = (int)(blockIdx.x - (unsigned)chunk * (unsigned)H);
    cmap.locate(chunk, seq, tok0, len, cidx);
    uint8_t* out = ws + (size_t)((size_t)chunk * H + h) * kChunkBytes;

    if (tid == 0) {
        sflags[0] = 0;
        sflags[1] = 0;
        mbar_init(&mbar, 1);
        mbar_init(&mbar_k, 1);
        mbar_init(&mbar_never, 1);
        mbar_init_fence();
    }
    if (warp == 0) {
        tmem_alloc(&sflags[2], 256);
        tmem_relinquish();
    }
    __syncthreads();   // barriers initialised
    // log alpha rows by plain 16-byte loads (thread: 4 pieces of 8 channels), staged below;
    // the SM's bulk-copy engine is busy with the other CTA's workspace stores
    uint4 la_pc[4];
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int e = tid + 256 * it, r = e >> 4, c8 = (e & 15) * 8;
        la_pc[it] = make_uint4(0u, 0u, 0u, 0u);
        if (r < len) la_pc[it] = *reinterpret_cast<const uint4*>(la + ((size_t)(tok0 + r) * H + h) * kD + c8);
    }
    // key / query rows for the normalisation, read row-wise (coalesced) before anything
    // waits: warp w takes rows 16 (w % 4) .. + 15 of k (w < 4) or q (w >= 4), lane l
    // channels 4l .. 4l + 3
    uint2 nu[16];
    if (PREP && (prep & KDA_PREP_QK_L2NORM)) {
        const __nv_bfloat16* src = warp < 4 ? k : q;
        const int rb = 16 * (warp & 3);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            nu[i] = make_uint2(0u, 0u);
            if (rb + i < len)
                nu[i] = *reinterpret_cast<const uint2*>(src + ((size_t)(tok0 + rb + i) * H + h) * kD + 4 * lane);
        }
    }
    // beta stays as raw bits until it is stored, so that nothing waits for this load
    const unsigned short beta_raw =
        (tid < len && tid < 64) ? reinterpret_cast<const unsigned short*>(beta)[(size_t)(tok0 + tid) * H + h] : 0;
    // ---- log alpha of 8 rows x 4 channels; k, q, v prefetched into L2 ---------
    // (k and q of a channel half are read one phase before the round that uses
    // them, v at the end; holding them in registers through the chunk would push
    // the kernel past 128 registers)
    float g[8][4];
    uint32_t kv[8], qv[8];
    auto load_kq = [&](int hr) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = r0 + j;
            kv[j] = qv[j] = 0u;
            if (r < len) {
                const size_t off = ((size_t)(tok0 + r) * H + h) * kD + 64 * hr + kc;
                kv[j] = *reinterpret_cast<const uint32_t*>(k + off);
                qv[j] = *reinterpret_cast<const uint32_t*>(q + off);
            }
        }
    };
    if (lane < 16) {
        const int r = r0 + (lane & 7);
        if (r < len) {
            const size_t off = ((size_t)(tok0 + r) * H + h) * kD + 64 * (lane >> 3);
            asm volatile("prefetch.global.L2 [%0];" ::"l"(k + off));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(q + off));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(v + off));
        }
    }
    load_kq(0);
    // key / query normalisation factors: the sums of squares are formed here, from
    // the rows loaded at the start
    if (PREP && (prep & KDA_PREP_QK_L2NORM)) {
        float ss[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float a = bf16_lo(nu[i].x), b = bf16_hi(nu[i].x), c = bf16_lo(nu[i].y), d = bf16_hi(nu[i].y);
            ss[i] = fmaf(a, a, fmaf(b, b, fmaf(c, c, d * d)));
        }
        // halving exchanges (distance 16, 8, 4, 2: each keeps the half of the rows that
        // the lane's bit selects), then the pair (2m, 2m + 1) adds its two halves of row m
#pragma unroll
        for (int w = 8; w >= 1; w >>= 1) {
            const bool up = (lane & (2 * w)) != 0;
#pragma unroll
            for (int m = 0; m < w; ++m) {
                const float keep = up ? ss[m + w] : ss[m];
                const float give = up ? ss[m] : ss[m + w];
                ss[m] = keep + __shfl_xor_sync(0xffffffffu, give, 2 * w);
            }
        }
        const float tot = ss[0] + __shfl_xor_sync(0xffffffffu, ss[0], 1);
        if ((lane & 1) == 0) inv_nk[(warp < 4 ? 0 : 64) + 16 * (warp & 3) + (lane >> 1)] = inv_norm_from_sq(tot);
    } else if (PREP && tid < 128) {
        inv_nk[tid] = 1.f;   // inv_nk [0, 64) and inv_nq [64, 128) are adjacent
    }
#pragma unroll
    for (int it = 0; it < 4; ++it) {
        const int e = tid + 256 * it, r = e >> 4, c8 = (e & 15) * 8;
        *reinterpret_cast<uint4*>(sm + kLaStage + r * 256 + c8 * 2) = la_pc[it];
    }
    __syncthreads();
    // test of the failure path (stall_ns != 0, set through kda_set_test_wait_limit):
    // the first CTA waits, bounded by stall_ns, on a barrier that nothing completes,
    // then records the timeout and takes the abort path like any expired wait
    if (stall_ns != 0ull && blockIdx.x == 0 && tid == 0 && !mbar_wait(&mbar_never, 0, stall_ns)) {
        record_error(err, KDA_ERR_TIMEOUT);
        atomicExch(&sflags[1], 1u);
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int r = r0 + j;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t a = 0u;
            if (r < len) a = *reinterpret_cast<const uint32_t*>(sm + kLaStage + r * 256 + (64 * hh + kc) * 2);
            const float2 l2 = prep_log_alpha2(unpack_bf16x2(a), prep);
            g[j][2 * hh] = (r < len) ? l2.x : 0.f;
            g[j][2 * hh + 1] = (r < len) ? l2.y : 0.f;
        }
    }
    if (tid < 64) sbeta[tid] = (tid < len) ? prep_beta(__uint_as_float((uint32_t)beta_raw << 16), prep) : 0.f;
    // ---- cumulative log decay (row a1): local prefix, then carries ----------
#pragma unroll
    for (int j = 1; j < 8; ++j)
#pragma unroll
        for (int x = 0; x < 4; ++x) g[j][x] += g[j - 1][x];
    float* tot = tab;   // [8][128] per-warp totals; the tables are built after their last use
#pragma unroll
    for (int x = 0; x < 4; ++x) tot[warp * 128 + 64 * (x >> 1) + kc + (x & 1)] = g[7][x];
    __syncthreads();
    float carry[4] = {0.f, 0.f, 0.f, 0.f};
    for (int p = 0; p < warp; ++p)
#pragma unroll
        for (int x = 0; x < 4; ++x) carry[x] += tot[p * 128 + 64 * (x >> 1) + kc + (x & 1)];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int x = 0; x < 4; ++x) g[j][x] += carry[x];
    // g is kept for the [beta V | beta K exp(g)] operand in TMEM columns 192-255, which no
    // product writes before that operand is built: warp w stores its 8 rows x 4 channels
    // in its own sub-partition (lane = its lane), 32 columns from 192 + 32 (w / 4)
    const uint32_t tbase = sflags[2];
    const uint32_t t_g = tmem_addr(tbase, 32 * (warp & 3), kGCol + 32 * (warp >> 2));
    {
        float gs[16];
#pragma unroll
        for (int hj = 0; hj < 2; ++hj) {
#pragma unroll
            for (int i = 0; i < 16; ++i) gs[i] = g[4 * hj + (i >> 2)][i & 3];
            tmem_st16(t_g + 16 * hj, gs);
        }
    }
    if (tid < 128) gb[tid] = 0.f;
    if (warp & 1) {
#pragma unroll
        for (int x = 0; x < 4; ++x) gb[(I + 1) * 128 + 64 * (x >> 1) + kc + (x & 1)] = g[7][x];
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
    if (tid < 128) reinterpret_cast<float*>(out + kOffGam)[tid] = __expf(gb[4 * 128 + tid]);

    uint32_t phase = 0;
    bool abort = false;

    // ---- first MMA in two channel halves --------------------------------------------
    // Round hr: every thread reads k and q of its 8 rows for its two channels in
    // half hr, builds that half's MMA operands and writes its Q exp(g) and Kd
    // values to the workspace.  (The two rounds share one copy of the code: the
    // kernel's largest stall is instruction fetch.)
#pragma unroll 1
    for (int hr = 0; hr < 2; ++hr) {
        const int ch = 64 * hr + kc;
        // e = exp(g - gb[I]), f = exp(gb[I+1] - g)
        // (pairs of channels as one 8-byte load: the lanes of a warp read 256
        // consecutive bytes without bank conflicts)
        auto pair = [](const float* p) { return *reinterpret_cast<const float2*>(p); };
        const float2 gref = pair(gb + I * 128 + ch);
        const float2 glast = pair(gb + (I + 1) * 128 + ch);
        const float2 xq = pair(tab + tab_e0(I) * 128 + ch);
        const float2 yk = pair(tab + tab_ec(I) * 128 + ch);
        float2 sgv[4];
#pragma unroll
        for (int R = 0; R < 4; ++R) {
            const float* sg = tab + ((R == I) ? tab_tau(R) : tab_sigma(R > I ? R : I + 1, I)) * 128 + ch;
            sgv[R] = (R < I) ? make_float2(0.f, 0.f) : pair(sg);
        }
        float kd0[8], kd1[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = r0 + j;
            const float2 gj = hr ? make_float2(g[j][2], g[j][3]) : make_float2(g[j][0], g[j][1]);
            const float2 e = exp_diff2(gj, gref), f = exp_diff2(glast, gj);
            float2 k2 = unpack_bf16x2(kv[j]), q2 = unpack_bf16x2(qv[j]);
            if (PREP) {
                k2 = mul2(k2, make_float2(inv_nk[r], inv_nk[r]));
                q2 = mul2(q2, make_float2(inv_nq[r], inv_nq[r]));
            }
            const float2 ke = mul2(k2, e), qe = mul2(q2, e), kf = mul2(k2, f);
            store2_split(sm + kAKQh, sm + kAKQl, sw128_offset(r, kc, 128), ke.x, ke.y);
            store2_split(sm + kAKQh, sm + kAKQl, sw128_offset(64 + r, kc, 128), qe.x, qe.y);
#pragma unroll
            for (int R = 0; R < 4; ++R) {
                if (R < I) continue;
                const float2 kfs = mul2(kf, sgv[R]);
                store2_split(sm + kKFh, sm + kKFl, sw128_offset(kf_off(R) + r, kc, 160), kfs.x, kfs.y);
            }
            const float2 qg = mul2(qe, xq), kd = mul2(kf, yk);
            store2_split(out + kOffWkQh, out + kOffWkQl, sw128_offset(64 + r, ch, 128), qg.x, qg.y);
            kd0[j] = kd.x;
            kd1[j] = kd.y;
        }
        // Kd^T rows ch, ch + 1 (this half's 64 rows are staged, then copied out whole).
        // Lanes 4m..4m+3 store the even row first when m is even and the odd row
        // first when m is odd, so each store covers all eight 16-byte bank groups.
        {
            uint4 h0, l0, h1, l1;
            split2(kd0[0], kd0[1], h0.x, l0.x); split2(kd0[2], kd0[3], h0.y, l0.y);
            split2(kd0[4], kd0[5], h0.z, l0.z); split2(kd0[6], kd0[7], h0.w, l0.w);
            split2(kd1[0], kd1[1], h1.x, l1.x); split2(kd1[2], kd1[3], h1.y, l1.y);
            split2(kd1[4], kd1[5], h1.z, l1.z); split2(kd1[6], kd1[7], h1.w, l1.w);
            const bool odd_first = (lane >> 2) & 1;
            const uint32_t oa = sw128_chunk(kc + (odd_first ? 1 : 0), r0, 64);
            const uint32_t ob = sw128_chunk(kc + (odd_first ? 0 : 1), r0, 64);
            *reinterpret_cast<uint4*>(sm + kKdStage + oa) = odd_first ? h1 : h0;
            *reinterpret_cast<uint4*>(sm + kKdStage + 8192 + oa) = odd_first ? l1 : l0;
            *reinterpret_cast<uint4*>(sm + kKdStage + ob) = odd_first ? h0 : h1;
            *reinterpret_cast<uint4*>(sm + kKdStage + 8192 + ob) = odd_first ? l0 : l1;
        }
        if (hr == 0) load_kq(1);   // in flight during this round's MMA
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == 0) {
            mma3(tbase, smem_u32(sm + kAKQh), smem_u32(sm + kAKQl), 128, smem_u32(sm + kKFh), smem_u32(sm + kKFl),
                 160, false, 4, idesc_bf16_f32(128, 160), hr > 0);
            mma_commit(&mbar);
            bulk_s2g(out + kOffKdTh + 64 * hr * 128, sm + kKdStage, 8192);
            bulk_s2g(out + kOffKdTl + 64 * hr * 128, sm + kKdStage + 8192, 8192);
            bulk_commit();
        }
        if (!mbar_wait(&mbar, phase)) {
            record_error(err, KDA_ERR_TIMEOUT);
            atomicExch(&sflags[1], 1u);
        }
        if (tid == 0) bulk_wait_read_all();   // the stage is rewritten next round (or by [T ; P T])
        phase ^= 1;
        tc_fence_after();
        __syncthreads();
        if (sflags[1]) {
            abort = true;
            break;
        }
    }

    float* As = reinterpret_cast<float*>(sm + kAs);
    float* Ts = reinterpret_cast<float*>(sm + kTs);
    float* scr = reinterpret_cast<float*>(sm + kScr);
    if (!abort) {
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
            const int col0 = cbeg + 16 * gi;
            tmem_ld16(tmem_addr(tbase, 32 * sp, col0), vals);
            tmem_ld_wait();
            const int i0 = col0 - kf_off(R);              // multiple of 16
            if (i0 < 0 || i0 >= 16 * R + 16) continue;    // another block's version
            if (!is_p) {
#pragma unroll
                for (int e = 0; e < 16; ++e) As[r * kAS + i0 + e] = (i0 + e < r) ? br * vals[e] : 0.f;
                if (at_store) {   // the backward pass: the key products before the beta scaling
                    float* dst = at_store + ((size_t)chunk * H + h) * (kC * kC) + r * kC + i0;
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4*>(dst + e) =
                            make_float4((i0 + e < r) ? vals[e] : 0.f, (i0 + e + 1 < r) ? vals[e + 1] : 0.f,
                                        (i0 + e + 2 < r) ? vals[e + 2] : 0.f, (i0 + e + 3 < r) ? vals[e + 3] : 0.f);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) vals[e] = (i0 + e <= r) ? vals[e] : 0.f;
                store8_split(sm + kPh, sm + kPl, sw128_chunk(r, i0, 64), vals);
                store8_split(sm + kPh, sm + kPl, sw128_chunk(r, i0 + 8, 64), vals + 8);
            }
        }
        if (warp < 4) {
            const float zero[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int i = 16 * R + 16; i < 64; i += 8) {
                if (!is_p) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) As[r * kAS + i + e] = 0.f;
                    if (at_store) {
                        float* dst = at_store + ((size_t)chunk * H + h) * (kC * kC) + r * kC + i;
                        *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
                        *reinterpret_cast<float4*>(dst + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                } else {
                    store8_split(sm + kPh, sm + kPl, sw128_chunk(r, i, 64), zero);
                }
            }
        }
    }
    __syncthreads();

    // ---- diagonal blocks with a large decay range: pairwise on CUDA cores ----------
    // Block R's 16 rows are staged in shared memory (k and q in fp32, normalised
    // when asked, and each token's decay alpha = exp(log alpha) per channel).  Warp w
    // forms the 17 pairs (r, i <= r) of rows w and 15 - w, each lane over 4 channels,
    // walking i down from r: the factor prod_{i < j <= r} alpha_j, carried already
    // multiplied into k_r and q_r, starts at 1 on the diagonal and takes one more
    // alpha per step.  A block so costs one exponential per (row, channel) instead of
    // one per (pair, channel), and each factor carries at most 15 roundings (the
    // difference of two cumulative sums would carry their absolute error, up to
    // 16 |log alpha| ulps, into the exponent).  The 34 per-lane sums (A and P of each
    // pair) are reduced across the warp by halving exchanges, after which lane l
    // holds sum number l.
    if (!abort && fbmask) {
        float* fk = reinterpret_cast<float*>(sm + kFbStage);   // [16][128] k
        float* fq = fk + 16 * 128;                              // [16][128] q
        float* fa = fq + 16 * 128;                              // [16][128] alpha
        // thread: one row, 8 consecutive channels of k, q and log alpha; the next
        // flagged block's are loaded while the current one's pairs are formed
        const int frow = tid >> 4, fc8 = (tid & 15) * 8;
        uint4 nk8, nq8, nl8;
        auto fetch = [&](int Rf) {
            const int rr = 16 * Rf + frow;
            nk8 = nq8 = nl8 = make_uint4(0u, 0u, 0u, 0u);
            if (rr < len) {
                const size_t off = ((size_t)(tok0 + rr) * H + h) * kD + fc8;
                nk8 = *reinterpret_cast<const uint4*>(k + off);
                nq8 = *reinterpret_cast<const uint4*>(q + off);
                nl8 = *reinterpret_cast<const uint4*>(la + off);
            }
        };
        int R = __ffs(fbmask) - 1;
        fetch(R);
        while (R < 4) {
            {
                const int rr = 16 * R + frow;
                const float2 sk = PREP ? make_float2(inv_nk[rr], inv_nk[rr]) : make_float2(1.f, 1.f);
                const float2 sq = PREP ? make_float2(inv_nq[rr], inv_nq[rr]) : make_float2(1.f, 1.f);
                const uint32_t kw[4] = {nk8.x, nk8.y, nk8.z, nk8.w}, qw[4] = {nq8.x, nq8.y, nq8.z, nq8.w};
                const uint32_t lw[4] = {nl8.x, nl8.y, nl8.z, nl8.w};
                float* dk_ = fk + frow * 128 + fc8;
                float* dq_ = fq + frow * 128 + fc8;
                float* da_ = fa + frow * 128 + fc8;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    *reinterpret_cast<float2*>(dk_ + 2 * m) = mul2(unpack_bf16x2(kw[m]), sk);
                    *reinterpret_cast<float2*>(dq_ + 2 * m) = mul2(unpack_bf16x2(qw[m]), sq);
                    // rows past the end are never a factor of a kept pair
                    const float2 l2 = prep_log_alpha2(unpack_bf16x2(lw[m]), prep);
                    *reinterpret_cast<float2*>(da_ + 2 * m) =
                        make_float2(ex2_approx(l2.x * kLog2e), ex2_approx(l2.y * kLog2e));
                }
            }
            const unsigned rest = fbmask & ~((2u << R) - 1u);
            const int Rn = rest ? __ffs(rest) - 1 : 4;
            if (Rn < 4) fetch(Rn);
            __syncthreads();
            {
                const int ra = warp, rb = 15 - warp;
                // the two rows' values, read once; the pairs select between them
                const float4 kra = *reinterpret_cast<const float4*>(fk + ra * 128 + 4 * lane);
                const float4 qra = *reinterpret_cast<const float4*>(fq + ra * 128 + 4 * lane);
                const float4 krb = *reinterpret_cast<const float4*>(fk + rb * 128 + 4 * lane);
                const float4 qrb = *reinterpret_cast<const float4*>(fq + rb * 128 + 4 * lane);
                float v[34];
                // k_r and q_r times the decay from row r down to token i: the diagonal
                // pair starts them at k_r, q_r and every later pair of the row multiplies
                // in one more alpha (warp w's rows switch after pair w, a uniform branch)
                float4 fA = kra, fP = qra;
#pragma unroll
                for (int jj = 0; jj < 17; ++jj) {
                    // pair jj: row ra with i = ra - jj, then row rb with i = 16 - jj
                    const bool first = jj < 8 && jj <= ra;
                    const int i = first ? ra - jj : 16 - jj;
                    if (jj > 0) {
                        // the row switch is a select (8 per pair of the first 8): a branch here
                        // keeps the compiler from overlapping consecutive pairs
                        const bool sw = jj <= 8 && jj == ra + 1;
                        const float4 ai = *reinterpret_cast<const float4*>(fa + min(i + 1, 15) * 128 + 4 * lane);
                        const float2 a01 = make_float2(ai.x, ai.y), a23 = make_float2(ai.z, ai.w);
                        const float2 A01 = mul2(make_float2(fA.x, fA.y), a01), A23 = mul2(make_float2(fA.z, fA.w), a23);
                        const float2 P01 = mul2(make_float2(fP.x, fP.y), a01), P23 = mul2(make_float2(fP.z, fP.w), a23);
                        fA = sw ? krb : make_float4(A01.x, A01.y, A23.x, A23.y);
                        fP = sw ? qrb : make_float4(P01.x, P01.y, P23.x, P23.y);
                    }
                    const float4 ki = *reinterpret_cast<const float4*>(fk + i * 128 + 4 * lane);
                    float2 a2 = mul2(make_float2(ki.x, ki.y), make_float2(fA.x, fA.y));
                    float2 p2 = mul2(make_float2(ki.x, ki.y), make_float2(fP.x, fP.y));
                    a2 = fma2(make_float2(ki.z, ki.w), make_float2(fA.z, fA.w), a2);
                    p2 = fma2(make_float2(ki.z, ki.w), make_float2(fP.z, fP.w), p2);
                    v[2 * jj] = a2.x + a2.y;
                    v[2 * jj + 1] = p2.x + p2.y;
                }
                // values 0-31: halving exchanges (distance 16 .. 1); lane l ends with sum l
#pragma unroll
                for (int w = 16; w >= 1; w >>= 1) {
                    const bool up = (lane & w) != 0;
#pragma unroll
                    for (int m = 0; m < w; ++m) {
                        const float keep = selp(up, v[m + w], v[m]);
                        const float give = selp(up, v[m], v[m + w]);
                        v[m] = keep + __shfl_xor_sync(0xffffffffu, give, w);
                    }
                }
                // values 32, 33 (the last pair: row rb with itself)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    v[32] += __shfl_xor_sync(0xffffffffu, v[32], o);
                    v[33] += __shfl_xor_sync(0xffffffffu, v[33], o);
                }
                auto put = [&](int jj, bool is_p, float val) {
                    const bool first = jj <= ra;
                    const int r = first ? ra : rb, i = first ? ra - jj : 16 - jj;
                    const int row = 16 * R + r, col = 16 * R + i;
                    if (!is_p) {
                        As[row * kAS + col] = (i < r && row < len) ? sbeta[row] * val : 0.f;
                        if (at_store)
                            at_store[((size_t)chunk * H + h) * (kC * kC) + row * kC + col] =
                                (i < r && row < len) ? val : 0.f;
                    } else {
                        __nv_bfloat16 ph, pl;
                        split1(row < len ? val : 0.f, ph, pl);
                        *reinterpret_cast<__nv_bfloat16*>(sm + kPh + sw128_offset(row, col, 64)) = ph;
                        *reinterpret_cast<__nv_bfloat16*>(sm + kPl + sw128_offset(row, col, 64)) = pl;
                    }
                };
                put(lane >> 1, lane & 1, v[0]);
                if (lane == 0) {
                    put(16, false, v[32]);
                    put(16, true, v[33]);
                }
            }
            __syncthreads();
            R = Rn;
        }
    }

    // ---- P (hi/lo image, complete after the fallback) to the workspace ---------------
    // The output's intra-chunk term P W is formed by the state carry, which knows W.
    fence_async_smem();
    __syncthreads();
    if (tid == 0 && !abort) {
        bulk_s2g(out + kOffPh, sm + kPh, 8192);
        bulk_s2g(out + kOffPl, sm + kPl, 8192);
        bulk_commit();
    }
    // v and k for the [beta V | beta K exp(g)] operand are read again (from L2)
    // while T is solved, and g comes back from TMEM, so that no per-row state stays
    // in registers through the middle of the kernel.
    uint32_t vv[8][2], kx[8][2];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int r = r0 + j;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            vv[j][hh] = kx[j][hh] = 0u;
            if (r < len && !abort) {
                const size_t off = ((size_t)(tok0 + r) * H + h) * kD + 64 * hh + kc;
                vv[j][hh] = *reinterpret_cast<const uint32_t*>(v + off);
                kx[j][hh] = *reinterpret_cast<const uint32_t*>(k + off);
            }
        }
    }

    // ---- T = (I + A)^{-1}: diagonal 16 x 16 blocks, then by block distance -----------
    if (!abort) {
        if (warp < 4) {
            // inverse of the unit lower-triangular diagonal block K = warp by
            // right-looking elimination: lane = (row rr, column half hc); pivot row i
            // is final after step i - 1 and reaches the rows below by shuffles
            const int K = warp, rr = lane & 15, hc = lane >> 4;
            float arow[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) arow[i] = As[(16 * K + rr) * kAS + 16 * K + i];   // zero for i >= rr
            float t[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) t[c] = (8 * hc + c == rr) ? 1.f : 0.f;
#pragma unroll
            for (int i = 0; i < 15; ++i)
#pragma unroll
                for (int c = 0; c < 8; ++c) t[c] = fmaf(-arow[i], __shfl_sync(0xffffffffu, t[c], i + 16 * hc), t[c]);
            float* trow = Ts + (16 * K + rr) * kTS + 16 * K + 8 * hc;
            reinterpret_cast<float4*>(trow)[0] = make_float4(t[0], t[1], t[2], t[3]);
            reinterpret_cast<float4*>(trow)[1] = make_float4(t[4], t[5], t[6], t[7]);
        }
        __syncthreads();
        // off-diagonal blocks, column by column (columns of T are independent):
        // T_RI = -T_RR sum_{I <= J < R} A_RJ T_JI for R = I+1 .. 3, one warp per
        // slice of a block column, so the levels need only warp-level syncs.
        // Warps 0-3: block column 0 (4 columns each), 4-5: block column 1 and
        // 6-7: block column 2 (8 columns each).
        float* Yw = scr + warp * 128;   // [16][8] per warp
        if (warp < 4)
            tsolve_cols<2>(As, Ts, Yw, 0, 4 * warp, lane);
        else   // one inlined copy for both block columns
            tsolve_cols<4>(As, Ts, Yw, warp < 6 ? 1 : 2, warp < 6 ? 16 + 8 * (warp - 4) : 32 + 8 * (warp - 6), lane);
        __syncthreads();
        // for the backward pass: T itself, fp32 [64][64] per (chunk, head)
        if (t_store) {
            float* dst = t_store + ((size_t)chunk * H + h) * (kC * kC);
            for (int e = tid; e < kC * kC / 4; e += kIntraThreads) {
                const int rr = e >> 4, c4 = (e & 15) * 4;
                const float4 x = ((c4 >> 4) <= (rr >> 4)) ? *reinterpret_cast<const float4*>(Ts + rr * kTS + c4)
                                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4*>(dst + rr * kC + c4) = x;
            }
        }
        // T (hi/lo) as a K-major tile; blocks above the diagonal are zero
        for (int e = tid; e < 64 * 8; e += kIntraThreads) {
            const int rr = e >> 3, k8 = (e & 7) * 8;
            float t8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if ((k8 >> 4) <= (rr >> 4)) {
                const float4 x0 = *reinterpret_cast<const float4*>(Ts + rr * kTS + k8);
                const float4 x1 = *reinterpret_cast<const float4*>(Ts + rr * kTS + k8 + 4);
                t8[0] = x0.x; t8[1] = x0.y; t8[2] = x0.z; t8[3] = x0.w;
                t8[4] = x1.x; t8[5] = x1.y; t8[6] = x1.z; t8[7] = x1.w;
            }
            store8_split(sm + kTPh, sm + kTPl, sw128_chunk(rr, k8, 128), t8);
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (tid == 0) bulk_wait_read_all();   // P has left shared memory (the operand below overwrites it)
    __syncthreads();

    if (!abort) {
        // ---- [beta V | beta K exp(g)] (MN-major, 64 token rows x 256 columns) ----------
        // first beta V (columns 0-127), whose product starts while beta K exp(g) is built
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = r0 + j;
            const float2 b2 = make_float2(sbeta[r], sbeta[r]);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float2 vb = mul2(b2, unpack_bf16x2(vv[j][hh]));
                store2_split(sm + kXh, sm + kXl, mn_offset(r, 64 * hh + kc, 64), vb.x, vb.y);
            }
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- [U | Wk] = T [beta V | beta K exp(g)]  (M = 64), in two halves -----------------
    const uint32_t tp_h = smem_u32(sm + kTPh), tp_l = smem_u32(sm + kTPl);
    const uint32_t x_h = smem_u32(sm + kXh), x_l = smem_u32(sm + kXl);
    if (tid == 0 && !abort) {
        mma3(tmem_addr(tbase, 0, 0), tp_h, tp_l, 64, x_h, x_l, 64, true, kC / 16, idesc_bf16_f32_bmn(64, 128),
             false);
        mma_commit(&mbar);
    }
    if (!abort) {
        float gs[2][16];
        tmem_st_wait();
        tmem_ld16(t_g, gs[0]);
        tmem_ld16(t_g + 16, gs[1]);
        tmem_ld_wait();
        const float2 zero2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int r = r0 + j;
            const float2 b2 = make_float2(sbeta[r], sbeta[r]);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const float2 gj = make_float2(gs[j >> 2][4 * (j & 3) + 2 * hh], gs[j >> 2][4 * (j & 3) + 2 * hh + 1]);
                float2 kn = unpack_bf16x2(kx[j][hh]);
                if (PREP) kn = mul2(kn, make_float2(inv_nk[r], inv_nk[r]));
                const float2 kb = mul2(mul2(b2, kn), exp_diff2(gj, zero2));
                store2_split(sm + kXh, sm + kXl, mn_offset(r, 128 + 64 * hh + kc, 64), kb.x, kb.y);
            }
        }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0 && !abort) {
        mma3(tmem_addr(tbase, 0, 128), tp_h, tp_l, 64, x_h + 16384, x_l + 16384, 64, true, kC / 16,
             idesc_bf16_f32_bmn(64, 128), false);
        mma_commit(&mbar_k);
    }
    // both halves: the epilogue reuses the operand space as its staging area
    if (!abort && (!mbar_wait(&mbar, phase) || !mbar_wait(&mbar_k, 0))) {
        record_error(err, KDA_ERR_TIMEOUT);
        atomicExch(&sflags[1], 1u);
    }
    tc_fence_after();
    __syncthreads();
    abort = abort || sflags[1] != 0;

    // ---- epilogue: U (fp32) and Wk (hi/lo) ----------------------------------------------
    // M = 64 results: row r sits in TMEM lane 32 (r / 16) + r % 16, so warp w
    // (sub-partition w % 4) holds rows 16 (w % 4) .. + 15 in its lanes 0-15; the two
    // warp groups take 64 of the 128 columns of each part.  Rows go to
    // shared-memory copies of the workspace images (free after the last MMA) and
    // leave in whole bulk copies: a row per thread written straight to global
    // memory would put each warp store into 16 different lines.
    if (!abort) {
        uint8_t* st_u = sm;                    // U (32 KB, same bytes as the workspace)
        uint8_t* st_w = sm + 32768;            // Wk hi, K blocks 0 and 1 (8 KB each), then lo
        const int sp = warp & 3;
        const int r = 16 * sp + (lane & 15);
        const bool row_lane = lane < 16;
        const int cg = (warp >> 2) * 64;
        float* uo = reinterpret_cast<float*>(st_u);
#pragma unroll 1
        for (int bt = 0; bt < 2; ++bt) {
            const int j0 = cg + 32 * bt;
            float vals[2][16];
            tmem_ld16(tmem_addr(tbase, 32 * sp, j0), vals[0]);
            tmem_ld16(tmem_addr(tbase, 32 * sp, j0 + 16), vals[1]);
            tmem_ld_wait();
            if (row_lane) {
#pragma unroll
                for (int x = 0; x < 2; ++x)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        *reinterpret_cast<float4*>(uo + u_index(r, j0 + 16 * x + 4 * e)) =
                            make_float4(vals[x][4 * e], vals[x][4 * e + 1], vals[x][4 * e + 2], vals[x][4 * e + 3]);
            }
            tmem_ld16(tmem_addr(tbase, 32 * sp, 128 + j0), vals[0]);
            tmem_ld16(tmem_addr(tbase, 32 * sp, 128 + j0 + 16), vals[1]);
            tmem_ld_wait();
            if (row_lane) {
                uint8_t* wh = st_w + (j0 >> 6) * 8192;
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const int kk = (j0 & 63) + 16 * x;
                    store8_split(wh, wh + 16384, sw128_chunk(r, kk, 64), vals[x]);
                    store8_split(wh, wh + 16384, sw128_chunk(r, kk + 8, 64), vals[x] + 8);
                }
            }
        }
        fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            bulk_s2g(out + kOffU, st_u, 32768);
            // rows 0-63 of each 64-wide K block of the [Wk ; Q exp(g)] hi and lo images
            bulk_s2g(out + kOffWkQh, st_w, 8192);
            bulk_s2g(out + kOffWkQh + 16384, st_w + 8192, 8192);
            bulk_s2g(out + kOffWkQl, st_w + 16384, 8192);
            bulk_s2g(out + kOffWkQl + 16384, st_w + 24576, 8192);
            bulk_commit();
            bulk_wait_read_all();                // shared memory stays valid until read
        }
    }
    tmem_st_wait();   // the g stash has landed (returns at once unless the kernel aborted early)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tbase, 256);
}

// ============================================================================
// tc_recur
// ============================================================================
// 256 threads: warp w reads TMEM lanes 32 (w % 4) .. + 31 and owns the state
// columns [BV/2 (w / 4), BV/2 (w / 4 + 1)) of its rows.  Warps with w % 4 < 2
// form W (rows 0-63 of D); the others finish the outputs.  The output product
// [0 ; P] W of chunk n is issued (by thread 64, after thread 0 has issued chunk
// n + 1's first product) into chunk n's D buffer, and runs on the tensor core
// while the CUDA cores form chunk n + 1's W: D and W alternate between two
// buffers, so nothing on the chain waits for it.
constexpr int kRecurThreads = 256;

template <int BV>
struct RecurLayout {
    static constexpr uint32_t kWkQ = 0;                                        // hi 32 KB + lo 32 KB
    static constexpr uint32_t kKdT = 65536;                                    // hi 16 KB + lo 16 KB
    static constexpr uint32_t kUtile = (uint32_t)BV * 64 * 4;                  // U tile, fp32
    static constexpr uint32_t kUStage = kUtile + 512;                          // U, Gamma_C
    static constexpr uint32_t kUU = 98304;                                     // two U stages
    static constexpr uint32_t kP = (kUU + 2 * kUStage + 1023) / 1024 * 1024;  // [0 ; P] hi 16 KB + lo 16 KB
    static constexpr uint32_t kS = kP + 2 * 16384;                             // S hi/lo: 128 rows x 128 B (MN-major)
    static constexpr uint32_t kW = kS + 2 * 16384;                             // W hi/lo: 64 rows x 128 B (MN-major), x2
    static constexpr uint32_t kBars = kW + 2 * 2 * 8192;
    static constexpr uint32_t kSmem = kBars + 128;
    static constexpr uint32_t kAlloc = kSmem + 1024;
    // The products take [hi | lo] B operands (mma2w): D and S in two column ranges each
    // (D buffers 2 x 2 BV, S 2 BV).  At 64 columns the lo tiles of S and W are the
    // 64-wide blocks after the hi tiles; at 32 the second halves of the same rows.
    static_assert(BV == 32 || BV == 64, "state column tiles of 32 or 64");
    static constexpr uint32_t kCols = 6 * BV;
    static constexpr uint32_t kTmemCols = (kCols <= 32) ? 32 : (kCols <= 64) ? 64 : (kCols <= 128) ? 128
                                                       : (kCols <= 256) ? 256 : 512;
};

// MODE 0: the prefill.  MODE 1 (for the backward pass): also every chunk's start
// state S_n to s_store [chunks, H, 128, 128] and W_n to w_store [tokens, H, 128],
// both fp32.  MODE 2 (a segment's affine map S_end = M S_start + F, for splitting
// one sequence over several devices): no outputs; the first 128 / BV column tiles
// carry the state from zero (F, written to final_state), the next 128 / BV carry
// the columns of the identity with the values' term U left out (M, written to
// s_store as [N, H, 128, 128]).
template <int BV, int MODE>
__global__ void __launch_bounds__(kRecurThreads, 1)
tc_recur(const uint8_t* __restrict__ ws, const float* __restrict__ init_state, float* __restrict__ final_state,
         __nv_bfloat16* __restrict__ o, int* __restrict__ err, SeqMap smap, int H, float* __restrict__ s_store,
         float* __restrict__ w_store, unsigned long long stall_ns) {
    constexpr bool STORE = MODE == 1, MAP = MODE == 2;
    using Lay = RecurLayout<BV>;
    constexpr int HB = BV / 2;          // state columns per thread
    constexpr int NG = HB / 16;         // 16-column TMEM groups per thread
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, formed as an offset from the shared array so that every
    // access through it stays a shared-memory access (32-bit addressing)
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Lay::kBars);
    uint64_t* wkq_full = bars + 0;
    uint64_t* kdt_full = bars + 1;
    uint64_t* uu_full = bars + 2;     // [2]
    uint64_t* bar_d = bars + 4;       // D = [Wk ; Q exp(g)] S done
    uint64_t* bar_s = bars + 5;       // S update done
    uint64_t* bar_o = bars + 6;       // D += [0 ; P] W done (outputs ready)
    uint64_t* p_full = bars + 7;      // P landed
    uint64_t* d_issued = bars + 8;    // the chunk's first product has been issued
    uint32_t* sflags = reinterpret_cast<uint32_t*>(bars + 9);        // [0] tmem base, [1] abort
    uint64_t* never = bars + 10;      // completed by nothing (failure test)
    uint8_t* s_h = sm + Lay::kS;
    uint8_t* s_l = s_h + 16384;
    auto w_hi = [&](int n) { return sm + Lay::kW + (n & 1) * 16384; };   // lo parts 8 KB further

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int sp = warp & 3;            // TMEM sub-partition: lanes 32 sp .. 32 sp + 31
    const int cq = (warp >> 2) * HB;    // first state column of this thread (relative to j0)
    // grid order: column tile fastest, then head, then sequence (longest first), so
    // that the tiles of one (sequence, head) run side by side and read its
    // workspace images from L2 after the first of them has brought them in
    constexpr int kTiles = (MAP ? 2 : 1) * (kD / BV);
    const int z = (int)(blockIdx.x % kTiles);
    const int h = (int)((blockIdx.x / kTiles) % (unsigned)H);
    const SeqInfo sq = smap.get((int)(blockIdx.x / (kTiles * (unsigned)H)));
    const bool mcols = MAP && z >= kD / BV;      // a tile of M: identity start, no U term
    const int j0 = (mcols ? z - kD / BV : z) * BV;
    const int nch = (sq.len + kC - 1) / kC;
    const int cb0 = j0 / 32;   // first 32-column block of U

    if (tid == 0) {
        for (int i = 0; i < 9; ++i) mbar_init(&bars[i], 1);
        mbar_init(never, 1);
        sflags[1] = 0;
        mbar_init_fence();
    }
    if (warp == 0) {
        tmem_alloc(&sflags[0], Lay::kTmemCols);
        tmem_relinquish();
    }
    // rows 0-63 of the [0 ; P] operand are zero (hi and lo)
    for (int i = tid; i < 1024; i += kRecurThreads) {
        const int img = i >> 9, off = (i & 511) * 16;
        *reinterpret_cast<uint4*>(sm + Lay::kP + img * 16384 + off) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = sflags[0];
    // D of chunk n: columns [DW (n % 2), + DW); S: from 2 DW.  D and S are each the sum
    // of two BV-column ranges (the A_hi B_lo term of the products in the second).
    constexpr uint32_t DW = 2 * BV;
    const uint32_t t_s = tbase + 2 * DW;
    auto t_dbuf = [&](int m) { return tbase + (uint32_t)(DW * (m & 1)); };
    // 16 columns of D or S at column offset col: the sum of the two ranges
    auto ld_sum16 = [&](uint32_t t, int col, float (&v)[16]) {
        float w[16];
        tmem_ld16(tmem_addr(t, 32 * sp, col), v);
        tmem_ld16(tmem_addr(t, 32 * sp, BV + col), w);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] += w[e];
    };

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
        bulk_g2s(dst + Lay::kUtile, src + kOffGam, 512, &uu_full[stage]);
    };
    auto load_p = [&](int n) {   // P into rows 64-127 of the [0 ; P] hi and lo tiles
        const uint8_t* src = chunk_src(n);
        mbar_arrive_expect_tx(p_full, 16384);
        bulk_g2s(sm + Lay::kP + 8192, src + kOffPh, 8192, p_full);
        bulk_g2s(sm + Lay::kP + 16384 + 8192, src + kOffPl, 8192, p_full);
    };
    auto fail = [&]() {
        record_error(err, KDA_ERR_TIMEOUT);
        atomicExch(&sflags[1], 1u);
    };
    if (tid == 0 && nch > 0) {
        load_wkq(0);
        load_kdt(0);
        load_uu(0, 0);
        if (!MAP) load_p(0);
        if (nch > 1) load_uu(1, 1);
    }

    // this thread's state row c, columns j0 + cq + [0, HB)
    const int c = 32 * sp + lane;
    float s[HB];
    {
        const size_t base = (((size_t)sq.seq * H + h) * kD + c) * kD + j0 + cq;
#pragma unroll
        for (int j = 0; j < HB; j += 4) {
            float4 x = (!MAP && init_state) ? *reinterpret_cast<const float4*>(init_state + base + j)
                                            : make_float4(0.f, 0.f, 0.f, 0.f);
            s[j] = x.x; s[j + 1] = x.y; s[j + 2] = x.z; s[j + 3] = x.w;
        }
        if (mcols) {
#pragma unroll
            for (int j = 0; j < HB; ++j) s[j] = (c == j0 + cq + j) ? 1.f : 0.f;
        }
    }

    // D(m) += [0 ; P] W(m): the output product of chunk m (thread 64)
    auto issue_o = [&](int m) {
        if (!mbar_wait(p_full, (uint32_t)m & 1u)) {
            fail();
        } else {
            const uint32_t a = smem_u32(sm + Lay::kP);
            const uint32_t wh = smem_u32(w_hi(m));
            mma2w(t_dbuf(m), a, a + 16384, 128, wh, 64, kC / 16, idesc_bf16_f32_bmn(128, 2 * BV),
                  idesc_bf16_f32_bmn(128, BV), true);
        }
        mma_commit(bar_o);
    };
    // O rows of chunk m out of D (warps with sp >= 2: rows 64-127 = token rows 0-63)
    auto emit_o = [&](int m) {
        const uint32_t t_d = t_dbuf(m);
        float d[NG][16];
#pragma unroll
        for (int g = 0; g < NG; ++g) ld_sum16(t_d, cq + 16 * g, d[g]);
        tmem_ld_wait();
        const int r = c - 64;
        if (r < min(kC, sq.len - m * kC)) {
            __nv_bfloat16* dst = o + ((size_t)(sq.tok0 + m * kC + r) * H + h) * kD + j0 + cq;
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                uint4 w0, w1;
                w0.x = pack_bf16(d[g][0], d[g][1]); w0.y = pack_bf16(d[g][2], d[g][3]);
                w0.z = pack_bf16(d[g][4], d[g][5]); w0.w = pack_bf16(d[g][6], d[g][7]);
                w1.x = pack_bf16(d[g][8], d[g][9]); w1.y = pack_bf16(d[g][10], d[g][11]);
                w1.z = pack_bf16(d[g][12], d[g][13]); w1.w = pack_bf16(d[g][14], d[g][15]);
                reinterpret_cast<uint4*>(dst + 16 * g)[0] = w0;
                reinterpret_cast<uint4*>(dst + 16 * g)[1] = w1;
            }
        }
    };

    int n = 0;
    for (; n < nch; ++n) {
        const int stage = n & 1;
        const uint8_t* uu = sm + Lay::kUU + stage * Lay::kUStage;
        const uint32_t par = (uint32_t)n & 1u;
        const uint32_t t_d = t_dbuf(n);
        if (STORE) {
            float* dst = s_store + ((((size_t)sq.chunk0 + n) * H + h) * kD + c) * kD + j0 + cq;
#pragma unroll
            for (int j = 0; j < HB; j += 4)
                *reinterpret_cast<float4*>(dst + j) = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
        }
        // S_n as the MN-major B operand (K = channel row c, N = columns), hi and lo tiles
#pragma unroll
        for (int j = 0; j < HB; j += 8)
            store8_split2(s_h, mn_chunk(c, cq + j, 128), BV == 32 ? s_h : s_l,
                          mn_chunk(c, (BV == 32 ? 32 : 0) + cq + j, 128), s + j);
        if (!mbar_wait(&uu_full[stage], (uint32_t)(n >> 1) & 1u)) fail();
        // Diag(Gamma_C) S_n into TMEM; the S update accumulates on top of it
        const float gam = reinterpret_cast<const float*>(uu + Lay::kUtile)[c];
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            float t[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) t[e] = gam * s[16 * g + e];
            tmem_st16(tmem_addr(t_s, 32 * sp, cq + 16 * g), t);
            // the second range starts from zero (one accumulate flag covers both)
#pragma unroll
            for (int e = 0; e < 16; ++e) t[e] = 0.f;
            tmem_st16(tmem_addr(t_s, 32 * sp, BV + cq + 16 * g), t);
        }
        tmem_st_wait();
        // test of the failure path (stall_ns != 0): the first CTA waits, bounded, on a
        // barrier that nothing completes before its first product, then aborts
        if (stall_ns != 0ull && n == 0 && blockIdx.x == 0 && tid == 0 && !mbar_wait(never, 0, stall_ns)) fail();
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (sflags[1]) break;
        tc_fence_after();
        if (tid == 0) {
            if (!mbar_wait(wkq_full, par)) {
                fail();
            } else {
                const uint32_t a = smem_u32(sm + Lay::kWkQ);
                mma2w(t_d, a, a + 32768, 128, smem_u32(s_h), 128, kD / 16, idesc_bf16_f32_bmn(128, 2 * BV),
                      idesc_bf16_f32_bmn(128, BV), false);
            }
            mma_commit(bar_d);
            mbar_arrive(d_issued);   // the previous chunk's output product may follow it
        }
        if (!mbar_wait(bar_d, par)) fail();
        tc_fence_after();
        if (tid == 0 && n + 1 < nch) load_wkq(n + 1);   // the product is done with the buffer
        if (sp < 2) {
            // W = U - Wk S (rows are tokens) -> MN-major B operand of the S update and of [0 ; P] W
            const int r = c;
            const float* ut = reinterpret_cast<const float*>(uu);
            uint8_t* w_h = w_hi(n);
            float d[NG][16];
#pragma unroll
            for (int g = 0; g < NG; ++g) ld_sum16(t_d, cq + 16 * g, d[g]);
            tmem_ld_wait();
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                const int jb = cq + 16 * g;
#pragma unroll
                for (int e = 0; e < 16; e += 4) {
                    const float4 u = mcols ? make_float4(0.f, 0.f, 0.f, 0.f)
                                           : *reinterpret_cast<const float4*>(ut + u_index(r, jb + e));
                    d[g][e] = u.x - d[g][e]; d[g][e + 1] = u.y - d[g][e + 1];
                    d[g][e + 2] = u.z - d[g][e + 2]; d[g][e + 3] = u.w - d[g][e + 3];
                }
                uint8_t* w_l = BV == 32 ? w_h : w_h + 8192;
                const int lc = BV == 32 ? 32 : 0;
                store8_split2(w_h, mn_chunk(r, jb, 64), w_l, mn_chunk(r, lc + jb, 64), d[g]);
                store8_split2(w_h, mn_chunk(r, jb + 8, 64), w_l, mn_chunk(r, lc + jb + 8, 64), d[g] + 8);
                if (STORE && r < min(kC, sq.len - n * kC)) {
                    float* dst = w_store + ((size_t)(sq.tok0 + n * kC + r) * H + h) * kD + j0 + jb;
#pragma unroll
                    for (int e = 0; e < 16; e += 4)
                        *reinterpret_cast<float4*>(dst + e) = make_float4(d[g][e], d[g][e + 1], d[g][e + 2], d[g][e + 3]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            asm volatile("bar.sync 1, 128;" ::: "memory");   // warps 0, 1, 4, 5: W is ready
            tc_fence_after();
            if (tid == 0) {
                if (!mbar_wait(kdt_full, par)) {
                    fail();
                } else {
                    const uint32_t a = smem_u32(sm + Lay::kKdT);
                    mma2w(t_s, a, a + 16384, 128, smem_u32(w_h), 64, kC / 16, idesc_bf16_f32_bmn(128, 2 * BV),
                          idesc_bf16_f32_bmn(128, BV), true);
                }
                mma_commit(bar_s);
            }
        } else if (!MAP && n > 0) {
            // outputs of the previous chunk: its product goes in behind this chunk's
            // first one and runs while W is formed; then its P tile may be replaced
            if (tid == 64) {
                if (!mbar_wait(d_issued, par)) fail();
                issue_o(n - 1);
            }
            if (!mbar_wait(bar_o, par ^ 1u)) {
                fail();
            } else if (tid == 64) {
                load_p(n);
            }
            tc_fence_after();
            emit_o(n - 1);
        }
        if (!mbar_wait(bar_s, par)) fail();
        tc_fence_after();
        if (sp < 2) {
            // the W warps are past their reads of this chunk's U stage (the other warps
            // read only its Gamma, before the barrier ahead of this chunk's first
            // product), so the output warps do not hold the chain up here
            asm volatile("bar.sync 2, 128;" ::: "memory");
            if (tid == 0) {
                if (n + 1 < nch) load_kdt(n + 1);          // the S update is done with Kd^T
                if (n + 2 < nch) load_uu(n + 2, stage);
            }
        }
        {
            float t[NG][16];
#pragma unroll
            for (int g = 0; g < NG; ++g) ld_sum16(t_s, cq + 16 * g, t[g]);
            tmem_ld_wait();
#pragma unroll
            for (int g = 0; g < NG; ++g)
#pragma unroll
                for (int e = 0; e < 16; ++e) s[16 * g + e] = t[g][e];
        }
    }
    __syncthreads();
    const bool failed = sflags[1] != 0;
    if (!MAP && !failed && nch > 0 && sp >= 2) {
        // outputs of the last chunk
        if (tid == 64) issue_o(nch - 1);
        if (!mbar_wait(bar_o, (uint32_t)(nch - 1) & 1u)) fail();
        tc_fence_after();
        emit_o(nch - 1);
    }
    float* fdst = mcols ? s_store : final_state;
    if (!failed && fdst) {
        const size_t base = (((size_t)sq.seq * H + h) * kD + c) * kD + j0 + cq;
#pragma unroll
        for (int j = 0; j < HB; j += 4)
            *reinterpret_cast<float4*>(fdst + base + j) = make_float4(s[j], s[j + 1], s[j + 2], s[j + 3]);
    }
    __syncthreads();
    if (sflags[1] && tid == 0) {
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

template <int BV, int MODE = 0>
cudaError_t launch_recur(const uint8_t* ws, const float* init_state, float* final_state, __nv_bfloat16* o, int* err,
                         const SeqMap& smap, int n_seqs, int H, cudaStream_t stream, float* s_store = nullptr,
                         float* w_store = nullptr, unsigned long long stall_ns = 0ull) {
    using Lay = RecurLayout<BV>;
    cudaError_t e =
        cudaFuncSetAttribute(tc_recur<BV, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::kAlloc);
    if (e != cudaSuccess) return e;
    const unsigned tiles = (MODE == 2 ? 2u : 1u) * (unsigned)(kD / BV);
    tc_recur<BV, MODE><<<dim3((unsigned)(n_seqs * H) * tiles), kRecurThreads, Lay::kAlloc, stream>>>(
        ws, init_state, final_state, o, err, smap, H, s_store, w_store, stall_ns);
    return cudaGetLastError();
}


// multiprocessors of the current device, looked up once per device
int sm_count() {
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

}  // namespace

bool tc_available() { return true; }

// Requests for 64- or 128-token chunks are both served with 64-token chunks.
bool tc_supports(int C) { return C == kC || C == 2 * kC; }
int tc_chunk() { return kC; }

size_t tc_workspace_bytes(int n_chunks, int H, int C) {
    if (C != kC) return 0;
    return kErrHeader + (size_t)n_chunks * H * kChunkBytes;
}

cudaError_t launch_tc_prefill(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                              const float* init_state, void* o, float* final_state, const ChunkMap& cmap,
                              const SeqMap& smap, int n_chunks, int n_seqs, int H, int C, void* tc_ws,
                              unsigned prep, cudaStream_t stream, unsigned long long stall_intra_ns,
                              unsigned long long stall_recur_ns) {
    if (C != kC) return cudaErrorNotSupported;
    int* err = reinterpret_cast<int*>(tc_ws);
    uint8_t* ws = reinterpret_cast<uint8_t*>(tc_ws) + kErrHeader;
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
    if (n_chunks > 0) {
        auto kern = prep ? tc_intra<true> : tc_intra<false>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kIntraAlloc);
        if (e != cudaSuccess) return e;
        kern<<<(unsigned)((long)n_chunks * H), kIntraThreads, kIntraAlloc, stream>>>(
            (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
            (const __nv_bfloat16*)log_alpha, (const __nv_bfloat16*)beta, ws, err, cmap, H, prep, stall_intra_ns, nullptr, nullptr);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    timing_mark(stream, 1);
    if (n_seqs > 0) {
        const long units = (long)n_seqs * H;
        if (units * 4 <= sm_count())
            e = launch_recur<32>(ws, init_state, final_state, (__nv_bfloat16*)o, err, smap, n_seqs, H, stream,
                                 nullptr, nullptr, stall_recur_ns);
        else
            e = launch_recur<64>(ws, init_state, final_state, (__nv_bfloat16*)o, err, smap, n_seqs, H, stream,
                                 nullptr, nullptr, stall_recur_ns);
        if (e != cudaSuccess) return e;
    }
    timing_mark(stream, 2);
    return cudaSuccess;
}

// The forward intermediates the backward pass needs, from the tensor-core path:
// the per-chunk images (read again by the gradient kernels), T and the key
// products, and every chunk's start state and W (fp32, from the state carry).
// o_scratch receives the outputs.
cudaError_t launch_tc_states(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                             const float* init_state, void* o_scratch, const ChunkMap& cmap, const SeqMap& smap,
                             int n_chunks, int n_seqs, int H, void* tc_ws, float* S_chunk, float* W,
                             float* T_store, float* At_store, cudaStream_t stream) {
    int* err = reinterpret_cast<int*>(tc_ws);
    uint8_t* ws = reinterpret_cast<uint8_t*>(tc_ws) + kErrHeader;
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
    if (n_chunks > 0) {
        e = cudaFuncSetAttribute(tc_intra<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kIntraAlloc);
        if (e != cudaSuccess) return e;
        tc_intra<false><<<(unsigned)((long)n_chunks * H), kIntraThreads, kIntraAlloc, stream>>>(
            (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
            (const __nv_bfloat16*)log_alpha, (const __nv_bfloat16*)beta, ws, err, cmap, H, 0u, 0ull, T_store, At_store);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (n_seqs > 0) {
        if ((long)n_seqs * H * 4 <= sm_count())
            e = launch_recur<32, 1>(ws, init_state, nullptr, (__nv_bfloat16*)o_scratch, err, smap, n_seqs, H, stream,
                                    S_chunk, W);
        else
            e = launch_recur<64, 1>(ws, init_state, nullptr, (__nv_bfloat16*)o_scratch, err, smap, n_seqs, H, stream,
                                    S_chunk, W);
    }
    return e;
}

// A segment's affine map (S_end = M S_start + F per sequence and head): the
// chunk-local kernel, then the state carry over 2 x 128 columns (F from a zero
// start, M from the identity without the values' term), no outputs.
cudaError_t launch_tc_segment_map(const void* q, const void* k, const void* v, const void* log_alpha,
                                  const void* beta, const ChunkMap& cmap, const SeqMap& smap, int n_chunks,
                                  int n_seqs, int H, void* tc_ws, float* M, float* F, cudaStream_t stream) {
    int* err = reinterpret_cast<int*>(tc_ws);
    uint8_t* ws = reinterpret_cast<uint8_t*>(tc_ws) + kErrHeader;
    cudaError_t e = cudaMemsetAsync(err, 0, sizeof(int), stream);
    if (e != cudaSuccess) return e;
    if (n_chunks > 0) {
        e = cudaFuncSetAttribute(tc_intra<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kIntraAlloc);
        if (e != cudaSuccess) return e;
        tc_intra<false><<<(unsigned)((long)n_chunks * H), kIntraThreads, kIntraAlloc, stream>>>(
            (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
            (const __nv_bfloat16*)log_alpha, (const __nv_bfloat16*)beta, ws, err, cmap, H, 0u, 0ull, nullptr, nullptr);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    timing_mark(stream, 1);
    if (n_seqs > 0) {
        if ((long)n_seqs * H * 8 <= sm_count())
            e = launch_recur<32, 2>(ws, nullptr, F, nullptr, err, smap, n_seqs, H, stream, M, nullptr);
        else
            e = launch_recur<64, 2>(ws, nullptr, F, nullptr, err, smap, n_seqs, H, stream, M, nullptr);
        if (e != cudaSuccess) return e;
    }
    timing_mark(stream, 2);
    return cudaSuccess;
}

}  // namespace kda
