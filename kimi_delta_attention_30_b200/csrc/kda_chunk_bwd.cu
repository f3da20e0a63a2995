// Chunkwise KDA backward pass (CUDA cores, fp32 arithmetic): the gradients of
// the loss  L = <dO, O> + <dS_final, S_final>  with respect to q, k, v,
// log alpha, beta and the initial state.
//
// The pages say training needs the chunkwise parallel form ("From GPT-2 to
// Kimi K3" essay, pwwt.cn/news/3716252, chunkwise paragraph) but derive no
// backward pass; this one is the chain rule applied to the chunk form that
// the forward kernels compute.  Per chunk, with start state S, cumulative
// decay g (rows r = 0..L-1), Gam = exp(g_{L-1}) and
//   Qg = Q . exp(g),  Kg = K . exp(g),  Kd = K . exp(g_{L-1} - g),
//   At[r][i] = sum_c k_rc k_ic exp(g_rc - g_ic)   (i < r),  A = Diag(beta) At,
//   P[r][i]  = sum_c q_rc k_ic exp(g_rc - g_ic)   (i <= r),
//   U = (I + A)^-1 Diag(beta) V,  Wk = (I + A)^-1 Diag(beta) Kg,  W = U - Wk S,
//   O = Qg S + P W,   S' = Diag(Gam) S + Kd^T W,
// the chunk is affine in S, so the state gradient runs backwards over the
// chunks (kb_chain):
//   dW = P^T dO + Kd dS',    dS = Diag(Gam) dS' + Qg^T dO - Wk^T dW,
// and everything else is chunk-parallel (kb_a, kb_b, kb_c):
//   dQg = dO S^T, dKd = W dS'^T, dWk = -dW S^T, dGam = rowsum(dS' . S),
//   dP = dO W^T (i <= r),
//   [Y | Z] = (I + A)^-T [dW | dWk]           (back substitution),
//   dv = Diag(beta) Y,  dKg = Diag(beta) Z,
//   dA = -(Y U^T + Z Wk^T) (i < r),  dAt = Diag(beta) dA,
//   dbeta_r = v_r.Y_r + Kg_r.Z_r + sum_i dA_ri At_ri,
// then the pairwise terms of At and P give dq and dk (with E = exp(g_r - g_i)),
// the elementwise factors add theirs, and dlog alpha sums, for each token j,
// exactly the terms whose decay spans it (see kb_c).
// Every decay is exp of a non-positive difference, as in the forward split, of
// cumulative decays held as fp32 (hi, lo) pairs (exp_gdiff, exp_g).
// The forward intermediates (g, U, Wk, W, chunk start states) are recomputed by
// the tensor-core forward (bf16, d = 128; g by the CUDA-core K1) or by the
// CUDA-core forward kernels.
#include <algorithm>
#include <type_traits>

#include "kda_internal.cuh"

namespace kda {
namespace {

constexpr int kT = 256;
constexpr int kTW = 512;      // kb_chain: more warps to hide latency
constexpr int kBV = 32;       // d_v columns per chain block / per tile
constexpr int kBP = kBV + 1;  // padded row stride of the d_v tiles

constexpr int kBwdC = 64;     // the backward kernels tile by 64 tokens

__device__ __forceinline__ float wsum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

__device__ __forceinline__ size_t tok_off(int t, int H, int h, int d) { return ((size_t)t * H + h) * d; }

// Four consecutive elements as fp32 (8 bytes of bf16 or 16 bytes of fp32, aligned).
__device__ __forceinline__ void load4(const float* p, float* v) {
    const float4 x = *reinterpret_cast<const float4*>(p);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
__device__ __forceinline__ void load4(const __nv_bfloat16* p, float* v) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);   // element 0 in the low half of u.x
    v[0] = __uint_as_float(u.x << 16); v[1] = __uint_as_float(u.x & 0xffff0000u);
    v[2] = __uint_as_float(u.y << 16); v[3] = __uint_as_float(u.y & 0xffff0000u);
}

constexpr int kPThreads = 544;   // kb_p: 136 tiles x 4 lanes = 17 warps
constexpr int kPS = 68;          // row stride of kb_p's channel-major arrays (float4-aligned)

// P[r][i] = sum_c q_rc k_ic exp(g_rc - g_ic) for i <= r < L and At[r][i] (the same
// with k_r, i < r), zero elsewhere, from one exponential per (r, i, c); and the
// elementwise Qg = q exp(g), Kd = k exp(g_C - g) the chain and the later kernels read.
// One block per (chunk, head).  The lower triangle of the 64 x 64 pair grid is
// cut into 136 tiles of 4 x 4 pairs (rows 4a..4a+3, columns 4b..4b+3, b <= a);
// four adjacent lanes share a tile, lane s summing the channels s, s + 4, ...,
// and two shuffles add their partial sums.  Shared memory holds q, k, g and its
// low part channel-major ([c][r], row stride kPS), so a lane reads the four rows
// (or columns) of its tile for one channel as one float4.  Rows past the end of
// a short chunk hold q = k = 0 and the last row's g, which keeps every exponent
// of a pair i <= r non-positive; their outputs are written as zero, as are the
// pairs i > r of the diagonal tiles (computed, then discarded).
template <typename Tin, int DK>
__global__ void __launch_bounds__(kPThreads, 1) kb_p(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                     const float* __restrict__ g, const float* __restrict__ gl,
                                                     float* __restrict__ P, float* __restrict__ At,
                                                     float* __restrict__ Qg, float* __restrict__ Kd, ChunkMap cmap,
                                                     int H) {
    constexpr int C = kBwdC;
    extern __shared__ __align__(16) float smem[];
    float* Qt = smem;
    float* Kt = Qt + DK * kPS;
    float* Gt = Kt + DK * kPS;
    float* GLt = Gt + DK * kPS;
    int seq, tok0, len, idx;
    cmap.locate(blockIdx.x, seq, tok0, len, idx);
    const int h = blockIdx.y, tid = threadIdx.x;

    // Staging in groups of 4 channels.  A warp covers 16 rows x 2 groups, so the
    // transposed shared stores of its lanes fall in 32 different banks.
    const size_t last = tok_off(tok0 + len - 1, H, h, DK);
    for (int e4 = tid; e4 < C * DK / 4; e4 += kPThreads) {
        const int w = e4 >> 5, ln = e4 & 31;
        const int r = (ln & 15) + 16 * (w & 3);
        const int c = 4 * (2 * (w >> 2) + (ln >> 4));
        float gL[4], lL[4], gv[4], lv[4], qv[4] = {0.f, 0.f, 0.f, 0.f}, kv[4] = {0.f, 0.f, 0.f, 0.f};
        load4(g + last + c, gL);
        load4(gl + last + c, lL);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            gv[u] = gL[u];
            lv[u] = lL[u];
        }
        if (r < len) {
            const size_t off = tok_off(tok0 + r, H, h, DK) + c;
            load4(q + off, qv);
            load4(k + off, kv);
            load4(g + off, gv);
            load4(gl + off, lv);
            float4 qg, kd;
            qg.x = qv[0] * exp_g(gv[0], lv[0]);
            qg.y = qv[1] * exp_g(gv[1], lv[1]);
            qg.z = qv[2] * exp_g(gv[2], lv[2]);
            qg.w = qv[3] * exp_g(gv[3], lv[3]);
            kd.x = kv[0] * exp_gdiff(gL[0], lL[0], gv[0], lv[0]);
            kd.y = kv[1] * exp_gdiff(gL[1], lL[1], gv[1], lv[1]);
            kd.z = kv[2] * exp_gdiff(gL[2], lL[2], gv[2], lv[2]);
            kd.w = kv[3] * exp_gdiff(gL[3], lL[3], gv[3], lv[3]);
            *reinterpret_cast<float4*>(Qg + off) = qg;
            *reinterpret_cast<float4*>(Kd + off) = kd;
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            Qt[(c + u) * kPS + r] = qv[u];
            Kt[(c + u) * kPS + r] = kv[u];
            Gt[(c + u) * kPS + r] = gv[u];
            GLt[(c + u) * kPS + r] = lv[u];
        }
    }
    __syncthreads();

    const int t = tid >> 2, s = tid & 3;   // tile t of the lower triangle, channel phase s
    int a = 0;
    while ((a + 1) * (a + 2) / 2 <= t) ++a;
    const int b = t - a * (a + 1) / 2;
    float pa[4][4], aa[4][4];
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) pa[x][y] = aa[x][y] = 0.f;
#pragma unroll 2
    for (int j = 0; j < DK / 4; ++j) {
        const int row = (4 * j + s) * kPS;
        const float4 qr = *reinterpret_cast<const float4*>(Qt + row + 4 * a);
        const float4 kr = *reinterpret_cast<const float4*>(Kt + row + 4 * a);
        const float4 gr = *reinterpret_cast<const float4*>(Gt + row + 4 * a);
        const float4 lr = *reinterpret_cast<const float4*>(GLt + row + 4 * a);
        const float4 ki = *reinterpret_cast<const float4*>(Kt + row + 4 * b);
        const float4 gi = *reinterpret_cast<const float4*>(Gt + row + 4 * b);
        const float4 li = *reinterpret_cast<const float4*>(GLt + row + 4 * b);
        const float qx[4] = {qr.x, qr.y, qr.z, qr.w}, kx[4] = {kr.x, kr.y, kr.z, kr.w};
        const float gx[4] = {gr.x, gr.y, gr.z, gr.w}, lx[4] = {lr.x, lr.y, lr.z, lr.w};
        const float ky[4] = {ki.x, ki.y, ki.z, ki.w}, gy[4] = {gi.x, gi.y, gi.z, gi.w};
        const float ly[4] = {li.x, li.y, li.z, li.w};
#pragma unroll
        for (int x = 0; x < 4; ++x)
#pragma unroll
            for (int y = 0; y < 4; ++y) {
                const float ke = ky[y] * exp_gdiff(gx[x], lx[x], gy[y], ly[y]);
                pa[x][y] = fmaf(qx[x], ke, pa[x][y]);
                aa[x][y] = fmaf(kx[x], ke, aa[x][y]);
            }
    }
#pragma unroll
    for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            pa[x][y] += __shfl_xor_sync(0xffffffffu, pa[x][y], 1);
            aa[x][y] += __shfl_xor_sync(0xffffffffu, aa[x][y], 1);
            pa[x][y] += __shfl_xor_sync(0xffffffffu, pa[x][y], 2);
            aa[x][y] += __shfl_xor_sync(0xffffffffu, aa[x][y], 2);
        }
    // lane s of the quad writes row 4a + s of the tile
    float pr[4], ar[4];
#pragma unroll
    for (int y = 0; y < 4; ++y) {
        pr[y] = pa[0][y];
        ar[y] = aa[0][y];
    }
#pragma unroll
    for (int x = 1; x < 4; ++x)
        if (s == x) {
#pragma unroll
            for (int y = 0; y < 4; ++y) {
                pr[y] = pa[x][y];
                ar[y] = aa[x][y];
            }
        }
    const int r = 4 * a + s, i0 = 4 * b;
    const bool live = r < len;
    float* Pc = P + ((size_t)blockIdx.x * H + h) * C * C;
    float* Ac = At + ((size_t)blockIdx.x * H + h) * C * C;
    float4 po, ao;
    po.x = (live && i0 <= r) ? pr[0] : 0.f;
    po.y = (live && i0 + 1 <= r) ? pr[1] : 0.f;
    po.z = (live && i0 + 2 <= r) ? pr[2] : 0.f;
    po.w = (live && i0 + 3 <= r) ? pr[3] : 0.f;
    ao.x = (live && i0 < r) ? ar[0] : 0.f;
    ao.y = (live && i0 + 1 < r) ? ar[1] : 0.f;
    ao.z = (live && i0 + 2 < r) ? ar[2] : 0.f;
    ao.w = (live && i0 + 3 < r) ? ar[3] : 0.f;
    *reinterpret_cast<float4*>(Pc + r * C + i0) = po;
    *reinterpret_cast<float4*>(Ac + r * C + i0) = ao;
    // the tiles above the diagonal
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e4 = tid; e4 < C * C / 4; e4 += kPThreads) {
        const int rr = e4 >> 4, bb = e4 & 15;
        if (bb > (rr >> 2)) {
            *reinterpret_cast<float4*>(Pc + rr * C + 4 * bb) = zero;
            *reinterpret_cast<float4*>(Ac + rr * C + 4 * bb) = zero;
        }
    }
}

// Reverse chain over one sequence's chunks, one block of kTW threads per
// (sequence, head, kBV state columns), two blocks per SM (its loads are latency bound).  Stores each chunk's end-state gradient dS' and dW, and
// the initial-state gradient.  Shared: dS [dk][kBV], M1 [C][dk] (Kd, then Qg),
// M2 [C][dk] (Wk), dOs [C][kBV], dWs [C][kBV], Ps [C][C], gC, gCl [dk].
template <typename Tin>
__global__ void __launch_bounds__(kTW, 2) kb_chain(const float* __restrict__ Qg, const float* __restrict__ Kd,
                                               const float* __restrict__ g, const float* __restrict__ gl,
                                               const float* __restrict__ Wk,
                                               const float* __restrict__ P, const Tin* __restrict__ d_o,
                                               const float* __restrict__ d_final, float* __restrict__ dS_chunk,
                                               float* __restrict__ dW, float* __restrict__ d_init, SeqMap smap,
                                               int H, int dk, int dv, int C) {
    extern __shared__ float smem[];
    const SeqInfo sq = smap.get(blockIdx.x);
    const int h = blockIdx.y, j0 = blockIdx.z * kBV, tid = threadIdx.x;
    float* dS = smem;
    float* M1 = dS + dk * kBV;
    float* M2 = M1 + C * dk;
    float* dOs = M2 + C * dk;
    float* dWs = dOs + C * kBV;
    float* Ps = dWs + C * kBV;
    float* gC = Ps + C * C;
    float* gCl = gC + dk;

    const size_t st_base = ((size_t)sq.seq * H + h) * dk * dv;
    for (int e = tid; e < dk * kBV; e += kTW) {
        const int c = e / kBV, j = e - c * kBV;
        dS[e] = d_final ? d_final[st_base + (size_t)c * dv + j0 + j] : 0.f;
    }
    __syncthreads();
    const int nch = (sq.len + C - 1) / C;
    for (int n = nch - 1; n >= 0; --n) {
        const int t0 = sq.tok0 + n * C;
        const int L = min(C, sq.len - n * C);
        const size_t chunk = (size_t)sq.chunk0 + n;
        const size_t sc_base = (chunk * H + h) * dk * dv;
        for (int e = tid; e < dk * kBV; e += kTW) {
            const int c = e / kBV, j = e - c * kBV;
            dS_chunk[sc_base + (size_t)c * dv + j0 + j] = dS[e];
        }
        if (n > 0) {
            // the previous chunk (next in this walk) into L2 while this one is worked on:
            // its Kd, Qg, Wk rows (4 lines of 128 bytes each), P (128 lines) and dO tile
            const int tp = t0 - C;
            for (int e = tid; e < 3 * C * (dk / 32) + (C * C) / 32 + C; e += kTW) {
                const char* a = nullptr;
                if (e < 3 * C * (dk / 32)) {
                    const int mtx = e / (C * (dk / 32)), rem = e - mtx * (C * (dk / 32));
                    const int r = rem / (dk / 32), ln = rem - r * (dk / 32);
                    const float* base = mtx == 0 ? Kd : mtx == 1 ? Qg : Wk;
                    a = reinterpret_cast<const char*>(base + tok_off(tp + r, H, h, dk) + 32 * ln);
                } else if (e < 3 * C * (dk / 32) + (C * C) / 32) {
                    a = reinterpret_cast<const char*>(P + (((size_t)chunk - 1) * H + h) * C * C +
                                                      32 * (e - 3 * C * (dk / 32)));
                } else {
                    const int r = e - 3 * C * (dk / 32) - (C * C) / 32;
                    a = reinterpret_cast<const char*>(d_o + tok_off(tp + r, H, h, dv) + j0);
                }
                asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
            }
        }
        const float* Pc = P + (chunk * H + h) * C * C;
        for (int e = tid; e < C * C; e += kTW) Ps[e] = Pc[e];
        for (int e = tid; e < L * kBV; e += kTW) {
            const int r = e / kBV, j = e - r * kBV;
            dOs[e] = to_f32(d_o[tok_off(t0 + r, H, h, dv) + j0 + j]);
        }
        for (int c = tid; c < dk; c += kTW) {
            gC[c] = g[tok_off(t0 + L - 1, H, h, dk) + c];
            gCl[c] = gl[tok_off(t0 + L - 1, H, h, dk) + c];
        }
        __syncthreads();
        for (int e = tid; e < L * dk; e += kTW) {
            const int r = e / dk, c = e - r * dk;
            const size_t off = tok_off(t0 + r, H, h, dk) + c;
            M1[e] = Kd[off];
            M2[e] = Wk[off];
        }
        __syncthreads();
        // dW = P^T dO + Kd dS' (P is zero above its diagonal): thread t forms column
        // t % 32 of rows 4 (t / 32) .. 4 (t / 32) + 3, so the rows of P and Kd it reads
        // are one float4 (the same for the whole warp) per column or channel group
        {
            const int j = tid & 31, i0 = 4 * (tid >> 5);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int r = 0; r < L; ++r) {
                const float o = dOs[r * kBV + j];
                const float4 p = *reinterpret_cast<const float4*>(Ps + r * C + i0);
                acc[0] = fmaf(p.x, o, acc[0]);
                acc[1] = fmaf(p.y, o, acc[1]);
                acc[2] = fmaf(p.z, o, acc[2]);
                acc[3] = fmaf(p.w, o, acc[3]);
            }
            for (int c = 0; c < dk; c += 4) {
                float ds[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) ds[u] = dS[(c + u) * kBV + j];
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float4 kd = *reinterpret_cast<const float4*>(M1 + (i0 + m) * dk + c);
                    acc[m] = fmaf(kd.x, ds[0], acc[m]);
                    acc[m] = fmaf(kd.y, ds[1], acc[m]);
                    acc[m] = fmaf(kd.z, ds[2], acc[m]);
                    acc[m] = fmaf(kd.w, ds[3], acc[m]);
                }
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int i = i0 + m;
                if (i < L) {
                    dWs[i * kBV + j] = acc[m];
                    dW[tok_off(t0 + i, H, h, dv) + j0 + j] = acc[m];
                }
            }
        }
        __syncthreads();
        for (int e = tid; e < L * dk; e += kTW) {
            const int r = e / dk, c = e - r * dk;
            const size_t off = tok_off(t0 + r, H, h, dk) + c;
            M1[e] = Qg[off];
        }
        __syncthreads();
        // dS = Diag(Gam) dS' + Qg^T dO - Wk^T dW: thread t forms column t % 32 of
        // channels 8 (t / 32) .. 8 (t / 32) + 7, read as two float4 of each of Qg and
        // Wk per row (each element is read and written by its own thread)
        {
            const int j = tid & 31, c0 = 8 * (tid >> 5);
            if (c0 < dk) {
                float acc[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) acc[m] = exp_g(gC[c0 + m], gCl[c0 + m]) * dS[(c0 + m) * kBV + j];
                for (int r = 0; r < L; ++r) {
                    const float o = dOs[r * kBV + j], w = dWs[r * kBV + j];
                    const float4 qa = *reinterpret_cast<const float4*>(M1 + r * dk + c0);
                    const float4 qb = *reinterpret_cast<const float4*>(M1 + r * dk + c0 + 4);
                    const float4 wa = *reinterpret_cast<const float4*>(M2 + r * dk + c0);
                    const float4 wb = *reinterpret_cast<const float4*>(M2 + r * dk + c0 + 4);
                    const float qv[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
                    const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
                    for (int m = 0; m < 8; ++m) acc[m] += qv[m] * o - wv[m] * w;
                }
#pragma unroll
                for (int m = 0; m < 8; ++m) dS[(c0 + m) * kBV + j] = acc[m];
            }
        }
        __syncthreads();
    }
    if (d_init) {
        for (int e = tid; e < dk * kBV; e += kTW) {
            const int c = e / kBV, j = e - c * kBV;
            d_init[st_base + (size_t)c * dv + j0 + j] = dS[e];
        }
    }
}

// Per (chunk, head): dQg = dO S^T, dKd = W dS'^T, dWk = -dW S^T (rows x DK),
// dGam = rowsum(dS' . S), and dP = dO W^T (i <= r, written over P).  d_v is
// walked in tiles of kBV columns.  Register tiles: thread t forms rows
// t / 16 + 16 m (m < 4) and channels t % 16 + 16 n (n < DK / 16) of the three
// products, and rows t / 16 + 16 m, columns t % 16 + 16 n (n < 4) of dP, so a
// shared-memory load feeds several multiply-adds and a warp's loads spread over
// the banks.  Shared: St, dSt [kBV][DK + 1] (transposed tiles), dOs, Ws, dWs [C][kBP].
template <typename Tin, int DK>
__global__ void __launch_bounds__(kT) kb_a(const Tin* __restrict__ d_o, const float* __restrict__ W,
                                           const float* __restrict__ dW, const float* __restrict__ S_chunk,
                                           const float* __restrict__ dS_chunk, float* __restrict__ dQg,
                                           float* __restrict__ dKd, float* __restrict__ dWk, float* __restrict__ dGam,
                                           float* __restrict__ dP, ChunkMap cmap, int H, int dv) {
    constexpr int C = 64;
    constexpr int NC = DK / 16;    // channels per thread
    static_assert(kT == 256, "tiles of 16 x 16 threads");
    extern __shared__ float smem[];
    int seq, tok0, len, idx;
    cmap.locate(blockIdx.x, seq, tok0, len, idx);
    const int h = blockIdx.y, tid = threadIdx.x, rb = tid >> 4, cb = tid & 15;
    constexpr int SP = DK + 1;     // padded row stride of the transposed state tiles
    float* St = smem;
    float* dSt = St + kBV * SP;
    float* dOs = dSt + kBV * SP;
    float* Ws = dOs + C * kBP;
    float* dWs = Ws + C * kBP;
    const size_t chunk = blockIdx.x;
    const size_t sc_base = (chunk * H + h) * DK * dv;
    float aQ[4][NC], aD[4][NC], aW[4][NC], aP[4][4];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
#pragma unroll
        for (int n = 0; n < NC; ++n) aQ[m][n] = aD[m][n] = aW[m][n] = 0.f;
#pragma unroll
        for (int n = 0; n < 4; ++n) aP[m][n] = 0.f;
    }
    float gam[NC];
#pragma unroll
    for (int n = 0; n < NC; ++n) gam[n] = 0.f;
    for (int jt = 0; jt < dv; jt += kBV) {
        for (int e = tid; e < kBV * DK; e += kT) {
            const int cc = e / kBV, j = e - cc * kBV;
            St[j * SP + cc] = S_chunk[sc_base + (size_t)cc * dv + jt + j];
            dSt[j * SP + cc] = dS_chunk[sc_base + (size_t)cc * dv + jt + j];
        }
        for (int e = tid; e < C * kBV; e += kT) {
            const int r = e / kBV, j = e - r * kBV;
            float a = 0.f, b = 0.f, d = 0.f;
            if (r < len) {
                a = to_f32(d_o[tok_off(tok0 + r, H, h, dv) + jt + j]);
                b = W[tok_off(tok0 + r, H, h, dv) + jt + j];
                d = dW[tok_off(tok0 + r, H, h, dv) + jt + j];
            }
            dOs[r * kBP + j] = a;
            Ws[r * kBP + j] = b;
            dWs[r * kBP + j] = d;
        }
        __syncthreads();
#pragma unroll 4
        for (int j = 0; j < kBV; ++j) {
            float o[4], w[4], dw[4], s[NC], ds[NC], wp[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int r = rb + 16 * m;
                o[m] = dOs[r * kBP + j];
                w[m] = Ws[r * kBP + j];
                dw[m] = dWs[r * kBP + j];
                wp[m] = Ws[(cb + 16 * m) * kBP + j];
            }
#pragma unroll
            for (int n = 0; n < NC; ++n) {
                s[n] = St[j * SP + cb + 16 * n];
                ds[n] = dSt[j * SP + cb + 16 * n];
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
#pragma unroll
                for (int n = 0; n < NC; ++n) {
                    aQ[m][n] = fmaf(o[m], s[n], aQ[m][n]);
                    aD[m][n] = fmaf(w[m], ds[n], aD[m][n]);
                    aW[m][n] = fmaf(-dw[m], s[n], aW[m][n]);
                }
#pragma unroll
                for (int n = 0; n < 4; ++n) aP[m][n] = fmaf(o[m], wp[n], aP[m][n]);
            }
            if (rb == 0) {
#pragma unroll
                for (int n = 0; n < NC; ++n) gam[n] = fmaf(ds[n], s[n], gam[n]);
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int r = rb + 16 * m;
        if (r < len) {
#pragma unroll
            for (int n = 0; n < NC; ++n) {
                const size_t off = tok_off(tok0 + r, H, h, DK) + cb + 16 * n;
                dQg[off] = aQ[m][n];
                dKd[off] = aD[m][n];
                dWk[off] = aW[m][n];
            }
        }
    }
    if (rb == 0) {
#pragma unroll
        for (int n = 0; n < NC; ++n) dGam[(chunk * H + h) * DK + cb + 16 * n] = gam[n];
    }
    float* dPc = dP + (chunk * H + h) * C * C;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int r = rb + 16 * m;
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            const int i = cb + 16 * n;
            dPc[r * C + i] = (r < len && i <= r) ? aP[m][n] : 0.f;
        }
    }
}

// Per (chunk, head): At, the back substitution for [Y | Z], dv, dKg, dbeta and
// dAt.  Shared: At, dA [C][C], bs, db [C], X = [Y | Z] [C][dv + dk + 1] (rows padded
// by one float against bank conflicts); U and Wk are read through L1 (98 KB of
// shared memory at d = 128, so two blocks share an SM).
template <typename Tin>
__global__ void __launch_bounds__(kT, 2) kb_b(const Tin* __restrict__ k, const Tin* __restrict__ v,
                                           const Tin* __restrict__ beta, const float* __restrict__ g,
                                           const float* __restrict__ gl, const float* __restrict__ Atg,
                                           const float* __restrict__ U, const float* __restrict__ Wk,
                                           const float* __restrict__ dW, const float* __restrict__ dWk,
                                           Tin* __restrict__ dv_out, Tin* __restrict__ dbeta_out,
                                           float* __restrict__ dKg, float* __restrict__ dAt, ChunkMap cmap, int H,
                                           int dk, int dv, int C) {
    extern __shared__ float smem[];
    int seq, tok0, len, idx;
    cmap.locate(blockIdx.x, seq, tok0, len, idx);
    const int h = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int ncol = dv + dk, xs = ncol + 1;
    float* At = smem;
    float* dA = At + C * C;
    float* bs = dA + C * C;
    float* db = bs + C;
    float* X = db + C;

    for (int e = tid; e < C * C; e += kT) At[e] = Atg[((size_t)blockIdx.x * H + h) * C * C + e];
    for (int r = tid; r < C; r += kT) {
        bs[r] = r < len ? to_f32(beta[(size_t)(tok0 + r) * H + h]) : 0.f;
        db[r] = 0.f;
    }
    __syncthreads();
    // (I + A)^T [Y | Z] = [dW | dWk]: right-hand sides loaded whole, then one
    // column per thread, rows from the last (A_ir = beta_i At_ir scaled once)
    for (int e = tid; e < len * ncol; e += kT) {
        const int r = e / ncol, j = e - r * ncol;
        X[r * xs + j] = j < dv ? dW[tok_off(tok0 + r, H, h, dv) + j] : dWk[tok_off(tok0 + r, H, h, dk) + j - dv];
    }
    for (int e = len * xs + tid; e < C * xs; e += kT) X[e] = 0.f;
    for (int e = tid; e < C * C; e += kT) dA[e] = bs[e / C] * At[e];   // A, until dA is formed
    __syncthreads();
    for (int j = tid; j < ncol; j += kT) {
        for (int r = len - 1; r >= 0; --r) {
            float s = X[r * xs + j];
            for (int i = r + 1; i < len; ++i) s -= dA[i * C + r] * X[i * xs + j];
            X[r * xs + j] = s;
        }
    }
    __syncthreads();
    // dv = beta Y, dKg = beta Z, dbeta_r = v_r . Y_r + Kg_r . Z_r (one warp per row)
    for (int r = warp; r < len; r += kT / 32) {
        const float b = bs[r];
        float s = 0.f;
        for (int j = lane; j < ncol; j += 32) {
            const float x = X[r * xs + j];
            if (j < dv) {
                const size_t off = tok_off(tok0 + r, H, h, dv) + j;
                dv_out[off] = from_f32<Tin>(b * x);
                s += to_f32(v[off]) * x;
            } else {
                const size_t off = tok_off(tok0 + r, H, h, dk) + j - dv;
                dKg[off] = b * x;
                s += to_f32(k[off]) * exp_g(g[off], gl[off]) * x;
            }
        }
        s = wsum(s);
        if (lane == 0) db[r] = s;
    }
    __syncthreads();   // the rows of X are read by other threads below (and dA is overwritten)
    // dA = -(Y U^T + Z Wk^T), i < r: one warp per 4 x 4 tile of the lower triangle
    // (rows 4a..4a+3, columns 4b..4b+3, b <= a), its lanes splitting the columns of
    // [Y | Z] and [U | Wk], so each load of a U or Wk row is one coalesced line;
    // five shuffle rounds add the lanes' partial sums.  Rows i >= len of U and Wk
    // are read as zero; the tiles above the diagonal are set to zero.
    for (int t = warp; t < 136; t += kT / 32) {
        int a = 0;
        while ((a + 1) * (a + 2) / 2 <= t) ++a;
        const int b = t - a * (a + 1) / 2;
        const float* urow[4];
        const float* wrow[4];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
            const int i = 4 * b + n;
            urow[n] = i < len ? U + tok_off(tok0 + i, H, h, dv) : nullptr;
            wrow[n] = i < len ? Wk + tok_off(tok0 + i, H, h, dk) : nullptr;
        }
        float acc[4][4];
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int n = 0; n < 4; ++n) acc[m][n] = 0.f;
        for (int j = lane; j < ncol; j += 32) {
            float xr[4], ui[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) xr[m] = X[(4 * a + m) * xs + j];
#pragma unroll
            for (int n = 0; n < 4; ++n)
                ui[n] = urow[n] ? (j < dv ? __ldg(urow[n] + j) : __ldg(wrow[n] + j - dv)) : 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int n = 0; n < 4; ++n) acc[m][n] = fmaf(xr[m], ui[n], acc[m][n]);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int n = 0; n < 4; ++n) acc[m][n] = wsum(acc[m][n]);
        if (lane == 0) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int r = 4 * a + m, i0 = 4 * b;
                float4 o;
                o.x = (r < len && i0 < r) ? -acc[m][0] : 0.f;
                o.y = (r < len && i0 + 1 < r) ? -acc[m][1] : 0.f;
                o.z = (r < len && i0 + 2 < r) ? -acc[m][2] : 0.f;
                o.w = (r < len && i0 + 3 < r) ? -acc[m][3] : 0.f;
                *reinterpret_cast<float4*>(dA + r * C + i0) = o;
            }
        }
    }
    for (int e4 = tid; e4 < C * C / 4; e4 += kT) {
        const int r = e4 >> 4, bb = e4 & 15;
        if (bb > (r >> 2)) *reinterpret_cast<float4*>(dA + r * C + 4 * bb) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    float* dAc = dAt + ((size_t)blockIdx.x * H + h) * C * C;
    for (int r = tid; r < C; r += kT) {
        float s = db[r];
        for (int i = 0; i < r; ++i) s += dA[r * C + i] * At[r * C + i];
        if (r < len) dbeta_out[(size_t)(tok0 + r) * H + h] = from_f32<Tin>(s);
    }
    for (int e = tid; e < C * C; e += kT) dAc[e] = bs[e / C] * dA[e];
}

constexpr int kCThreads = 512;   // kb_c: 8 pairs of row blocks x 64 channels
constexpr int kCH = 64;          // kb_c: channels per pass

// Per (chunk, head): the pairwise terms of At and P, the elementwise factors,
// and dlog alpha.  A pairwise term T_ri = (dAt_ri k_r + dP_ri q_r) k_i E_ri depends
// on log alpha_j exactly for i < j <= r, so its share of dlog alpha_j is
// F(j) = sum_{r >= j} sum_{i < j} T_ri.  Likewise Qg_r, Kg_r depend on log alpha_j
// for j <= r, Kd_r for r < j, and Gam for every j:
//   dlog alpha_j = F(j) + sum_{r>=j} (dQg Qg + dKg Kg)_r + sum_{r<j} (dKd Kd)_r + dGam Gam.
// The pair grid is cut into 4 x 4 tiles (rows of block a: 4a..4a+3, columns of
// block b: 4b..4b+3, b <= a).  A thread owns one channel and the row blocks a and
// 15 - a (17 tiles), so each exponential is formed once and the row sums (dq and
// the row part of dk) stay in registers; the column sums (the rest of dk) are
// added per tile into shared memory.  F is assembled from tile sums without any
// term that is added and later cancelled: for j = 4m + u (0 <= u < 4),
//   F(j) = sum_{a > m} [ sum_{b < m} S_ab + sum_{y < u} colT_am(y) ]   (rows below block m)
//        + sum_{b < m} sum_{x >= u} rowT_mb(x)                         (rows of block m, u..3)
//        + sum_{y < u <= x} T_{4m+x, 4m+y}                              (diagonal tile)
// with S_ab the sum of tile (a, b) and rowT / colT its row and column sums; the
// thread of row block a adds the first line's terms of tile (a, m) to F(4m + u)
// and keeps the other two in registers until its row block is done.
// Channels are processed in passes of 64; q, k, g and its low part are staged
// channel-major ([c][r], row stride kPS), padded rows as in kb_p.  The dAt and
// dP tiles are staged with their masks applied (zero for i >= r, resp. i > r, and
// for rows past the end of the chunk).
// Shared: Qt, Kt, Gt, GLt [kCH][kPS], dAs, dPs [C][C], Fs, Ys, Xs, dQs, dKgs, dKds
// [C][kCH], PX, PY [8][kCH] (the dlog alpha scan's segment sums).
template <typename Tin, int DK>
__global__ void __launch_bounds__(kCThreads, 1) kb_c(const Tin* __restrict__ q, const Tin* __restrict__ k,
                                                     const Tin* __restrict__ la, const float* __restrict__ g,
                                                     const float* __restrict__ gl,
                                                     const float* __restrict__ dAt, const float* __restrict__ dP,
                                                     const float* __restrict__ dQg, const float* __restrict__ dKd,
                                                     const float* __restrict__ dKg, const float* __restrict__ dGam,
                                                     Tin* __restrict__ dq_out, Tin* __restrict__ dk_out,
                                                     Tin* __restrict__ dla_out, ChunkMap cmap, int H) {
    constexpr int C = kBwdC;
    static_assert(DK % kCH == 0, "whole passes of channels");
    extern __shared__ __align__(16) float smem[];
    float* Qt = smem;
    float* Kt = Qt + kCH * kPS;
    float* Gt = Kt + kCH * kPS;
    float* GLt = Gt + kCH * kPS;
    float* dAs = GLt + kCH * kPS;
    float* dPs = dAs + C * C;
    float* Fs = dPs + C * C;
    float* Ys = Fs + C * kCH;
    float* Xs = Ys + C * kCH;
    float* dQs = Xs + C * kCH;       // this pass's dQg, dKg, dKd [C][kCH]
    float* dKgs = dQs + C * kCH;
    float* dKds = dKgs + C * kCH;
    float* PX = dKds + C * kCH;      // per-segment sums of the dlog alpha scan [8][kCH]
    float* PY = PX + 8 * kCH;
    int seq, tok0, len, idx;
    cmap.locate(blockIdx.x, seq, tok0, len, idx);
    const int h = blockIdx.y, tid = threadIdx.x;
    const size_t chunk = blockIdx.x;
    const size_t tbase = (chunk * H + h) * C * C;
    for (int e4 = tid; e4 < C * C / 4; e4 += kCThreads) {
        const int r = e4 >> 4, i0 = 4 * (e4 & 15);
        const bool live = r < len;
        const float4 av = *reinterpret_cast<const float4*>(dAt + tbase + r * C + i0);
        const float4 pv = *reinterpret_cast<const float4*>(dP + tbase + r * C + i0);
        float4 ao, po;
        ao.x = (live && i0 < r) ? av.x : 0.f;
        ao.y = (live && i0 + 1 < r) ? av.y : 0.f;
        ao.z = (live && i0 + 2 < r) ? av.z : 0.f;
        ao.w = (live && i0 + 3 < r) ? av.w : 0.f;
        po.x = (live && i0 <= r) ? pv.x : 0.f;
        po.y = (live && i0 + 1 <= r) ? pv.y : 0.f;
        po.z = (live && i0 + 2 <= r) ? pv.z : 0.f;
        po.w = (live && i0 + 3 <= r) ? pv.w : 0.f;
        *reinterpret_cast<float4*>(dAs + r * C + i0) = ao;
        *reinterpret_cast<float4*>(dPs + r * C + i0) = po;
    }
    const size_t last = tok_off(tok0 + len - 1, H, h, DK);
    const int c = tid & (kCH - 1), ap = tid / kCH;   // this thread's channel in the pass, row-block pair

    for (int c0 = 0; c0 < DK; c0 += kCH) {
        if (c0 > 0) __syncthreads();   // the previous pass is done with the shared arrays
        // staging, groups of 4 channels; a warp covers 16 rows x 2 groups (32 banks)
        for (int e4 = tid; e4 < C * kCH / 4; e4 += kCThreads) {
            const int w = e4 >> 5, ln = e4 & 31;
            const int r = (ln & 15) + 16 * (w & 3);
            const int cq = 4 * (2 * (w >> 2) + (ln >> 4));
            float gv[4], lv[4], qv[4] = {0.f, 0.f, 0.f, 0.f}, kv[4] = {0.f, 0.f, 0.f, 0.f};
            if (r < len) {
                const size_t off = tok_off(tok0 + r, H, h, DK) + c0 + cq;
                load4(q + off, qv);
                load4(k + off, kv);
                load4(g + off, gv);
                load4(gl + off, lv);
            } else {
                load4(g + last + c0 + cq, gv);
                load4(gl + last + c0 + cq, lv);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                Qt[(cq + u) * kPS + r] = qv[u];
                Kt[(cq + u) * kPS + r] = kv[u];
                Gt[(cq + u) * kPS + r] = gv[u];
                GLt[(cq + u) * kPS + r] = lv[u];
            }
        }
        for (int e = tid; e < 2 * C * kCH; e += kCThreads) Fs[e] = 0.f;   // Fs and Ys
        for (int e4 = tid; e4 < len * kCH / 4; e4 += kCThreads) {
            const int r = e4 / (kCH / 4), cq = 4 * (e4 - r * (kCH / 4));
            const size_t off = tok_off(tok0 + r, H, h, DK) + c0 + cq;
            *reinterpret_cast<float4*>(dQs + r * kCH + cq) = *reinterpret_cast<const float4*>(dQg + off);
            *reinterpret_cast<float4*>(dKgs + r * kCH + cq) = *reinterpret_cast<const float4*>(dKg + off);
            *reinterpret_cast<float4*>(dKds + r * kCH + cq) = *reinterpret_cast<const float4*>(dKd + off);
        }
        __syncthreads();

        const float* qc = Qt + c * kPS;
        const float* kc = Kt + c * kPS;
        const float* gc = Gt + c * kPS;
        const float* lc = GLt + c * kPS;
        for (int half = 0; half < 2; ++half) {
            const int a = half == 0 ? ap : 15 - ap;
            float qr[4], kr[4], gr[4], lr[4];
            {
                const float4 q4 = *reinterpret_cast<const float4*>(qc + 4 * a);
                const float4 k4 = *reinterpret_cast<const float4*>(kc + 4 * a);
                const float4 g4 = *reinterpret_cast<const float4*>(gc + 4 * a);
                const float4 l4 = *reinterpret_cast<const float4*>(lc + 4 * a);
                qr[0] = q4.x; qr[1] = q4.y; qr[2] = q4.z; qr[3] = q4.w;
                kr[0] = k4.x; kr[1] = k4.y; kr[2] = k4.z; kr[3] = k4.w;
                gr[0] = g4.x; gr[1] = g4.y; gr[2] = g4.z; gr[3] = g4.w;
                lr[0] = l4.x; lr[1] = l4.y; lr[2] = l4.z; lr[3] = l4.w;
            }
            float x1[4] = {0.f, 0.f, 0.f, 0.f}, x2[4] = {0.f, 0.f, 0.f, 0.f};
            float rs[4] = {0.f, 0.f, 0.f, 0.f};   // F terms of rows 4a + u.. (second and third lines)
            float pref = 0.f;                      // sum of the tiles (a, b' < b)
            for (int b = 0; b < a; ++b) {
                const float4 k4 = *reinterpret_cast<const float4*>(kc + 4 * b);
                const float4 g4 = *reinterpret_cast<const float4*>(gc + 4 * b);
                const float4 l4 = *reinterpret_cast<const float4*>(lc + 4 * b);
                const float ki[4] = {k4.x, k4.y, k4.z, k4.w}, gi[4] = {g4.x, g4.y, g4.z, g4.w};
                const float li[4] = {l4.x, l4.y, l4.z, l4.w};
                float colT[4] = {0.f, 0.f, 0.f, 0.f}, yc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float4 a4 = *reinterpret_cast<const float4*>(dAs + (4 * a + x) * C + 4 * b);
                    const float4 p4 = *reinterpret_cast<const float4*>(dPs + (4 * a + x) * C + 4 * b);
                    const float da[4] = {a4.x, a4.y, a4.z, a4.w}, dp[4] = {p4.x, p4.y, p4.z, p4.w};
                    float tx[4];
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        // with w = dAt k_r + dP q_r: T_ri = w k_i E and the column term is w E
                        const float e = exp_gdiff(gr[x], lr[x], gi[y], li[y]);
                        const float ke = ki[y] * e;
                        x1[x] = fmaf(da[y], ke, x1[x]);
                        x2[x] = fmaf(dp[y], ke, x2[x]);
                        const float w = fmaf(da[y], kr[x], dp[y] * qr[x]);
                        yc[y] = fmaf(w, e, yc[y]);
                        tx[y] = w * ke;
                    }
                    const float rowT = (tx[0] + tx[1]) + (tx[2] + tx[3]);
#pragma unroll
                    for (int y = 0; y < 4; ++y) colT[y] += tx[y];
                    // rows x >= u of this tile count for F(4a + u)
#pragma unroll
                    for (int u = 0; u <= x; ++u) rs[u] += rowT;
                }
                atomicAdd(&Fs[(4 * b) * kCH + c], pref);
                atomicAdd(&Fs[(4 * b + 1) * kCH + c], pref + colT[0]);
                atomicAdd(&Fs[(4 * b + 2) * kCH + c], pref + (colT[0] + colT[1]));
                atomicAdd(&Fs[(4 * b + 3) * kCH + c], pref + (colT[0] + colT[1] + colT[2]));
                pref += (colT[0] + colT[1]) + (colT[2] + colT[3]);
#pragma unroll
                for (int y = 0; y < 4; ++y) atomicAdd(&Ys[(4 * b + y) * kCH + c], yc[y]);
            }
            // the diagonal tile: pairs y <= x (E = 1 on the diagonal)
            {
                float yc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float4 a4 = *reinterpret_cast<const float4*>(dAs + (4 * a + x) * C + 4 * a);
                    const float4 p4 = *reinterpret_cast<const float4*>(dPs + (4 * a + x) * C + 4 * a);
                    const float da[4] = {a4.x, a4.y, a4.z, a4.w}, dp[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
                    for (int y = 0; y <= x; ++y) {
                        const float e = y == x ? 1.f : exp_gdiff(gr[x], lr[x], gr[y], lr[y]);
                        const float ke = kr[y] * e;
                        const float av = da[y] * ke, bv = dp[y] * ke;
                        x1[x] += av;
                        x2[x] += bv;
                        yc[y] = fmaf(fmaf(da[y], kr[x], dp[y] * qr[x]), e, yc[y]);
                        if (y < x) {
                            const float t = fmaf(kr[x], av, qr[x] * bv);
#pragma unroll
                            for (int u = y + 1; u <= x; ++u) rs[u] += t;
                        }
                    }
                }
#pragma unroll
                for (int y = 0; y < 4; ++y) atomicAdd(&Ys[(4 * a + y) * kCH + c], yc[y]);
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) atomicAdd(&Fs[(4 * a + u) * kCH + c], rs[u]);
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int r = 4 * a + x;
                Xs[r * kCH + c] = x1[x];
                if (r < len) {
                    const size_t off = tok_off(tok0 + r, H, h, DK) + c0 + c;
                    dq_out[off] = from_f32<Tin>(x2[x] + dQs[r * kCH + c] * exp_g(gr[x], lr[x]));
                }
            }
        }
        __syncthreads();
        // dk, and the per-(row, channel) terms of dlog alpha (into Xs and Ys, which
        // each element's thread has just read)
        for (int e = tid; e < len * kCH; e += kCThreads) {
            const int r = e / kCH, cc = e - r * kCH;
            const size_t off = tok_off(tok0 + r, H, h, DK) + c0 + cc;
            const float gv = Gt[cc * kPS + r], lv = GLt[cc * kPS + r];
            const float eg = exp_g(gv, lv);
            const float ed = exp_gdiff(Gt[cc * kPS + len - 1], GLt[cc * kPS + len - 1], gv, lv);
            const float dkg = dKgs[e], dkd = dKds[e];
            dk_out[off] = from_f32<Tin>(Xs[e] + Ys[e] + dkg * eg + dkd * ed);
            Xs[e] = dkd * Kt[cc * kPS + r] * ed;                              // dKd Kd
            Ys[e] = (dQs[e] * Qt[cc * kPS + r] + dkg * Kt[cc * kPS + r]) * eg;   // dQg Qg + dKg Kg
        }
        __syncthreads();
        // dlog alpha (zero where the forward's floor on log alpha was active):
        //   F(j) + sum_{r<j} dKd Kd + sum_{r>=j} (dQg Qg + dKg Kg) + dGam Gam,
        // the two sums as scans over 8 segments of 8 rows per channel
        const int seg = ap, j0 = 8 * seg;
        {
            float sx = 0.f, sy = 0.f;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (j0 + u < len) {
                    sx += Xs[(j0 + u) * kCH + c];
                    sy += Ys[(j0 + u) * kCH + c];
                }
            PX[seg * kCH + c] = sx;
            PY[seg * kCH + c] = sy;
        }
        __syncthreads();
        if (j0 < len) {
            float pre = 0.f, suf = 0.f;   // sum of the segments before / after this one
            for (int s2 = 0; s2 < seg; ++s2) pre += PX[s2 * kCH + c];
            for (int s2 = seg + 1; s2 < 8; ++s2) suf += PY[s2 * kCH + c];
            const float gam = dGam[(chunk * H + h) * DK + c0 + c] *
                              exp_g(Gt[c * kPS + len - 1], GLt[c * kPS + len - 1]);
            float prej[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                prej[u] = pre;
                if (j0 + u < len) pre += Xs[(j0 + u) * kCH + c];
            }
#pragma unroll
            for (int u = 7; u >= 0; --u) {
                const int j = j0 + u;
                if (j < len) {
                    suf += Ys[j * kCH + c];
                    const size_t off = tok_off(tok0 + j, H, h, DK) + c0 + c;
                    dla_out[off] = from_f32<Tin>(to_f32(la[off]) >= kLogAlphaFloor
                                                     ? Fs[j * kCH + c] + prej[u] + suf + gam : 0.f);
                }
            }
        }
    }
}

template <typename Tin, int DK>
cudaError_t run_bwd_dk(const Tin* q, const Tin* k, const Tin* v, const Tin* la, const Tin* beta,
                       const Tin* d_o, Tin* dq, Tin* dk_, Tin* dv_, Tin* dla, Tin* dbeta, const ChunkMap& cmap,
                       int n_chunks, int H, int dv, const BwdWorkspace& ws, cudaStream_t stream) {
    constexpr int C = 64;
    const size_t smem_a = sizeof(float) * (2 * (size_t)kBV * (DK + 1) + 3 * (size_t)C * kBP);
    const size_t smem_b = sizeof(float) * (2 * (size_t)C * C + 2 * C + (size_t)C * (dv + DK + 1));
    const size_t smem_c = sizeof(float) * (4 * (size_t)kCH * kPS + 2 * (size_t)C * C + 6 * (size_t)C * kCH +
                                           2 * 8 * (size_t)kCH);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(kb_a<Tin, DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a))) return e;
    if ((e = cudaFuncSetAttribute(kb_b<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b))) return e;
    if ((e = cudaFuncSetAttribute(kb_c<Tin, DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_c))) return e;
    const dim3 grid(n_chunks, H);
    if (std::is_same<Tin, __nv_bfloat16>::value && DK == 128 && dv == 128 && ws.tc_ws) {
        // bf16, d = 128: the four chunk-local products on the tensor cores
        e = launch_kb_a_tc(d_o, ws.fwd.W, ws.dW, ws.fwd.S_chunk, ws.dS_chunk, ws.dQg, ws.dKd, ws.dWk, ws.dGam, ws.P,
                           reinterpret_cast<int*>(ws.tc_ws), cmap, n_chunks, H, stream);
        if (e != cudaSuccess) return e;
    } else {
        kb_a<Tin, DK><<<grid, kT, smem_a, stream>>>(d_o, ws.fwd.W, ws.dW, ws.fwd.S_chunk, ws.dS_chunk, ws.dQg,
                                                   ws.dKd, ws.dWk, ws.dGam, ws.P, cmap, H, dv);
    }
    timing_mark(stream, 4);
    if (std::is_same<Tin, __nv_bfloat16>::value && DK == 128 && dv == 128 && ws.tc_ws && ws.T) {
        // bf16, d = 128: the back substitution as two tensor-core products with T
        e = launch_kb_b_tc(ws.T, ws.At, ws.tc_ws, ws.dW, ws.dWk, k, v, beta, ws.fwd.g, ws.fwd.gl, dv_,
                           dbeta, ws.dKg, ws.dAt, reinterpret_cast<int*>(ws.tc_ws), cmap, n_chunks, H, stream);
        if (e != cudaSuccess) return e;
    } else {
        kb_b<Tin><<<grid, kT, smem_b, stream>>>(k, v, beta, ws.fwd.g, ws.fwd.gl, ws.At, ws.fwd.U, ws.fwd.Wk, ws.dW,
                                                ws.dWk, dv_, dbeta, ws.dKg, ws.dAt, cmap, H, DK, dv, C);
    }
    timing_mark(stream, 5);
    if (std::is_same<Tin, __nv_bfloat16>::value && DK == 128 && dv == 128 && ws.tc_ws) {
        // bf16, d = 128: the pairwise terms as block-referenced tensor-core products
        e = launch_kb_c_tc(q, k, la, ws.fwd.g, ws.fwd.gl, ws.dAt, ws.P, ws.dQg, ws.dKd, ws.dKg, ws.dGam, dq, dk_, dla,
                           reinterpret_cast<int*>(ws.tc_ws), cmap, n_chunks, H, stream);
        if (e != cudaSuccess) return e;
    } else {
        kb_c<Tin, DK><<<grid, kCThreads, smem_c, stream>>>(q, k, la, ws.fwd.g, ws.fwd.gl, ws.dAt, ws.P, ws.dQg,
                                                         ws.dKd, ws.dKg, ws.dGam, dq, dk_, dla, cmap, H);
    }
    timing_mark(stream, 6);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t run_bwd(const Tin* q, const Tin* k, const Tin* v, const Tin* la, const Tin* beta, const float* init_state,
                    const Tin* d_o, const float* d_final, Tin* dq, Tin* dk_, Tin* dv_, Tin* dla, Tin* dbeta,
                    float* d_init, const ChunkMap& cmap, const SeqMap& smap, int n_chunks, int n_seqs, int H, int dk,
                    int dv, const BwdWorkspace& ws, cudaStream_t stream, kda_dtype dtype) {
    constexpr int C = 64;
    cudaError_t e;
    if (ws.tc_ws) {
        // bf16, d = 128: the tensor-core forward recomputes U, Wk, W and the chunk start states
        if ((e = launch_simt_g(dtype, la, cmap, n_chunks, H, dk, ws.fwd, stream)) != cudaSuccess) return e;
        e = launch_tc_states(q, k, v, la, beta, init_state, ws.o_scratch, cmap, smap, n_chunks, n_seqs, H, ws.tc_ws,
                             ws.fwd.S_chunk, ws.fwd.W, ws.T, ws.At, stream);
    } else {
        e = launch_simt_states(dtype, k, v, la, beta, init_state, cmap, smap, n_chunks, n_seqs, H, dk, dv, C, ws.fwd,
                               stream);
    }
    if (e != cudaSuccess) return e;
    timing_mark(stream, 1);
    const size_t smem_p = sizeof(float) * 4 * (size_t)kPS * dk;
    const size_t smem_chain = sizeof(float) * ((size_t)dk * kBV + 2 * (size_t)C * dk + 2 * (size_t)C * kBV +
                                               (size_t)C * C + 2 * dk);
    // the tensor-core path takes At from the recompute and P from its images, and kb_a_tc
    // writes the whole dP buffer: no pairwise pass runs there
    const bool tc_chain = std::is_same<Tin, __nv_bfloat16>::value && dk == 128 && dv == 128 && ws.tc_ws;
    if (!tc_chain) {
        auto kern_p = dk == 128 ? kb_p<Tin, 128> : kb_p<Tin, 64>;
        if ((e = cudaFuncSetAttribute(kern_p, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_p))) return e;
        if ((e = cudaFuncSetAttribute(kb_chain<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_chain)))
            return e;
        // two chain blocks per SM (115,712 bytes each at d = 128) need the whole shared-memory carveout
        if ((e = cudaFuncSetAttribute(kb_chain<Tin>, cudaFuncAttributePreferredSharedMemoryCarveout, 100))) return e;
        if (n_chunks > 0)
            kern_p<<<dim3(n_chunks, H), kPThreads, smem_p, stream>>>(q, k, ws.fwd.g, ws.fwd.gl, ws.P, ws.At, ws.Qg,
                                                                     ws.Kd, cmap, H);
    }
    timing_mark(stream, 2);
    if (n_seqs > 0) {
        if (tc_chain) {
            // bf16, d = 128: the reverse chain on the tensor cores, from the recompute's images
            if ((e = launch_tc_chain(ws.tc_ws, d_o, d_final, ws.dS_chunk, ws.dW, d_init, smap, n_seqs, H, stream)) !=
                cudaSuccess)
                return e;
        } else {
            kb_chain<Tin><<<dim3(n_seqs, H, dv / kBV), kTW, smem_chain, stream>>>(
                ws.Qg, ws.Kd, ws.fwd.g, ws.fwd.gl, ws.fwd.Wk, ws.P, d_o, d_final, ws.dS_chunk, ws.dW, d_init, smap,
                H, dk, dv, C);
        }
    }
    timing_mark(stream, 3);
    if ((e = cudaGetLastError()) != cudaSuccess || n_chunks == 0) return e;
    if (dk == 128) return run_bwd_dk<Tin, 128>(q, k, v, la, beta, d_o, dq, dk_, dv_, dla, dbeta, cmap, n_chunks, H, dv,
                                               ws, stream);
    return run_bwd_dk<Tin, 64>(q, k, v, la, beta, d_o, dq, dk_, dv_, dla, dbeta, cmap, n_chunks, H, dv, ws, stream);
}

}  // namespace

cudaError_t launch_simt_backward(kda_dtype dtype, const void* q, const void* k, const void* v,
                                 const void* log_alpha, const void* beta, const float* init_state,
                                 const void* d_o, const float* d_final_state, void* dq, void* dk, void* dv,
                                 void* dlog_alpha, void* dbeta, float* d_init_state, const ChunkMap& cmap,
                                 const SeqMap& smap, int n_chunks, int n_seqs, int H, int dkk, int dvv, int C,
                                 const BwdWorkspace& ws, cudaStream_t stream) {
    if (C != 64) return cudaErrorNotSupported;
    if (dtype == KDA_F32)
        return run_bwd<float>((const float*)q, (const float*)k, (const float*)v, (const float*)log_alpha,
                              (const float*)beta, init_state, (const float*)d_o, d_final_state, (float*)dq,
                              (float*)dk, (float*)dv, (float*)dlog_alpha, (float*)dbeta, d_init_state, cmap, smap,
                              n_chunks, n_seqs, H, dkk, dvv, ws, stream, dtype);
    using bf = __nv_bfloat16;
    return run_bwd<bf>((const bf*)q, (const bf*)k, (const bf*)v, (const bf*)log_alpha, (const bf*)beta, init_state,
                       (const bf*)d_o, d_final_state, (bf*)dq, (bf*)dk, (bf*)dv, (bf*)dlog_alpha, (bf*)dbeta,
                       d_init_state, cmap, smap, n_chunks, n_seqs, H, dkk, dvv, ws, stream, dtype);
}

}  // namespace kda
