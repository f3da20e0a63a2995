// sm_100a building blocks for the tensor-core KDA path: shared-memory operand
// layout, UMMA descriptors, tcgen05 MMA / TMEM access, mbarriers and bulk
// copies.  Inline PTX only; every wait is bounded.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace kda {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// Operand tiles in shared memory: K-major, 128-byte swizzle, bf16.
// A tile of `rows` rows (multiple of 8) and K columns (multiple of 64) is
// stored as K/64 column blocks of rows x 128 bytes; inside a block, row r
// occupies bytes [128 r, 128 r + 128) and its eight 16-byte chunks are
// permuted by chunk ^ (r % 8).  Tile bases are 1024-byte aligned, so the
// hardware's address-bit swizzle matches this layout.
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ uint32_t sw128_offset(int row, int k, int rows) {
    const int kb = k >> 6, kk = k & 63;
    return (uint32_t)(kb * rows * 128 + row * 128 + ((((kk >> 3) ^ (row & 7))) << 4) + ((kk & 7) << 1));
}

// Byte offset of the 16-byte chunk holding elements k..k+7 (k % 8 == 0).
__host__ __device__ __forceinline__ uint32_t sw128_chunk(int row, int k, int rows) {
    return (uint32_t)((k >> 6) * rows * 128 + row * 128 + ((((k & 63) >> 3) ^ (row & 7)) << 4));
}

// Shared-memory matrix descriptor for a K-major SW128 tile whose first
// element sits at byte address `addr` (for K offsets inside a 128-byte row the
// caller adds 32 bytes per 16 elements).  LBO = 16 B (unused by this layout),
// SBO = 1024 B between 8-row groups, version 1, layout type 2 (128B swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t addr) {
    uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Descriptor of the K-slice [16 s, 16 s + 16) of a tile with `rows` rows.
__device__ __forceinline__ uint64_t sw128_desc_k(uint32_t tile_addr, int rows, int s) {
    return sw128_desc(tile_addr + (uint32_t)((s >> 2) * rows * 128 + (s & 3) * 32));
}

// Instruction descriptor, kind::f16: bf16 A and B (both K-major), fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Same with B MN-major (N contiguous).
__host__ __device__ constexpr uint32_t idesc_bf16_f32_bmn(int M, int N) {
    return idesc_bf16_f32(M, N) | (1u << 16);
}

// ---------------------------------------------------------------------------
// MN-major B tiles (K rows, N contiguous), 128-byte swizzle, bf16.
// N is split into blocks of 64 elements; block b holds K rows of 128 bytes at
// byte offset b * K * 128, with the same chunk ^ (row % 8) permutation as the
// K-major tiles.  (A 64-wide MN-major tile and a 64-deep K-major tile of the
// same row-major matrix therefore have the same bytes.)
// ---------------------------------------------------------------------------
__host__ __device__ __forceinline__ uint32_t mn_chunk(int k, int n, int K) {   // n % 8 == 0
    return (uint32_t)((n >> 6) * K * 128 + k * 128 + ((((n & 63) >> 3) ^ (k & 7)) << 4));
}
__host__ __device__ __forceinline__ uint32_t mn_offset(int k, int n, int K) {
    return mn_chunk(k, n & ~7, K) + ((n & 7) << 1);
}

// Descriptor of the K-slice [16 s, 16 s + 16) of an MN-major tile with K rows:
// LBO = K * 128 bytes between 64-wide N blocks, SBO = 1024 bytes between
// 8-row groups.
__device__ __forceinline__ uint64_t mn_desc_k(uint32_t tile_addr, int K, int s) {
    const uint32_t addr = tile_addr + (uint32_t)s * 2048u;
    uint64_t d = (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)(((uint32_t)K * 128u >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// D[tmem] (+)= A[smem] * B[smem]^T, issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

// Arrive on `bar` once all previously issued MMAs of this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Generic-proxy shared-memory writes -> visible to the async proxy (MMA, bulk copies).
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ---------------------------------------------------------------------------
// TMEM allocation (one full warp executes these)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// TMEM address of (lane, column) relative to an allocation base.
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, int lane, int col) {
    return base + ((uint32_t)lane << 16) + (uint32_t)col;
}

// 32 lanes x 16 columns: thread t of the warp receives lane (lane0 + t),
// columns [col, col + 16).  The warp must own the 32-lane sub-partition.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// mbarriers and bulk copies
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

// Plain arrival (no transaction count).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase with the given parity to complete; gives up after
// `limit_ns` nanoseconds and returns false (the caller records the error).
// The clock is read once per 64 polls (each poll already suspends the thread
// for a while inside try_wait).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns = 2000000000ull) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63u) == 0u && globaltimer_ns() - t0 > limit_ns) return false;
    }
}

// 1-D bulk copy global -> shared, completion counted on `bar` (16-byte
// aligned addresses, size a multiple of 16).
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst_smem)),
                 "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Shared -> global bulk copy (TMA engine, one destination), tracked by bulk groups.
// Both addresses 16-byte aligned, size a multiple of 16.
__device__ __forceinline__ void bulk_s2g(void* dst_gmem, const void* src_smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst_gmem),
                 "r"(smem_u32(src_smem)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk group has finished reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Same, but the most recently committed group may still be reading.
__device__ __forceinline__ void bulk_wait_read_but1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ float bf16_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// Split two fp32 values into bf16 pairs hi + lo with hi = RN(x), lo = RN(x - hi):
// hi + lo carries about 16 significant bits.  Products computed as
// a_hi b_hi + a_hi b_lo + a_lo b_hi ("three-term bf16") keep a relative error
// near 2^-16 while running on the bf16 tensor-core path.
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t x) { return make_float2(bf16_lo(x), bf16_hi(x)); }

__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
    hi = pack_bf16(a, b);
    // x - hi is exact in fp32; one packed fma forms both differences
    const float2 d = __ffma2_rn(unpack_bf16x2(hi), make_float2(-1.f, -1.f), make_float2(a, b));
    lo = pack_bf16(d.x, d.y);
}

// c ? a : b as one select instruction (keeps the compiler from turning a choice
// between two elements of a register array into an indexed local-memory load).
__device__ __forceinline__ float selp(bool c, float a, float b) {
    float r;
    asm("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %3, 0;\n\tselp.f32 %0, %1, %2, p;\n\t}"
        : "=f"(r)
        : "f"(a), "f"(b), "r"((int)c));
    return r;
}

// Packed fp32 pair arithmetic (one instruction for both lanes of the pair).
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// exp(a - b) for a pair, as 2^((a - b) log2 e) (ex2_approx: kda_internal.cuh).
// The difference is formed first (exact when a and b are close, as cumulative
// decays within a block are), so large |a|, |b| cost no accuracy.
__device__ __forceinline__ float2 exp_diff2(float2 a, float2 b) {
    const float2 t = __fmul2_rn(__ffma2_rn(b, make_float2(-1.f, -1.f), a), make_float2(kLog2e, kLog2e));
    return make_float2(ex2_approx(t.x), ex2_approx(t.y));
}

// prep_log_alpha (kda_internal.cuh) for a pair, the softplus polynomial as packed
// fused multiply-adds.
__device__ __forceinline__ float2 prep_log_alpha2(float2 x, unsigned prep) {
    if (prep & KDA_PREP_GATE_SOFTPLUS) {
        const float2 u = make_float2(ex2_approx(-fabsf(x.x) * kLog2e), ex2_approx(-fabsf(x.y) * kLog2e));
        float2 p = make_float2(l1p_coef(8), l1p_coef(8));
#pragma unroll
        for (int i = 7; i >= 0; --i) p = __ffma2_rn(p, u, make_float2(l1p_coef(i), l1p_coef(i)));
        p = __fmul2_rn(p, u);
        x = make_float2(-(fmaxf(x.x, 0.f) + p.x), -(fmaxf(x.y, 0.f) + p.y));
    }
    return make_float2(fmaxf(x.x, kLogAlphaFloor), fmaxf(x.y, kLogAlphaFloor));
}

__device__ __forceinline__ void split1(float a, __nv_bfloat16& hi, __nv_bfloat16& lo) {
    hi = __float2bfloat16_rn(a);
    lo = __float2bfloat16_rn(a - __bfloat162float(hi));
}

}  // namespace tc
}  // namespace kda
