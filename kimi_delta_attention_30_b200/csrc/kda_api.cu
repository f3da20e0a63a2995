// Host side of the C ABI declared in include/kda.h: argument validation,
// workspace planning, the sequence table and kernel dispatch.  Nothing here
// allocates device memory; all scratch lives in the caller's workspace.
#include <algorithm>
#include <cstring>
#include <mutex>
#include <vector>

#include "kda_internal.cuh"

namespace kda {

cudaError_t launch_tc_prefill(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                              const float* init_state, void* o, float* final_state, const ChunkMap& cmap,
                              const SeqMap& smap, int n_chunks, int n_seqs, int H, int C, void* tc_ws,
                              unsigned prep, cudaStream_t stream, unsigned long long stall_intra_ns,
                              unsigned long long stall_recur_ns);
size_t tc_workspace_bytes(int n_chunks, int H, int C);
bool tc_available();
bool tc_supports(int C);
int tc_chunk();

TimingHook& timing_hook() {
    static thread_local TimingHook hook{{nullptr}, 0, 0};
    return hook;
}

// kda_set_test_wait_limit: armed per host thread, consumed by the next
// tensor-core prefill from that thread.
struct TestWait {
    unsigned kernels;
    unsigned long long ns;
};
TestWait& test_wait() {
    static thread_local TestWait w{0u, 0ull};
    return w;
}

extern const char* const kTcKernelNames[];
extern const int kTcKernelCount;

namespace {

constexpr size_t kAlign = 256;
const char* const kSimtKernelNames[] = {"k1_cumsum", "k2_wy", "k3_state", "k4_output"};

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Sequence tables reach the device as kernel arguments: the launch copies its
// parameters when it is issued, so the host neither waits for the stream nor
// keeps a buffer alive past the call (a copy from pageable host memory would
// first wait for the stream's earlier work).  One launch carries up to
// kTableBatch entries (16 KiB of parameters).
constexpr int kTableBatch = 1024;
struct TableBatch {
    SeqInfo e[kTableBatch];
};

__global__ void __launch_bounds__(256) seq_table_write(SeqInfo* __restrict__ dst, int n, const __grid_constant__ TableBatch b) {
    for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = b.e[i];
}

// The per-chunk table (first token, length, sequence, index in the sequence), one
// thread per chunk, from the natural-order sequence table written just before.
__global__ void __launch_bounds__(256) chunk_table_fill(const SeqInfo* __restrict__ seqs, int n_seqs, int n_chunks,
                                                        int C, int4* __restrict__ dst) {
    const int c = (int)(blockIdx.x * blockDim.x + threadIdx.x);
    if (c >= n_chunks) return;
    int lo = 0, hi = n_seqs - 1;
    while (lo < hi) {   // last sequence whose first chunk is <= c
        const int mid = (lo + hi + 1) >> 1;
        if (seqs[mid].chunk0 <= c) lo = mid; else hi = mid - 1;
    }
    const SeqInfo sq = seqs[lo];
    const int idx = c - sq.chunk0;
    dst[c] = make_int4(sq.tok0 + idx * C, min(C, sq.len - idx * C), sq.seq, idx);
}

// the per-chunk table follows the two sequence tables
int4* chunk_table(SeqInfo* tables, size_t n_seqs) { return reinterpret_cast<int4*>(tables + 2 * n_seqs); }

// natural order then longest first, 2 n_seqs entries at `dst`, then the per-chunk
// table of n_chunks entries of C tokens; returns the number of launches (with `mark`,
// timing-hook event i follows the i-th of them)
int upload_tables(SeqInfo* dst, const std::vector<SeqInfo>& natural, const std::vector<SeqInfo>& by_len,
                  int n_chunks, int C, cudaStream_t s, cudaError_t* err, bool mark = false) {
    const size_t n = natural.size();
    int launches = 0;
    TableBatch b;
    for (size_t i0 = 0; i0 < 2 * n; i0 += kTableBatch) {
        const int cnt = (int)std::min<size_t>(kTableBatch, 2 * n - i0);
        for (int i = 0; i < cnt; ++i) {
            const size_t j = i0 + i;
            b.e[i] = j < n ? natural[j] : by_len[j - n];
        }
        seq_table_write<<<1, 256, 0, s>>>(dst + i0, cnt, b);
        ++launches;
        if ((*err = cudaGetLastError()) != cudaSuccess) return launches;
        if (mark) timing_mark_abs(s, launches);
    }
    if (n_chunks > 0) {
        chunk_table_fill<<<(n_chunks + 255) / 256, 256, 0, s>>>(dst, (int)n, n_chunks, C, chunk_table(dst, n));
        ++launches;
        if ((*err = cudaGetLastError()) != cudaSuccess) return launches;
        if (mark) timing_mark_abs(s, launches);
    }
    *err = cudaSuccess;
    return launches;
}

// launches of upload_tables: the sequence-table batches, then the chunk table
int table_launches(size_t n_seqs, int n_chunks) {
    return (int)((2 * n_seqs + kTableBatch - 1) / kTableBatch) + (n_chunks > 0 ? 1 : 0);
}

// Problem geometry shared by the workspace query and the launch.
struct Plan {
    int n_seqs = 0;
    int n_chunks = 0;
    long long total_tokens = 0;
    bool varlen = false;
    std::vector<SeqInfo> natural;   // chunk0 non-decreasing (varlen only)
    std::vector<SeqInfo> by_len;    // longest first (varlen only)
};

kda_status make_plan(int B, int T, int H, int dk, int dv, int C, const int32_t* cu, int n_seqs, Plan& p) {
    if (H <= 0 || B < 0 || T < 0) return KDA_ERR_SHAPE;
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_SHAPE;
    if (C != 64 && C != 128) return KDA_ERR_CHUNK;
    if (cu == nullptr) {
        p.n_seqs = B;
        long long ncps = (T + C - 1) / C;
        if ((long long)B * ncps > 0x7fffffffLL || (long long)B * T > 0x7fffffffLL) return KDA_ERR_SHAPE;
        p.n_chunks = (int)(B * ncps);
        p.total_tokens = (long long)B * T;
        return KDA_OK;
    }
    if (B != 1 || n_seqs < 1) return KDA_ERR_SEQLENS;
    if (cu[0] != 0 || cu[n_seqs] != T) return KDA_ERR_SEQLENS;
    p.varlen = true;
    p.n_seqs = n_seqs;
    p.total_tokens = T;
    p.natural.resize(n_seqs);
    long long chunks = 0;
    for (int s = 0; s < n_seqs; ++s) {
        if (cu[s + 1] < cu[s]) return KDA_ERR_SEQLENS;
        int len = cu[s + 1] - cu[s];
        p.natural[s] = SeqInfo{cu[s], len, (int)chunks, s};
        chunks += (len + C - 1) / C;
    }
    if (chunks > 0x7fffffffLL) return KDA_ERR_SHAPE;
    p.n_chunks = (int)chunks;
    p.by_len = p.natural;
    std::stable_sort(p.by_len.begin(), p.by_len.end(),
                     [](const SeqInfo& a, const SeqInfo& b) { return a.len > b.len; });
    return KDA_OK;
}

// Workspace layout: [sequence tables, chunk table][algorithm scratch]
size_t table_bytes(const Plan& p) {
    return p.varlen ? align_up(2 * sizeof(SeqInfo) * (size_t)p.n_seqs + sizeof(int4) * (size_t)p.n_chunks) : 0;
}

struct SimtLayout {
    size_t off[6];
    size_t total;
};

SimtLayout simt_layout(const Plan& p, int H, int dk, int dv) {
    SimtLayout L;
    size_t o = table_bytes(p);
    const size_t tok = (size_t)p.total_tokens * H;
    L.off[0] = o; o = align_up(o + tok * dk * sizeof(float));               // g
    L.off[1] = o; o = align_up(o + tok * dv * sizeof(float));               // U
    L.off[2] = o; o = align_up(o + tok * dk * sizeof(float));               // Wk
    L.off[3] = o; o = align_up(o + tok * dv * sizeof(float));               // W
    L.off[4] = o; o = align_up(o + (size_t)p.n_chunks * H * dk * dv * sizeof(float));  // S_chunk
    L.off[5] = o; o = align_up(o + tok * dk * sizeof(float));               // g, low part
    L.total = o;
    return L;
}

// Backward workspace: the CUDA-core forward's scratch, then the gradient scratch.
struct BwdLayout {
    SimtLayout fwd;
    size_t off[12];
    size_t tc = 0, o_scratch = 0, T = 0;   // tensor-core recompute (0: not used)
    size_t total;
};

bool tc_shape(kda_dtype dtype, int dk, int dv, int C);

BwdLayout bwd_layout(const Plan& p, int H, int dk, int dv, int C, bool tc = false) {
    BwdLayout L;
    L.fwd = simt_layout(p, H, dk, dv);
    size_t o = L.fwd.total;
    const size_t tok = (size_t)p.total_tokens * H;
    const size_t ch = (size_t)p.n_chunks * H;
    const size_t sizes[12] = {ch * dk * dv, tok * dv, ch * C * C, tok * dk, tok * dk, tok * dk, tok * dk,
                              ch * dk, ch * C * C, ch * C * C, tok * dk, tok * dk};
    // dS_chunk dW P dQg dKd dWk dKg dGam dAt At Qg Kd
    for (int i = 0; i < 12; ++i) {
        L.off[i] = o;
        o = align_up(o + sizes[i] * sizeof(float));
    }
    if (tc) {
        L.tc = o;
        o = align_up(o + tc_workspace_bytes(p.n_chunks, H, C));
        L.o_scratch = o;
        o = align_up(o + tok * dv * sizeof(uint16_t));
        L.T = o;                                   // (I + A)^-1 per (chunk, head), fp32
        o = align_up(o + ch * C * C * sizeof(float));
    }
    L.total = o;
    return L;
}

constexpr int kBwdChunk = 64;   // the backward kernels tile by 64 tokens

bool tc_shape(kda_dtype dtype, int dk, int dv, int C) {
    return dtype == KDA_BF16 && dk == 128 && dv == 128 && tc_supports(C);
}

kda_algo resolve(kda_algo algo, kda_dtype dtype, int dk, int dv, int C) {
    if (algo != KDA_ALGO_AUTO) return algo;
    return (tc_available() && tc_shape(dtype, dk, dv, C)) ? KDA_ALGO_TC : KDA_ALGO_SIMT;
}

size_t workspace_for(const Plan& p, int H, int dk, int dv, int C, kda_algo algo) {
    if (algo == KDA_ALGO_TC) return align_up(table_bytes(p) + tc_workspace_bytes(p.n_chunks, H, C));
    return simt_layout(p, H, dk, dv).total;
}

// Device capability check, cached per device ordinal.
kda_status check_device() {
    static std::mutex mu;
    static int cached[64];
    static bool init = false;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(mu);
    if (!init) { std::fill(cached, cached + 64, -1); init = true; }
    if (dev < 0 || dev >= 64) return KDA_ERR_DEVICE;
    if (cached[dev] < 0) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return KDA_ERR_CUDA;
        cached[dev] = (major == 10 && minor == 0) ? 1 : 0;
    }
    return cached[dev] ? KDA_OK : KDA_ERR_DEVICE;
}

}  // namespace
}  // namespace kda

using namespace kda;

extern "C" {

const char* kda_status_string(int status) {
    switch (status) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_NULL: return "KDA_ERR_NULL: a required pointer is NULL";
        case KDA_ERR_SHAPE: return "KDA_ERR_SHAPE: unsupported or inconsistent sizes";
        case KDA_ERR_DTYPE: return "KDA_ERR_DTYPE: unknown dtype";
        case KDA_ERR_ALIGN: return "KDA_ERR_ALIGN: pointer not 16-byte aligned";
        case KDA_ERR_CHUNK: return "KDA_ERR_CHUNK: chunk size must be 64 or 128";
        case KDA_ERR_SEQLENS: return "KDA_ERR_SEQLENS: invalid cu_seqlens";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE: workspace missing or too small";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA: CUDA runtime error";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT: bounded device wait expired";
        case KDA_ERR_DEVICE: return "KDA_ERR_DEVICE: current device is not sm_100 (B200)";
        case KDA_ERR_SCRATCH:
            return "KDA_ERR_SCRATCH: problem needs more scratch than the built-in KDA_NOALLOC_SCRATCH_BYTES";
        default: return "KDA: unknown status";
    }
}

int kda_version(void) { return 100; }

size_t kda_chunk_fwd_workspace_size_ex(int B, int T, int H, int dk, int dv, int C, kda_dtype dtype,
                                       const int32_t* cu_seqlens_host, int n_seqs, kda_algo algo) {
    if (dtype != KDA_BF16 && dtype != KDA_F32) return 0;
    Plan p;
    if (make_plan(B, T, H, dk, dv, C, cu_seqlens_host, n_seqs, p) != KDA_OK) return 0;
    algo = resolve(algo, dtype, dk, dv, C);
    if (algo == KDA_ALGO_TC && !tc_shape(dtype, dk, dv, C)) return 0;
    if (algo == KDA_ALGO_TC && C != tc_chunk()) {
        C = tc_chunk();
        if (make_plan(B, T, H, dk, dv, C, cu_seqlens_host, n_seqs, p) != KDA_OK) return 0;
    }
    return std::max<size_t>(workspace_for(p, H, dk, dv, C, algo), kAlign);
}

size_t kda_chunk_fwd_workspace_size(int B, int T, int H, int dk, int dv, int C, kda_dtype dtype,
                                    const int32_t* cu_seqlens_host, int n_seqs) {
    return kda_chunk_fwd_workspace_size_ex(B, T, H, dk, dv, C, dtype, cu_seqlens_host, n_seqs, KDA_ALGO_AUTO);
}

kda_status kda_chunk_simt_offsets(int B, int T, int H, int dk, int dv, int C, const int32_t* cu_seqlens_host,
                                  int n_seqs, size_t offsets[5]) {
    if (!offsets) return KDA_ERR_NULL;
    Plan p;
    kda_status st = make_plan(B, T, H, dk, dv, C, cu_seqlens_host, n_seqs, p);
    if (st != KDA_OK) return st;
    SimtLayout L = simt_layout(p, H, dk, dv);
    for (int i = 0; i < 5; ++i) offsets[i] = L.off[i];
    return KDA_OK;
}

}  // extern "C"

namespace {

constexpr unsigned kPrepAll = KDA_PREP_QK_L2NORM | KDA_PREP_GATE_SOFTPLUS | KDA_PREP_BETA_SIGMOID;

kda_status chunk_fwd_impl(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                          kda_dtype dtype, unsigned prep, const float* init_state, const int32_t* cu_seqlens_host,
                          int n_seqs, int B, int T, int H, int dk, int dv, int C, void* o, float* final_state,
                          void* workspace, size_t workspace_bytes, void* stream, kda_algo algo) {
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_DTYPE;
    if (algo != KDA_ALGO_AUTO && algo != KDA_ALGO_SIMT && algo != KDA_ALGO_TC) return KDA_ERR_SHAPE;
    if (prep & ~kPrepAll) return KDA_ERR_SHAPE;
    Plan p;
    kda_status st = make_plan(B, T, H, dk, dv, C, cu_seqlens_host, n_seqs, p);
    if (st != KDA_OK) return st;
    algo = resolve(algo, dtype, dk, dv, C);
    if (algo == KDA_ALGO_TC && !tc_shape(dtype, dk, dv, C)) return KDA_ERR_SHAPE;
    if (prep != 0 && algo != KDA_ALGO_TC) return KDA_ERR_SHAPE;   // preprocessing is fused into the TC kernels
    if (algo == KDA_ALGO_TC && C != tc_chunk()) {
        // the tensor-core kernels tile by 64 tokens; the chunk form gives the
        // same result for either chunk length
        C = tc_chunk();
        if ((st = make_plan(B, T, H, dk, dv, C, cu_seqlens_host, n_seqs, p)) != KDA_OK) return st;
    }
    const bool has_tokens = p.total_tokens > 0;
    if (has_tokens && (!q || !k || !v || !log_alpha || !beta || !o)) return KDA_ERR_NULL;
    if (!workspace) return KDA_ERR_WORKSPACE;
    const void* ptrs[] = {q, k, v, log_alpha, beta, init_state, o, final_state};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDA_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return KDA_ERR_ALIGN;
    if (workspace_bytes < workspace_for(p, H, dk, dv, C, algo)) return KDA_ERR_WORKSPACE;
    if ((st = check_device()) != KDA_OK) return st;
    if (p.n_seqs == 0) return KDA_OK;

    cudaStream_t s = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    const int ncps = (int)((T + C - 1) / C);
    ChunkMap cmap{nullptr, p.n_seqs, T, C, ncps};
    SeqMap smap{nullptr, T, C, ncps};
    timing_mark(s, 0);
    if (p.varlen) {
        cudaError_t terr;
        timing_hook().base = upload_tables((SeqInfo*)ws, p.natural, p.by_len, p.n_chunks, C, s, &terr, true);
        if (terr != cudaSuccess) {
            timing_hook().n = 0;
            timing_hook().base = 0;
            return KDA_ERR_CUDA;
        }
        cmap.seqs = (const SeqInfo*)ws;
        cmap.chunks = chunk_table((SeqInfo*)ws, p.n_seqs);
        smap.order = (const SeqInfo*)ws + p.n_seqs;
    }
    cudaError_t err;
    if (algo == KDA_ALGO_SIMT) {
        SimtLayout L = simt_layout(p, H, dk, dv);
        SimtWorkspace w{(float*)(ws + L.off[0]), (float*)(ws + L.off[5]), (float*)(ws + L.off[1]),
                        (float*)(ws + L.off[2]), (float*)(ws + L.off[3]), (float*)(ws + L.off[4])};
        err = launch_simt_prefill(dtype, q, k, v, log_alpha, beta, init_state, o, final_state, cmap, smap,
                                  p.n_chunks, p.n_seqs, H, dk, dv, C, w, s);
    } else {
        const TestWait tw = test_wait();
        test_wait() = TestWait{0u, 0ull};
        err = launch_tc_prefill(q, k, v, log_alpha, beta, init_state, o, final_state, cmap, smap, p.n_chunks,
                                p.n_seqs, H, C, ws + table_bytes(p), prep, s, (tw.kernels & 1u) ? tw.ns : 0ull,
                                (tw.kernels & 2u) ? tw.ns : 0ull);
    }
    timing_hook().n = 0;
    timing_hook().base = 0;
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status segment_map_impl(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                            kda_dtype dtype, const int32_t* cu_seqlens_host, int n_seqs, int B, int T, int H, int dk,
                            int dv, int C, float* M, float* F, void* workspace, size_t workspace_bytes, void* stream) {
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_DTYPE;
    Plan p;
    kda_status st = make_plan(B, T, H, dk, dv, C, cu_seqlens_host, n_seqs, p);
    if (st != KDA_OK) return st;
    const kda_algo algo = resolve(KDA_ALGO_AUTO, dtype, dk, dv, C);
    if (algo == KDA_ALGO_TC && C != tc_chunk()) {
        C = tc_chunk();
        if ((st = make_plan(B, T, H, dk, dv, C, cu_seqlens_host, n_seqs, p)) != KDA_OK) return st;
    }
    if (!M || !F) return KDA_ERR_NULL;
    if (p.total_tokens > 0 && (!q || !k || !v || !log_alpha || !beta)) return KDA_ERR_NULL;
    if (!workspace) return KDA_ERR_WORKSPACE;
    const void* ptrs[] = {q, k, v, log_alpha, beta, M, F};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDA_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return KDA_ERR_ALIGN;
    if (workspace_bytes < workspace_for(p, H, dk, dv, C, algo)) return KDA_ERR_WORKSPACE;
    if ((st = check_device()) != KDA_OK) return st;
    if (p.n_seqs == 0) return KDA_OK;

    cudaStream_t s = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    const int ncps = (int)((T + C - 1) / C);
    ChunkMap cmap{nullptr, p.n_seqs, T, C, ncps};
    SeqMap smap{nullptr, T, C, ncps};
    timing_mark(s, 0);
    if (p.varlen) {
        cudaError_t terr;
        timing_hook().base = upload_tables((SeqInfo*)ws, p.natural, p.by_len, p.n_chunks, C, s, &terr, true);
        if (terr != cudaSuccess) {
            timing_hook().n = 0;
            timing_hook().base = 0;
            return KDA_ERR_CUDA;
        }
        cmap.seqs = (const SeqInfo*)ws;
        cmap.chunks = chunk_table((SeqInfo*)ws, p.n_seqs);
        smap.order = (const SeqInfo*)ws + p.n_seqs;
    }
    cudaError_t err;
    if (algo == KDA_ALGO_SIMT) {
        SimtLayout L = simt_layout(p, H, dk, dv);
        SimtWorkspace w{(float*)(ws + L.off[0]), (float*)(ws + L.off[5]), (float*)(ws + L.off[1]),
                        (float*)(ws + L.off[2]), (float*)(ws + L.off[3]), (float*)(ws + L.off[4])};
        err = launch_simt_segment_map(dtype, k, v, log_alpha, beta, cmap, smap, p.n_chunks, p.n_seqs, H, dk, dv, C, w,
                                      M, F, s);
    } else {
        err = launch_tc_segment_map(q, k, v, log_alpha, beta, cmap, smap, p.n_chunks, p.n_seqs, H,
                                    ws + table_bytes(p), M, F, s);
    }
    timing_hook().n = 0;
    timing_hook().base = 0;
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status decode_impl(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                       kda_dtype dtype, unsigned prep, float* state, int N, int H, int dk, int dv, void* o,
                       void* stream) {
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_DTYPE;
    if (prep & ~kPrepAll) return KDA_ERR_SHAPE;
    if (N < 0 || H <= 0 || !((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_SHAPE;
    if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_SHAPE;
    if (N == 0) return KDA_OK;
    if (!q || !k || !v || !log_alpha || !beta || !state || !o) return KDA_ERR_NULL;
    const void* ptrs[] = {q, k, v, log_alpha, beta, state, o};
    for (const void* ptr : ptrs)
        if (!aligned16(ptr)) return KDA_ERR_ALIGN;
    kda_status st = check_device();
    if (st != KDA_OK) return st;
    cudaError_t err =
        launch_decode(dtype, q, k, v, log_alpha, beta, state, N, H, dk, dv, o, prep, (cudaStream_t)stream);
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace

extern "C" {

kda_status kda_chunk_fwd_ex(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                            kda_dtype dtype, const float* init_state, const int32_t* cu_seqlens_host, int n_seqs,
                            int B, int T, int H, int dk, int dv, int C, void* o, float* final_state,
                            void* workspace, size_t workspace_bytes, void* stream, kda_algo algo) {
    return chunk_fwd_impl(q, k, v, log_alpha, beta, dtype, 0u, init_state, cu_seqlens_host, n_seqs, B, T, H, dk, dv,
                          C, o, final_state, workspace, workspace_bytes, stream, algo);
}

kda_status kda_chunk_fwd_prep(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                              kda_dtype dtype, unsigned int prep, const float* init_state,
                              const int32_t* cu_seqlens_host, int n_seqs, int B, int T, int H, int dk, int dv, int C,
                              void* o, float* final_state, void* workspace, size_t workspace_bytes, void* stream) {
    return chunk_fwd_impl(q, k, v, log_alpha, beta, dtype, prep, init_state, cu_seqlens_host, n_seqs, B, T, H, dk,
                          dv, C, o, final_state, workspace, workspace_bytes, stream, KDA_ALGO_AUTO);
}

kda_status kda_chunk_fwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                         kda_dtype dtype, const float* init_state, const int32_t* cu_seqlens_host, int n_seqs,
                         int B, int T, int H, int dk, int dv, int C, void* o, float* final_state, void* workspace,
                         size_t workspace_bytes, void* stream) {
    return kda_chunk_fwd_ex(q, k, v, log_alpha, beta, dtype, init_state, cu_seqlens_host, n_seqs, B, T, H, dk, dv,
                            C, o, final_state, workspace, workspace_bytes, stream, KDA_ALGO_AUTO);
}

kda_status kda_set_test_wait_limit(unsigned int kernels, unsigned long long limit_ns) {
    if (kernels & ~3u) return KDA_ERR_SHAPE;
    if (kernels != 0u && (limit_ns == 0ull || limit_ns > 1000000000ull)) return KDA_ERR_SHAPE;
    test_wait() = TestWait{kernels, kernels ? limit_ns : 0ull};
    return KDA_OK;
}

kda_status kda_set_timing_events(void* const* events, int n_events) {
    TimingHook& h = timing_hook();
    if (n_events < 0 || n_events > 32) return KDA_ERR_SHAPE;
    if (n_events > 0 && !events) return KDA_ERR_NULL;
    for (int i = 0; i < 32; ++i) h.ev[i] = (i < n_events) ? events[i] : nullptr;
    h.n = n_events;
    return KDA_OK;
}

int kda_chunk_fwd_kernels(int B, int T, int H, int dk, int dv, int C, kda_dtype dtype,
                          const int32_t* cu_seqlens_host, int n_seqs, kda_algo algo, const char** names,
                          int max_names) {
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_DTYPE;
    Plan p;
    kda_status st = make_plan(B, T, H, dk, dv, C, cu_seqlens_host, n_seqs, p);
    if (st != KDA_OK) return st;
    algo = resolve(algo, dtype, dk, dv, C);
    const char* const* list = (algo == KDA_ALGO_TC) ? kTcKernelNames : kSimtKernelNames;
    // the table writes come first: sequence-table batches, then the chunk table
    const int nt = p.varlen ? table_launches(p.natural.size(), p.n_chunks) : 0;
    const int n = (algo == KDA_ALGO_TC) ? kTcKernelCount : 4;
    for (int i = 0; names && i < nt + n && i < max_names; ++i)
        names[i] = i < nt ? (p.n_chunks > 0 && i == nt - 1 ? "chunk_table_fill" : "seq_table_write") : list[i - nt];
    return nt + n;
}

size_t kda_chunk_bwd_workspace_size(int B, int T, int H, int dk, int dv, int C, const int32_t* cu_seqlens_host,
                                    int n_seqs) {
    Plan p;
    if (C != 64 && C != 128) return 0;
    if (make_plan(B, T, H, dk, dv, kBwdChunk, cu_seqlens_host, n_seqs, p) != KDA_OK) return 0;
    // sized for the tensor-core recompute whenever the shape allows it (bf16 is not known here)
    return bwd_layout(p, H, dk, dv, kBwdChunk, dk == 128 && dv == 128).total;
}

kda_status kda_chunk_bwd(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                         kda_dtype dtype, const float* init_state, const int32_t* cu_seqlens_host, int n_seqs, int B,
                         int T, int H, int dk, int dv, int C, const void* d_o, const float* d_final_state, void* dq,
                         void* dk_out, void* dv_out, void* dlog_alpha, void* dbeta, float* d_init_state,
                         void* workspace, size_t workspace_bytes, void* stream) {
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_DTYPE;
    if (C != 64 && C != 128) return KDA_ERR_CHUNK;
    Plan p;
    kda_status st = make_plan(B, T, H, dk, dv, kBwdChunk, cu_seqlens_host, n_seqs, p);
    if (st != KDA_OK) return st;
    const bool has_tokens = p.total_tokens > 0;
    if (has_tokens && (!q || !k || !v || !log_alpha || !beta || !d_o || !dq || !dk_out || !dv_out || !dlog_alpha ||
                       !dbeta))
        return KDA_ERR_NULL;
    if (!workspace) return KDA_ERR_WORKSPACE;
    const void* ptrs[] = {q, k, v, log_alpha, beta, init_state, d_o, d_final_state, dq, dk_out, dv_out,
                          dlog_alpha, dbeta, d_init_state};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDA_ERR_ALIGN;
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0) return KDA_ERR_ALIGN;
    const bool use_tc = tc_available() && tc_shape(dtype, dk, dv, kBwdChunk);
    const BwdLayout L = bwd_layout(p, H, dk, dv, kBwdChunk, use_tc);
    if (workspace_bytes < L.total) return KDA_ERR_WORKSPACE;
    if ((st = check_device()) != KDA_OK) return st;
    if (p.n_seqs == 0) return KDA_OK;

    cudaStream_t s = (cudaStream_t)stream;
    char* ws = (char*)workspace;
    const int Cb = kBwdChunk;
    const int ncps = (int)((T + Cb - 1) / Cb);
    ChunkMap cmap{nullptr, p.n_seqs, T, Cb, ncps};
    SeqMap smap{nullptr, T, Cb, ncps};
    if (p.varlen) {
        cudaError_t terr;
        upload_tables((SeqInfo*)ws, p.natural, p.by_len, p.n_chunks, Cb, s, &terr);
        if (terr != cudaSuccess) return KDA_ERR_CUDA;
        cmap.seqs = (const SeqInfo*)ws;
        cmap.chunks = chunk_table((SeqInfo*)ws, p.n_seqs);
        smap.order = (const SeqInfo*)ws + p.n_seqs;
    }
    auto f = [&](size_t off) { return (float*)(ws + off); };
    BwdWorkspace w;
    w.fwd = SimtWorkspace{f(L.fwd.off[0]), f(L.fwd.off[5]), f(L.fwd.off[1]), f(L.fwd.off[2]), f(L.fwd.off[3]),
                          f(L.fwd.off[4])};
    w.dS_chunk = f(L.off[0]);
    w.dW = f(L.off[1]);
    w.P = f(L.off[2]);
    w.dQg = f(L.off[3]);
    w.dKd = f(L.off[4]);
    w.dWk = f(L.off[5]);
    w.dKg = f(L.off[6]);
    w.dGam = f(L.off[7]);
    w.dAt = f(L.off[8]);
    w.At = f(L.off[9]);
    w.Qg = f(L.off[10]);
    w.Kd = f(L.off[11]);
    w.tc_ws = use_tc ? (void*)(ws + L.tc) : nullptr;
    w.o_scratch = use_tc ? (void*)(ws + L.o_scratch) : nullptr;
    w.T = use_tc ? (float*)(ws + L.T) : nullptr;
    timing_mark(s, 0);
    cudaError_t err = launch_simt_backward(dtype, q, k, v, log_alpha, beta, init_state, d_o, d_final_state, dq,
                                           dk_out, dv_out, dlog_alpha, dbeta, d_init_state, cmap, smap, p.n_chunks,
                                           p.n_seqs, H, dk, dv, Cb, w, s);
    timing_hook().n = 0;
    return err == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // extern "C"

namespace {

// Copy the error word at `offset` of the workspace to the host after `stream` finishes.
kda_status read_error_word(const void* workspace, size_t offset, void* stream) {
    int word = 0;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&word, (const char*)workspace + offset, sizeof(int), cudaMemcpyDeviceToHost, s) !=
            cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return KDA_ERR_CUDA;
    return word == 0 ? KDA_OK : (kda_status)word;
}

}  // namespace

extern "C" {

kda_status kda_chunk_fwd_device_status(const void* workspace, kda_dtype dtype, const int32_t* cu_seqlens_host,
                                       int n_seqs, int B, int T, int H, int dk, int dv, int C, kda_algo algo,
                                       void* stream) {
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_DTYPE;
    if (algo != KDA_ALGO_AUTO && algo != KDA_ALGO_SIMT && algo != KDA_ALGO_TC) return KDA_ERR_SHAPE;
    Plan p;
    kda_status st = make_plan(B, T, H, dk, dv, C, cu_seqlens_host, n_seqs, p);
    if (st != KDA_OK) return st;
    if (!workspace) return KDA_ERR_NULL;
    if (p.n_seqs == 0 || resolve(algo, dtype, dk, dv, C) != KDA_ALGO_TC) return KDA_OK;   // nothing waited
    return read_error_word(workspace, table_bytes(p), stream);   // the tensor-core scratch starts with it
}

kda_status kda_chunk_bwd_device_status(const void* workspace, kda_dtype dtype, const int32_t* cu_seqlens_host,
                                       int n_seqs, int B, int T, int H, int dk, int dv, int C, void* stream) {
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_DTYPE;
    if (C != 64 && C != 128) return KDA_ERR_CHUNK;
    Plan p;
    kda_status st = make_plan(B, T, H, dk, dv, kBwdChunk, cu_seqlens_host, n_seqs, p);
    if (st != KDA_OK) return st;
    if (!workspace) return KDA_ERR_NULL;
    if (p.n_seqs == 0 || !(tc_available() && tc_shape(dtype, dk, dv, kBwdChunk))) return KDA_OK;
    return read_error_word(workspace, bwd_layout(p, H, dk, dv, kBwdChunk, true).tc, stream);
}

kda_status kda_chunk_segment_map(const void* q, const void* k, const void* v, const void* log_alpha,
                                 const void* beta, kda_dtype dtype, const int32_t* cu_seqlens_host, int n_seqs, int B,
                                 int T, int H, int dk, int dv, int C, float* M, float* F, void* workspace,
                                 size_t workspace_bytes, void* stream) {
    return segment_map_impl(q, k, v, log_alpha, beta, dtype, cu_seqlens_host, n_seqs, B, T, H, dk, dv, C, M, F,
                            workspace, workspace_bytes, stream);
}

kda_status kda_compose_states(const float* M, const float* F, const float* init_state, int R, int N, int H, int dk,
                              int dv, float* states, void* stream) {
    if (R < 0 || N < 0 || H <= 0 || !((dk == 64 || dk == 128) && (dv == 64 || dv == 128))) return KDA_ERR_SHAPE;
    if ((long long)N * H > 0x7fffffffLL) return KDA_ERR_SHAPE;
    if (!states || (R > 0 && (!M || !F))) return KDA_ERR_NULL;
    const void* ptrs[] = {M, F, init_state, states};
    for (const void* ptr : ptrs)
        if (ptr && !aligned16(ptr)) return KDA_ERR_ALIGN;
    kda_status st = check_device();
    if (st != KDA_OK) return st;
    if (N == 0) return KDA_OK;
    return launch_compose_states(M, F, init_state, R, N, H, dk, dv, states, (cudaStream_t)stream) == cudaSuccess
               ? KDA_OK
               : KDA_ERR_CUDA;
}

kda_status kda_decode_step(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                           kda_dtype dtype, float* state, int N, int H, int dk, int dv, void* o, void* stream) {
    return decode_impl(q, k, v, log_alpha, beta, dtype, 0u, state, N, H, dk, dv, o, stream);
}

kda_status kda_decode_step_prep(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                                kda_dtype dtype, unsigned int prep, float* state, int N, int H, int dk, int dv,
                                void* o, void* stream) {
    return decode_impl(q, k, v, log_alpha, beta, dtype, prep, state, N, H, dk, dv, o, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// kda_chunk_fwd_host: the prefill of a host-resident packed batch, in groups of
// sequences whose copies overlap the computation of their neighbours.
// ---------------------------------------------------------------------------
namespace kda {
// The first error a group's kernels recorded, kept in the host buffer's status word.
__global__ void accumulate_status(const int* __restrict__ word, int* __restrict__ acc) {
    const int w = *word;
    if (w != 0) atomicCAS(acc, 0, w);
}
}  // namespace kda

namespace {

struct HostGroup {
    int s0, s1;   // sequences [s0, s1)
};

// Consecutive sequences in groups of about equal token counts (at most n_groups,
// none empty of sequences).
std::vector<HostGroup> host_groups(const int32_t* cu, int n_seqs, int n_groups) {
    std::vector<HostGroup> g;
    const int G = std::max(1, std::min(n_groups, n_seqs));
    const long long T = cu[n_seqs];
    int s0 = 0;
    for (int i = 0; i < G && s0 < n_seqs; ++i) {
        int s1;
        if (i == G - 1) {
            s1 = n_seqs;
        } else {
            const long long target = T * (i + 1) / G;
            s1 = s0 + 1;
            while (s1 < n_seqs - (G - 1 - i) && cu[s1] < target) ++s1;
        }
        g.push_back(HostGroup{s0, s1});
        s0 = s1;
    }
    return g;
}

// Device buffer: [status word][workspace][slot 0][slot 1]; a slot holds one group's
// q, k, log alpha, v, beta, initial states, o and final states.
struct HostLayout {
    size_t ws_off = 0, ws_bytes = 0, slot_off[2] = {0, 0}, total = 0;
    size_t q = 0, k = 0, la = 0, v = 0, beta = 0, init = 0, o = 0, fin = 0;   // offsets inside a slot
};

kda_status host_layout(kda_dtype dtype, const int32_t* cu, int n_seqs, int H, int dk, int dv, int C,
                       const std::vector<HostGroup>& groups, HostLayout& L) {
    const size_t es = dtype == KDA_BF16 ? 2 : 4;
    long long max_tok = 0, max_seq = 0;
    size_t ws = 0;
    for (const HostGroup& g : groups) {
        const int ns = g.s1 - g.s0;
        std::vector<int32_t> cg(ns + 1);
        for (int i = 0; i <= ns; ++i) cg[i] = cu[g.s0 + i] - cu[g.s0];
        const size_t w = kda_chunk_fwd_workspace_size(1, cg[ns], H, dk, dv, C, dtype, cg.data(), ns);
        if (w == 0) return KDA_ERR_SHAPE;
        ws = std::max(ws, w);
        max_tok = std::max<long long>(max_tok, cg[ns]);
        max_seq = std::max<long long>(max_seq, ns);
    }
    const size_t tok = (size_t)max_tok * H, st = (size_t)max_seq * H * dk * dv * sizeof(float);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        const size_t at = o;
        o = align_up(o + bytes);
        return at;
    };
    L.q = take(tok * dk * es);
    L.k = take(tok * dk * es);
    L.la = take(tok * dk * es);
    L.v = take(tok * dv * es);
    L.beta = take(tok * es);
    L.init = take(st);
    L.o = take(tok * dv * es);
    L.fin = take(st);
    L.ws_off = kAlign;
    L.ws_bytes = ws;
    L.slot_off[0] = align_up(L.ws_off + ws);
    L.slot_off[1] = L.slot_off[0] + o;
    L.total = L.slot_off[1] + o;
    return KDA_OK;
}

// Streams and events of one call; destroyed when the call returns (the runtime
// releases them once the work queued on them has finished).
struct HostStreams {
    cudaStream_t in = nullptr, out = nullptr;
    std::vector<cudaEvent_t> ev;
    ~HostStreams() {
        for (cudaEvent_t e : ev) cudaEventDestroy(e);
        if (in) cudaStreamDestroy(in);
        if (out) cudaStreamDestroy(out);
    }
    cudaError_t make(int n_events) {
        cudaError_t e;
        if ((e = cudaStreamCreateWithFlags(&in, cudaStreamNonBlocking)) != cudaSuccess) return e;
        if ((e = cudaStreamCreateWithFlags(&out, cudaStreamNonBlocking)) != cudaSuccess) return e;
        ev.assign(n_events, nullptr);
        for (cudaEvent_t& x : ev)
            if ((e = cudaEventCreateWithFlags(&x, cudaEventDisableTiming)) != cudaSuccess) return e;
        return cudaSuccess;
    }
};

cudaError_t copy_async(void* dst, const void* src, size_t bytes, cudaMemcpyKind kind, cudaStream_t s) {
    return bytes ? cudaMemcpyAsync(dst, src, bytes, kind, s) : cudaSuccess;
}

}  // namespace

extern "C" {

size_t kda_chunk_fwd_host_buffer_size(kda_dtype dtype, const int32_t* cu_seqlens_host, int n_seqs, int H, int dk,
                                      int dv, int C, int n_groups) {
    if ((dtype != KDA_BF16 && dtype != KDA_F32) || !cu_seqlens_host || n_groups < 1) return 0;
    Plan p;
    if (make_plan(1, cu_seqlens_host[n_seqs >= 1 ? n_seqs : 0], H, dk, dv, C, cu_seqlens_host, n_seqs, p) != KDA_OK)
        return 0;
    HostLayout L;
    if (host_layout(dtype, cu_seqlens_host, n_seqs, H, dk, dv, C, host_groups(cu_seqlens_host, n_seqs, n_groups), L) !=
        KDA_OK)
        return 0;
    return L.total;
}

kda_status kda_chunk_fwd_host(const void* q, const void* k, const void* v, const void* log_alpha, const void* beta,
                              kda_dtype dtype, const float* init_state, const int32_t* cu_seqlens_host, int n_seqs,
                              int H, int dk, int dv, int C, void* o, float* final_state, int n_groups,
                              void* device_buffer, size_t device_buffer_bytes, void* stream) {
    if (dtype != KDA_BF16 && dtype != KDA_F32) return KDA_ERR_DTYPE;
    if (!cu_seqlens_host || n_seqs < 1) return KDA_ERR_SEQLENS;
    if (n_groups < 1) return KDA_ERR_SHAPE;
    const int T = cu_seqlens_host[n_seqs];
    Plan p;
    kda_status st = make_plan(1, T, H, dk, dv, C, cu_seqlens_host, n_seqs, p);
    if (st != KDA_OK) return st;
    if (T > 0 && (!q || !k || !v || !log_alpha || !beta || !o)) return KDA_ERR_NULL;
    if (!device_buffer) return KDA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(device_buffer) & (kAlign - 1)) != 0) return KDA_ERR_ALIGN;
    const std::vector<HostGroup> groups = host_groups(cu_seqlens_host, n_seqs, n_groups);
    HostLayout L;
    if ((st = host_layout(dtype, cu_seqlens_host, n_seqs, H, dk, dv, C, groups, L)) != KDA_OK) return st;
    if (device_buffer_bytes < L.total) return KDA_ERR_WORKSPACE;
    if ((st = check_device()) != KDA_OK) return st;

    const size_t es = dtype == KDA_BF16 ? 2 : 4;
    const size_t sb = (size_t)H * dk * dv * sizeof(float);
    const int G = (int)groups.size();
    cudaStream_t s = (cudaStream_t)stream;
    char* buf = (char*)device_buffer;
    HostStreams hs;
    // events: start, then per group: inputs in, computed, outputs out
    if (hs.make(1 + 3 * G) != cudaSuccess) return KDA_ERR_CUDA;
    cudaEvent_t ev0 = hs.ev[0];
    auto ev_in = [&](int g) { return hs.ev[1 + 3 * g]; };
    auto ev_comp = [&](int g) { return hs.ev[2 + 3 * g]; };
    auto ev_out = [&](int g) { return hs.ev[3 + 3 * g]; };
    const bool tc = resolve(KDA_ALGO_AUTO, dtype, dk, dv, C) == KDA_ALGO_TC;

    cudaError_t e = cudaMemsetAsync(buf, 0, sizeof(int), s);
    if (e == cudaSuccess) e = cudaEventRecord(ev0, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hs.in, ev0, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hs.out, ev0, 0);
    if (e != cudaSuccess) return KDA_ERR_CUDA;
    for (int g = 0; g < G; ++g) {
        const int s0 = groups[g].s0, ns = groups[g].s1 - s0;
        const long long t0 = cu_seqlens_host[s0], nt = cu_seqlens_host[s0 + ns] - t0;
        char* sl = buf + L.slot_off[g & 1];
        const size_t tk = (size_t)nt * H, ok = (size_t)t0 * H;
        // inputs, once the computation that last read this slot is done
        if (g >= 2) e = cudaStreamWaitEvent(hs.in, ev_comp(g - 2), 0);
        if (e == cudaSuccess) e = copy_async(sl + L.q, (const char*)q + ok * dk * es, tk * dk * es, cudaMemcpyHostToDevice, hs.in);
        if (e == cudaSuccess) e = copy_async(sl + L.k, (const char*)k + ok * dk * es, tk * dk * es, cudaMemcpyHostToDevice, hs.in);
        if (e == cudaSuccess)
            e = copy_async(sl + L.la, (const char*)log_alpha + ok * dk * es, tk * dk * es, cudaMemcpyHostToDevice, hs.in);
        if (e == cudaSuccess) e = copy_async(sl + L.v, (const char*)v + ok * dv * es, tk * dv * es, cudaMemcpyHostToDevice, hs.in);
        if (e == cudaSuccess) e = copy_async(sl + L.beta, (const char*)beta + ok * es, tk * es, cudaMemcpyHostToDevice, hs.in);
        if (e == cudaSuccess && init_state)
            e = copy_async(sl + L.init, init_state + (size_t)s0 * H * dk * dv, (size_t)ns * sb, cudaMemcpyHostToDevice, hs.in);
        if (e == cudaSuccess) e = cudaEventRecord(ev_in(g), hs.in);
        // the computation, once the inputs are in and this slot's previous outputs are out
        if (e == cudaSuccess) e = cudaStreamWaitEvent(s, ev_in(g), 0);
        if (e == cudaSuccess && g >= 2) e = cudaStreamWaitEvent(s, ev_out(g - 2), 0);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
        std::vector<int32_t> cg(ns + 1);
        for (int i = 0; i <= ns; ++i) cg[i] = cu_seqlens_host[s0 + i] - (int32_t)t0;
        st = chunk_fwd_impl(sl + L.q, sl + L.k, sl + L.v, sl + L.la, sl + L.beta, dtype, 0u,
                            init_state ? (const float*)(sl + L.init) : nullptr, cg.data(), ns, 1, (int)nt, H, dk, dv,
                            C, sl + L.o, final_state ? (float*)(sl + L.fin) : nullptr, buf + L.ws_off, L.ws_bytes,
                            stream, KDA_ALGO_AUTO);
        if (st != KDA_OK) return st;
        if (tc && ns > 0) {
            Plan pg;
            if ((st = make_plan(1, (int)nt, H, dk, dv, tc_chunk(), cg.data(), ns, pg)) != KDA_OK) return st;
            accumulate_status<<<1, 1, 0, s>>>((const int*)(buf + L.ws_off + table_bytes(pg)), (int*)buf);
            if (cudaGetLastError() != cudaSuccess) return KDA_ERR_CUDA;
        }
        if ((e = cudaEventRecord(ev_comp(g), s)) != cudaSuccess) return KDA_ERR_CUDA;
        // the outputs, once computed
        e = cudaStreamWaitEvent(hs.out, ev_comp(g), 0);
        if (e == cudaSuccess) e = copy_async((char*)o + ok * dv * es, sl + L.o, tk * dv * es, cudaMemcpyDeviceToHost, hs.out);
        if (e == cudaSuccess && final_state)
            e = copy_async(final_state + (size_t)s0 * H * dk * dv, sl + L.fin, (size_t)ns * sb, cudaMemcpyDeviceToHost, hs.out);
        if (e == cudaSuccess) e = cudaEventRecord(ev_out(g), hs.out);
        if (e != cudaSuccess) return KDA_ERR_CUDA;
    }
    // the caller's stream ends after the last copy back (the output stream runs in order)
    return cudaStreamWaitEvent(s, ev_out(G - 1), 0) == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

kda_status kda_chunk_fwd_host_device_status(const void* device_buffer, void* stream) {
    if (!device_buffer) return KDA_ERR_NULL;
    return read_error_word(device_buffer, 0, stream);
}

}  // extern "C"
