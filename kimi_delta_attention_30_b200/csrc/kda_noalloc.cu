// kda_chunk_fwd_noalloc: the chunkwise prefill for callers that cannot
// allocate device memory.
//
// Some callers have no way to obtain device scratch: a plugin host that hands
// the operator only its input and output buffers and no allocator, or a serving
// runtime whose memory pool has reserved the whole device so that a cudaMalloc
// from inside the operator would fail or would have to synchronise the device.
// This entry point needs nothing from them beyond the inputs and outputs: its
// scratch is a fixed array in device memory that belongs to the library (it is
// created when the library's code is loaded on a device and is held by every
// device that loads it until the process exits).
#include <mutex>

#include "kda_internal.cuh"

namespace {

// The library-owned scratch.  Host code sees only a host-side stand-in for this
// name, never its device address; the address is obtained per device below.
static __device__ __align__(256) unsigned char g_kda_noalloc_scratch[KDA_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch on each device ordinal, looked up once.
std::mutex g_mu;
void* g_addr[64] = {nullptr};

kda_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_CUDA;
    if (dev < 0 || dev >= 64) return KDA_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_addr[dev] == nullptr) {
        void* p = nullptr;
        // With `dev` current: the device address of the array on this device.
        if (cudaGetSymbolAddress(&p, g_kda_noalloc_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();   // reset the error state so a later, unrelated call does not report it
            return KDA_ERR_CUDA;
        }
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return KDA_OK;
}

}  // namespace

extern "C" kda_status kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const void* log_alpha,
                                            const void* beta, kda_dtype dtype, const float* init_state,
                                            const int32_t* cu_seqlens_host, int n_seqs, int B, int T, int H,
                                            int dk, int dv, int C, void* o, float* final_state, void* stream) {
    // Size check first, on the host: the same validation as kda_chunk_fwd runs
    // again inside the call below.
    const size_t need = kda_chunk_fwd_workspace_size(B, T, H, dk, dv, C, dtype, cu_seqlens_host, n_seqs);
    if (need == 0) {
        // invalid sizes: let the regular entry point report the precise reason
        return kda_chunk_fwd(q, k, v, log_alpha, beta, dtype, init_state, cu_seqlens_host, n_seqs, B, T, H, dk,
                             dv, C, o, final_state, nullptr, 0, stream);
    }
    if (need > (size_t)KDA_NOALLOC_SCRATCH_BYTES) return KDA_ERR_SCRATCH;
    void* scratch = nullptr;
    kda_status st = scratch_address(&scratch);
    if (st != KDA_OK) return st;
    // Every byte the prefill reads from its scratch is written earlier in the
    // same call, so the previous call's leftovers need no clearing.
    return kda_chunk_fwd(q, k, v, log_alpha, beta, dtype, init_state, cu_seqlens_host, n_seqs, B, T, H, dk, dv, C,
                         o, final_state, scratch, (size_t)KDA_NOALLOC_SCRATCH_BYTES, stream);
}

extern "C" kda_status kda_chunk_fwd_noalloc_device_status(kda_dtype dtype, const int32_t* cu_seqlens_host, int n_seqs,
                                                          int B, int T, int H, int dk, int dv, int C, void* stream) {
    void* scratch = nullptr;
    kda_status st = scratch_address(&scratch);
    if (st != KDA_OK) return st;
    return kda_chunk_fwd_device_status(scratch, dtype, cu_seqlens_host, n_seqs, B, T, H, dk, dv, C, KDA_ALGO_AUTO,
                                       stream);
}
