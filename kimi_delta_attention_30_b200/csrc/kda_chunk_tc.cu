// Tensor-core (tcgen05) chunkwise prefill for bf16, d_k = d_v = 128.
#include "kda_internal.cuh"

namespace kda {

extern const char* const kTcKernelNames[] = {"tc_intra", "tc_recur"};
extern const int kTcKernelCount = 2;

bool tc_available() { return false; }

size_t tc_workspace_bytes(int n_chunks, int H, int C) { return 0; }

cudaError_t launch_tc_prefill(const void*, const void*, const void*, const void*, const void*, const float*, void*,
                              float*, const ChunkMap&, const SeqMap&, int, int, int, int, void*, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace kda
