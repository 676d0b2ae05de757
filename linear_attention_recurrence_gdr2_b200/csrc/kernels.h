// Internal launch interface between the C ABI (gdr2_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace gdr2 {

struct DecodeArgs {
    const void *q, *k, *v, *b, *w;
    const float *log_alpha;
    float *state;
    void *o;
    int64_t N, H, dk, dv;
    bool bf16;
};

struct ChunkArgs {
    const void *q, *k, *v, *b, *w;
    const float *log_alpha;
    const float *init_state;   // may be null
    const int32_t *cu_seqlens; // may be null
    const int32_t *order;      // may be null: processing order of the sequences
    void *o;
    float *final_state;        // may be null
    int64_t B, T, H, dk, dv, num_seqs;
    bool bf16;
};

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

// Longest-first sequence order for packed batches (see order.cu).
constexpr int kMaxSortSeqs = 16384;
size_t order_bytes(int64_t num_seqs);
cudaError_t launch_order_by_length(const int32_t *cu_seqlens, int64_t num_seqs, int32_t *order,
                                   cudaStream_t stream);

// fp32 CUDA-core chunk forward (any dtype; the fp32 path of the library).
cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t stream);

// Tensor-core chunk forward (bf16, d_k = d_v = 128).
bool chunk_tc_supported(const ChunkArgs &a);
cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream);

// Reads and clears the tensor-core kernel's device error word (synchronous).
cudaError_t chunk_tc_read_and_clear_error(int *code);

// Failure-detection self-test: one bounded wait that runs out after timeout_us.
cudaError_t chunk_tc_wait_selftest(uint32_t timeout_us, cudaStream_t stream);

}  // namespace gdr2
