// Internal launch interface between the C ABI (gdr2_api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdr2.h"

namespace gdr2 {

// Workspace a chunk forward cannot run without (the packed-batch order); the
// public size query adds the optional segment split on top.
gdr2_status chunk_fwd_min_workspace(int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                                    int64_t num_seqs, gdr2_dtype dtype, size_t *bytes);

struct DecodeArgs {
    const void *q, *k, *v, *b, *w;
    const float *log_alpha;
    float *state;
    void *o;
    int64_t N, H, dk, dv;
    bool bf16;
    uint32_t pre = 0;          // GDR2_PROLOGUE_* flags applied on load
};

struct QedArgs {
    const void *q, *k, *v, *b, *w;
    const float *log_alpha;
    const float *strength;     // [H]
    const float *direction;    // [H, dk] or null (the query)
    uint32_t flags;            // GDR2_QED_*
    const float *init_state;   // may be null
    const int32_t *cu_seqlens; // may be null
    void *o;
    float *final_state;        // may be null
    int64_t B, T, H, dk, dv, num_seqs;
    bool bf16;
};
cudaError_t launch_qed(const QedArgs &a, cudaStream_t stream);

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
    // Segment-parallel scan (fixed-length bf16 batches of few long sequences;
    // see segments.cu): nseg segments of seg_len tokens per sequence, scratch
    // in seg_ws. nseg == 1: one serial pass per (sequence, head).
    int nseg = 1;
    int64_t seg_len = 0;
    void *seg_ws = nullptr;
    uint32_t pre = 0;          // GDR2_PROLOGUE_* flags applied on load
};

// The fused prologue's element-wise activations (fp32).
__device__ __forceinline__ float pre_sigmoid(float x) { return 1.f / (1.f + expf(-x)); }
__device__ __forceinline__ float pre_neg_softplus(float x) { return x > 20.f ? -x : -log1pf(expf(x)); }

// Segment plan of the tensor-core chunk forward: how many segments each
// sequence of a fixed-length batch is split into (1 = none), and the scratch
// the split needs.
struct SegPlan {
    int nseg;
    int64_t seg_len;   // tokens per segment (a multiple of 64)
    size_t ws_bytes;   // psi (tokens x H x 128 bf16) + two [N][nseg][H][128][128] fp32 arrays
};
SegPlan plan_segments(int64_t B, int64_t T, int64_t H, int64_t d, bool bf16);
// Byte offsets inside the segment scratch.
size_t seg_psi_offset();
size_t seg_state_offset(int64_t B, int64_t T, int64_t H);
size_t seg_phi_offset(int64_t B, int64_t T, int64_t H, int nseg);

// After the segmented chunk forward: chain the segment states, write the
// final states and add each later segment's entry-state contribution to o.
cudaError_t launch_segment_fix(const ChunkArgs &a, cudaStream_t stream);
// Reads and clears the segment correction's device error word (nonzero: a
// bounded wait gave up; the low byte is the wait site).
cudaError_t seg_read_and_clear_error(int *code);

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream);

// Gate-aware backward (bwd.cu): the vector-Jacobian product of the recurrence.
struct BwdArgs {
    const void *q, *k, *v, *b, *w, *d_o;
    const float *log_alpha;
    const float *init_state;    // may be null (zero)
    const float *d_final;       // may be null (zero)
    const int32_t *cu_seqlens;  // may be null
    void *dq, *dk, *dv, *db, *dw;
    float *d_log_alpha;
    float *d_init_state;        // may be null
    void *workspace;            // bwd_workspace_bytes(), 16-byte aligned
    int64_t B, T, H, d, num_seqs;
    bool bf16;
};
// Checkpoint slots (chunk-start states and chunk-end cotangents) of a batch.
int64_t bwd_slots(int64_t tokens, int64_t num_seqs);
size_t bwd_workspace_bytes(int64_t tokens, int64_t H, int64_t d, int64_t num_seqs);
cudaError_t launch_chunk_bwd(const BwdArgs &a, cudaStream_t stream);

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
