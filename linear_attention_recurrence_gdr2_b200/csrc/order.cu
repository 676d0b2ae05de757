// Longest-first processing order for packed variable-length batches.
//
// Each (sequence, head) of the chunk forward is one CTA whose run time grows
// with the sequence's chunk count. The hardware starts CTAs roughly in block
// order, so handing out the longest sequences first (longest-processing-time
// first) keeps long sequences from starting last and running alone at the
// end. This kernel writes that order: order[i] is the index of the sequence
// with the i-th largest chunk count (ties by index), computed on the device
// from cu_seqlens so the host never reads it. One CTA bitonic-sorts packed
// (chunk count, index) keys in shared memory; above kMaxSortSeqs sequences it
// writes the identity order instead.
#include "common.cuh"
#include "kernels.h"

namespace gdr2 {
namespace {

constexpr int kSortThreads = 1024;

__global__ void __launch_bounds__(kSortThreads)
order_by_length_kernel(const int32_t *__restrict__ cu_seqlens, int N, int32_t *__restrict__ order)
{
    extern __shared__ uint32_t keys[];
    const int tid = threadIdx.x;
    if (N > kMaxSortSeqs) {
        for (int i = tid; i < N; i += kSortThreads) order[i] = i;
        return;
    }
    int P = 1;
    while (P < N) P <<= 1;
    for (int i = tid; i < P; i += kSortThreads) {
        uint32_t key = 0xFFFFFFFFu;
        if (i < N) {
            const int64_t len = (int64_t)cu_seqlens[i + 1] - cu_seqlens[i];
            int64_t nc = (len + 63) / 64;
            if (nc < 0) nc = 0;
            if (nc > 65535) nc = 65535;
            key = ((uint32_t)(65535 - nc) << 16) | (uint32_t)i;  // ascending key = descending length
        }
        keys[i] = key;
    }
    __syncthreads();
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = tid; i < P; i += kSortThreads) {
                const int l = i ^ j;
                if (l > i) {
                    const uint32_t a = keys[i], b = keys[l];
                    const bool ascending = (i & k) == 0;
                    if ((a > b) == ascending) {
                        keys[i] = b;
                        keys[l] = a;
                    }
                }
            }
            __syncthreads();
        }
    }
    for (int i = tid; i < N; i += kSortThreads) order[i] = (int32_t)(keys[i] & 0xFFFFu);
}

}  // namespace

size_t order_bytes(int64_t num_seqs)
{
    return (size_t)((num_seqs * 4 + 255) / 256 * 256);
}

cudaError_t launch_order_by_length(const int32_t *cu_seqlens, int64_t num_seqs, int32_t *order,
                                   cudaStream_t stream)
{
    if (num_seqs <= 0) return cudaSuccess;
    int P = 1;
    while (P < num_seqs && P <= kMaxSortSeqs) P <<= 1;
    const size_t smem = num_seqs > kMaxSortSeqs ? 0 : (size_t)P * sizeof(uint32_t);
    if (smem > 48 * 1024) {
        cudaError_t e = ensure_dynamic_smem((const void *)order_by_length_kernel, (int)smem);
        if (e != cudaSuccess) return e;
    }
    order_by_length_kernel<<<1, kSortThreads, smem, stream>>>(cu_seqlens, (int)num_seqs, order);
    return cudaGetLastError();
}

}  // namespace gdr2
