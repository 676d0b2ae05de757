// gdr2_chunk_fwd_noalloc: the chunk forward for callers that cannot hand the
// library any scratch memory. The only scratch the chunk forward uses is the
// per-sequence processing order of a packed batch; this entry point keeps it
// in a fixed device array that lives inside the library instead of in a
// caller-provided workspace, and otherwise runs exactly gdr2_chunk_fwd.
#include "../../include/gdr2.h"
#include "kernels.h"

#include <cuda_runtime.h>

#include <mutex>

namespace {

// Room for the processing order of up to kNoAllocMaxSeqs packed sequences
// (4 bytes each). Every GPU that loads the library holds this array until the
// process exits.
constexpr int64_t kNoAllocMaxSeqs = 16384;
constexpr size_t kNoAllocScratchBytes = (size_t)kNoAllocMaxSeqs * 4;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void *g_scratch_ptr[kMaxDevices];  // null until a lookup on that device succeeded

// Device address of g_noalloc_scratch on the current device (the name itself
// is only a host-side stand-in). A successful lookup is kept for the life of
// the process, which assumes the device's primary context and no
// cudaDeviceReset in between; a failed one is not kept, so a later call
// tries again.
gdr2_status scratch_for_current_device(void **ptr)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GDR2_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return GDR2_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GDR2_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *ptr = g_scratch_ptr[dev];
    return GDR2_OK;
}

}  // namespace

extern "C" gdr2_status gdr2_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                              const float *log_alpha, const void *b, const void *w,
                                              const float *init_state, const int32_t *cu_seqlens,
                                              int64_t B, int64_t T, int64_t H, int64_t d_k,
                                              int64_t d_v, int64_t num_seqs, gdr2_dtype dtype,
                                              void *o, float *final_state, void *stream)
{
    size_t need = 0;  // (without the optional segment split, which needs far more)
    gdr2_status st = gdr2::chunk_fwd_min_workspace(B, T, H, d_k, d_v, num_seqs, dtype, &need);
    if (st != GDR2_OK) return st;
    if (need > kNoAllocScratchBytes) return GDR2_ERR_UNSUPPORTED;  // more sequences than the array holds
    void *scratch = nullptr;
    if (need > 0) {
        st = scratch_for_current_device(&scratch);
        if (st != GDR2_OK) return st;
    }
    return gdr2_chunk_fwd(q, k, v, log_alpha, b, w, init_state, cu_seqlens, B, T, H, d_k, d_v,
                          num_seqs, dtype, o, final_state, scratch, need > 0 ? kNoAllocScratchBytes : 0,
                          stream);
}
