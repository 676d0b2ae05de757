// C ABI of the Gated Delta Rule-2 library: argument validation and dispatch.
// Declarations and the full contract are in include/gdr2.h.
#include "../../include/gdr2.h"
#include "../../include/gdr2_testing.h"
#include "kernels.h"

#include <cuda_runtime.h>

namespace {

constexpr int kVersion = 300;  // 0.3.0
constexpr uint32_t kPrologueMask =
    GDR2_PROLOGUE_QK_L2NORM | GDR2_PROLOGUE_GATE_SIGMOID | GDR2_PROLOGUE_DECAY_SOFTPLUS;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_dim(int64_t d) { return d == 64 || d == 128; }

gdr2_status check_dims(int64_t d_k, int64_t d_v)
{
    if (d_k <= 0 || d_v <= 0) return GDR2_ERR_INVALID_ARG;
    if (d_k != d_v || !supported_dim(d_k)) return GDR2_ERR_UNSUPPORTED;
    return GDR2_OK;
}

}  // namespace

namespace gdr2 {

gdr2_status chunk_fwd_min_workspace(int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                                    int64_t num_seqs, gdr2_dtype dtype, size_t *bytes)
{
    if (B < 0 || T < 0 || H <= 0 || num_seqs < 0) return GDR2_ERR_INVALID_ARG;
    if (dtype != GDR2_FP32 && dtype != GDR2_BF16) return GDR2_ERR_INVALID_ARG;
    gdr2_status st = check_dims(d_k, d_v);
    if (st != GDR2_OK) return st;
    // A packed batch of several sequences (the only case with num_seqs != B)
    // needs room for its longest-first processing order.
    *bytes = (B == 1 && num_seqs > 1) ? order_bytes(num_seqs) : 0;
    return GDR2_OK;
}

}  // namespace gdr2

extern "C" {

const char *gdr2_status_string(gdr2_status s)
{
    switch (s) {
    case GDR2_OK: return "ok";
    case GDR2_ERR_INVALID_ARG: return "invalid argument";
    case GDR2_ERR_UNSUPPORTED: return "unsupported configuration";
    case GDR2_ERR_WORKSPACE: return "workspace missing or too small";
    case GDR2_ERR_CUDA: return "CUDA error";
    case GDR2_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    }
    return "unknown status";
}

int gdr2_version(void) { return kVersion; }

gdr2_status gdr2_chunk_fwd_workspace_size(int64_t B, int64_t T, int64_t H, int64_t d_k,
                                          int64_t d_v, int64_t num_seqs, gdr2_dtype dtype,
                                          size_t *bytes)
{
    if (!bytes) return GDR2_ERR_INVALID_ARG;
    size_t min_bytes = 0;
    gdr2_status st = gdr2::chunk_fwd_min_workspace(B, T, H, d_k, d_v, num_seqs, dtype, &min_bytes);
    if (st != GDR2_OK) return st;
    // A packed batch of several sequences needs its processing order; a
    // fixed-length batch of few long sequences may use the segment split.
    *bytes = (B == 1 && num_seqs > 1)
                 ? min_bytes
                 : gdr2::plan_segments(B, T, H, d_k, dtype == GDR2_BF16).ws_bytes;
    if (*bytes < min_bytes) *bytes = min_bytes;
    return GDR2_OK;
}

gdr2_status gdr2_chunk_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                           const void *b, const void *w, const float *init_state,
                           const int32_t *cu_seqlens, int64_t B, int64_t T, int64_t H,
                           int64_t d_k, int64_t d_v, int64_t num_seqs, gdr2_dtype dtype,
                           void *o, float *final_state, void *workspace,
                           size_t workspace_bytes, void *stream)
{
    return gdr2_chunk_fwd_preact(q, k, v, log_alpha, b, w, init_state, cu_seqlens, B, T, H, d_k, d_v,
                                 num_seqs, dtype, o, final_state, workspace, workspace_bytes, 0u, stream);
}

gdr2_status gdr2_chunk_fwd_preact(const void *q, const void *k, const void *v, const float *log_alpha,
                                  const void *b, const void *w, const float *init_state,
                                  const int32_t *cu_seqlens, int64_t B, int64_t T, int64_t H,
                                  int64_t d_k, int64_t d_v, int64_t num_seqs, gdr2_dtype dtype,
                                  void *o, float *final_state, void *workspace,
                                  size_t workspace_bytes, uint32_t prologue, void *stream)
{
    if (prologue & ~kPrologueMask) return GDR2_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H <= 0 || num_seqs < 0) return GDR2_ERR_INVALID_ARG;
    if (dtype != GDR2_FP32 && dtype != GDR2_BF16) return GDR2_ERR_INVALID_ARG;
    gdr2_status st = check_dims(d_k, d_v);
    if (st != GDR2_OK) return st;
    if (cu_seqlens) {
        if (B != 1) return GDR2_ERR_INVALID_ARG;
    } else if (num_seqs != B) {
        return GDR2_ERR_INVALID_ARG;
    }
    if (H > 65535 || num_seqs > 65535) return GDR2_ERR_UNSUPPORTED;
    const int64_t tokens = B * T;
    if (tokens > 0) {
        const void *ptrs[] = {q, k, v, log_alpha, b, w, o};
        for (const void *p : ptrs)
            if (!p || !aligned16(p)) return GDR2_ERR_INVALID_ARG;
    }
    if (init_state && !aligned16(init_state)) return GDR2_ERR_INVALID_ARG;
    if (final_state && !aligned16(final_state)) return GDR2_ERR_INVALID_ARG;
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return GDR2_ERR_INVALID_ARG;
    size_t need = 0;
    st = gdr2::chunk_fwd_min_workspace(B, T, H, d_k, d_v, num_seqs, dtype, &need);
    if (st != GDR2_OK) return st;
    if (need > 0 && (!workspace || workspace_bytes < need)) return GDR2_ERR_WORKSPACE;
    if ((need > 0 || workspace_bytes > 0) && workspace && !aligned16(workspace)) return GDR2_ERR_INVALID_ARG;
    if (num_seqs == 0) return GDR2_OK;
    // segment split when the workspace holds it (fixed-length bf16 batches only)
    gdr2::SegPlan plan{1, 0, 0};
    if (!cu_seqlens) {
        plan = gdr2::plan_segments(B, T, H, d_k, dtype == GDR2_BF16);
        if (plan.nseg > 1 && (!workspace || workspace_bytes < plan.ws_bytes)) plan = gdr2::SegPlan{1, 0, 0};
    }

    gdr2::ChunkArgs a;
    a.q = q; a.k = k; a.v = v; a.b = b; a.w = w;
    a.log_alpha = log_alpha;
    a.init_state = init_state;
    a.cu_seqlens = cu_seqlens;
    a.order = nullptr;
    a.o = o;
    a.final_state = final_state;
    a.B = B; a.T = T; a.H = H; a.dk = d_k; a.dv = d_v; a.num_seqs = num_seqs;
    a.bf16 = dtype == GDR2_BF16;
    a.nseg = plan.nseg;
    a.seg_len = plan.seg_len;
    a.seg_ws = plan.nseg > 1 ? workspace : nullptr;
    a.pre = prologue;
    cudaError_t e = cudaSuccess;
    if (cu_seqlens && num_seqs > 1) {
        a.order = static_cast<const int32_t *>(workspace);
        e = gdr2::launch_order_by_length(cu_seqlens, num_seqs, static_cast<int32_t *>(workspace),
                                         (cudaStream_t)stream);
        if (e != cudaSuccess) return GDR2_ERR_CUDA;
    }
    if (gdr2::chunk_tc_supported(a)) {
        e = gdr2::launch_chunk_tc(a, (cudaStream_t)stream);
        if (e == cudaSuccess && a.nseg > 1) e = gdr2::launch_segment_fix(a, (cudaStream_t)stream);
    } else {
        e = gdr2::launch_chunk_simt(a, (cudaStream_t)stream);
    }
    return e == cudaSuccess ? GDR2_OK : GDR2_ERR_CUDA;
}

gdr2_status gdr2_chunk_bwd_workspace_size(int64_t B, int64_t T, int64_t H, int64_t d_k,
                                          int64_t d_v, int64_t num_seqs, gdr2_dtype dtype,
                                          size_t *bytes)
{
    if (!bytes) return GDR2_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H <= 0 || num_seqs < 0) return GDR2_ERR_INVALID_ARG;
    if (dtype != GDR2_FP32 && dtype != GDR2_BF16) return GDR2_ERR_INVALID_ARG;
    gdr2_status st = check_dims(d_k, d_v);
    if (st != GDR2_OK) return st;
    *bytes = gdr2::bwd_workspace_bytes(B * T, H, d_k, num_seqs);
    return GDR2_OK;
}

gdr2_status gdr2_chunk_bwd(const void *q, const void *k, const void *v, const float *log_alpha,
                           const void *b, const void *w, const float *init_state,
                           const int32_t *cu_seqlens, const void *d_o, const float *d_final_state,
                           int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                           int64_t num_seqs, gdr2_dtype dtype, void *dq, void *dk, void *dv,
                           float *d_log_alpha, void *db, void *dw, float *d_init_state,
                           void *workspace, size_t workspace_bytes, void *stream)
{
    if (B < 0 || T < 0 || H <= 0 || num_seqs < 0) return GDR2_ERR_INVALID_ARG;
    if (dtype != GDR2_FP32 && dtype != GDR2_BF16) return GDR2_ERR_INVALID_ARG;
    gdr2_status st = check_dims(d_k, d_v);
    if (st != GDR2_OK) return st;
    if (cu_seqlens) {
        if (B != 1) return GDR2_ERR_INVALID_ARG;
    } else if (num_seqs != B) {
        return GDR2_ERR_INVALID_ARG;
    }
    if (H > 65535 || num_seqs * H > 0x7fffffffLL) return GDR2_ERR_UNSUPPORTED;
    const int64_t tokens = B * T;
    if (tokens > 0) {
        const void *ptrs[] = {q, k, v, log_alpha, b, w, d_o, dq, dk, dv, d_log_alpha, db, dw};
        for (const void *p : ptrs)
            if (!p || !aligned16(p)) return GDR2_ERR_INVALID_ARG;
    }
    const void *opt[] = {init_state, d_final_state, d_init_state};
    for (const void *p : opt)
        if (p && !aligned16(p)) return GDR2_ERR_INVALID_ARG;
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return GDR2_ERR_INVALID_ARG;
    if (num_seqs == 0) return GDR2_OK;
    const size_t need = gdr2::bwd_workspace_bytes(tokens, H, d_k, num_seqs);
    if (!workspace || workspace_bytes < need) return GDR2_ERR_WORKSPACE;
    if (!aligned16(workspace)) return GDR2_ERR_INVALID_ARG;
    if (gdr2::bwd_slots(tokens, num_seqs) > 0x7fffffffLL) return GDR2_ERR_UNSUPPORTED;

    gdr2::BwdArgs a;
    a.q = q; a.k = k; a.v = v; a.b = b; a.w = w; a.d_o = d_o;
    a.log_alpha = log_alpha;
    a.init_state = init_state;
    a.d_final = d_final_state;
    a.cu_seqlens = cu_seqlens;
    a.dq = dq; a.dk = dk; a.dv = dv; a.db = db; a.dw = dw;
    a.d_log_alpha = d_log_alpha;
    a.d_init_state = d_init_state;
    a.workspace = workspace;
    a.B = B; a.T = T; a.H = H; a.d = d_k; a.num_seqs = num_seqs;
    a.bf16 = dtype == GDR2_BF16;
    return gdr2::launch_chunk_bwd(a, (cudaStream_t)stream) == cudaSuccess ? GDR2_OK : GDR2_ERR_CUDA;
}

gdr2_status gdr2_recurrent_step(const void *q, const void *k, const void *v,
                                const float *log_alpha, const void *b, const void *w,
                                float *state, int64_t N, int64_t H, int64_t d_k, int64_t d_v,
                                gdr2_dtype dtype, void *o, void *stream)
{
    return gdr2_recurrent_step_preact(q, k, v, log_alpha, b, w, state, N, H, d_k, d_v, dtype, o, 0u,
                                      stream);
}

gdr2_status gdr2_recurrent_step_preact(const void *q, const void *k, const void *v,
                                       const float *log_alpha, const void *b, const void *w,
                                       float *state, int64_t N, int64_t H, int64_t d_k, int64_t d_v,
                                       gdr2_dtype dtype, void *o, uint32_t prologue, void *stream)
{
    if (prologue & ~kPrologueMask) return GDR2_ERR_INVALID_ARG;
    if (N < 0 || H <= 0) return GDR2_ERR_INVALID_ARG;
    if (dtype != GDR2_FP32 && dtype != GDR2_BF16) return GDR2_ERR_INVALID_ARG;
    gdr2_status st = check_dims(d_k, d_v);
    if (st != GDR2_OK) return st;
    if (N * H > 0x7fffffffLL) return GDR2_ERR_UNSUPPORTED;
    if (N == 0) return GDR2_OK;
    const void *ptrs[] = {q, k, v, log_alpha, b, w, state, o};
    for (const void *p : ptrs)
        if (!p || !aligned16(p)) return GDR2_ERR_INVALID_ARG;

    gdr2::DecodeArgs a;
    a.q = q; a.k = k; a.v = v; a.b = b; a.w = w;
    a.log_alpha = log_alpha;
    a.state = state;
    a.o = o;
    a.N = N; a.H = H; a.dk = d_k; a.dv = d_v;
    a.bf16 = dtype == GDR2_BF16;
    a.pre = prologue;
    cudaError_t e = gdr2::launch_decode(a, (cudaStream_t)stream);
    return e == cudaSuccess ? GDR2_OK : GDR2_ERR_CUDA;
}

gdr2_status gdr2_qed_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                         const void *b, const void *w, const float *strength,
                         const float *direction, uint32_t flags, const float *init_state,
                         const int32_t *cu_seqlens, int64_t B, int64_t T, int64_t H,
                         int64_t d_k, int64_t d_v, int64_t num_seqs, gdr2_dtype dtype,
                         void *o, float *final_state, void *stream)
{
    if (flags & ~(GDR2_QED_GATE | GDR2_QED_PROJECT)) return GDR2_ERR_INVALID_ARG;
    if (B < 0 || T < 0 || H <= 0 || num_seqs < 0) return GDR2_ERR_INVALID_ARG;
    if (dtype != GDR2_FP32 && dtype != GDR2_BF16) return GDR2_ERR_INVALID_ARG;
    gdr2_status st = check_dims(d_k, d_v);
    if (st != GDR2_OK) return st;
    if (cu_seqlens) {
        if (B != 1) return GDR2_ERR_INVALID_ARG;
    } else if (num_seqs != B) {
        return GDR2_ERR_INVALID_ARG;
    }
    if (H > 65535 || num_seqs * H > 0x7fffffffLL) return GDR2_ERR_UNSUPPORTED;
    if (!strength || (reinterpret_cast<uintptr_t>(strength) & 3u)) return GDR2_ERR_INVALID_ARG;
    if (direction && (reinterpret_cast<uintptr_t>(direction) & 3u)) return GDR2_ERR_INVALID_ARG;
    if (B * T > 0) {
        const void *ptrs[] = {q, k, v, log_alpha, b, w, o};
        for (const void *p : ptrs)
            if (!p || !aligned16(p)) return GDR2_ERR_INVALID_ARG;
    }
    if (init_state && !aligned16(init_state)) return GDR2_ERR_INVALID_ARG;
    if (final_state && !aligned16(final_state)) return GDR2_ERR_INVALID_ARG;
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return GDR2_ERR_INVALID_ARG;
    if (num_seqs == 0) return GDR2_OK;
    gdr2::QedArgs a;
    a.q = q; a.k = k; a.v = v; a.b = b; a.w = w;
    a.log_alpha = log_alpha;
    a.strength = strength;
    a.direction = direction;
    a.flags = flags;
    a.init_state = init_state;
    a.cu_seqlens = cu_seqlens;
    a.o = o;
    a.final_state = final_state;
    a.B = B; a.T = T; a.H = H; a.dk = d_k; a.dv = d_v; a.num_seqs = num_seqs;
    a.bf16 = dtype == GDR2_BF16;
    cudaError_t e = gdr2::launch_qed(a, (cudaStream_t)stream);
    return e == cudaSuccess ? GDR2_OK : GDR2_ERR_CUDA;
}

gdr2_status gdr2_check_device_error(void *stream)
{
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return GDR2_ERR_CUDA;
    int code = 0, seg_code = 0;
    if (gdr2::chunk_tc_read_and_clear_error(&code) != cudaSuccess) return GDR2_ERR_CUDA;
    if (gdr2::seg_read_and_clear_error(&seg_code) != cudaSuccess) return GDR2_ERR_CUDA;
    return (code || seg_code) ? GDR2_ERR_DEVICE_TIMEOUT : GDR2_OK;
}

gdr2_status gdr2_selftest_bounded_wait(uint32_t timeout_us, void *stream)
{
    if (timeout_us == 0 || timeout_us > 2000000u) return GDR2_ERR_INVALID_ARG;
    return gdr2::chunk_tc_wait_selftest(timeout_us, (cudaStream_t)stream) == cudaSuccess ? GDR2_OK
                                                                                         : GDR2_ERR_CUDA;
}

}  // extern "C"
