// Gated Delta Rule-2 with the QED second erase direction, token by token
// (CUDA cores, fp32 state).
//
// "The Query Knows What to Forget: A Second Erase Direction for Linear
// Attention" (thelatestinai.com listing, abstract and Table 1) adds to the
// key-directed erase a second one, taken from the query, projected orthogonal
// to the key, gated by b_t and scaled by a per-head strength; its equation (6)
// is not printed there. This kernel computes the reading the oracle states:
//   src = q_t (or a fixed per-head direction), p = src - (k.src / k.k) k
//   (with GDR2_QED_PROJECT), u = p / |p| (0 when |p|^2 <= 1e-12 |src|^2),
//   f = b . u (with GDR2_QED_GATE, else u),
//   S_t = (I - k (b . k)^T - lambda_h u f^T) Diag(alpha_t) S_{t-1} + k (w . v)^T,
//   o_t = S_t^T q_t.
// The rank-2 edit per token has no chunked form here: one CTA per (sequence,
// head, 32 value columns) runs the tokens in order. Columns of S evolve
// independently given k, u, b and alpha, so the value blocks of one head need
// no communication. Thread (warp w, lane l) keeps rows w*DK/4 .. of column l
// in registers. Every warp computes the token's direction u on its own (warp
// shuffles over the DK channels, lane l holding channels l + 32m) and keeps the
// per-channel factors in its own shared-memory slice, so a token costs two
// block barriers (the two reads of the decayed state, then the readout, summed
// over the warps); its inputs are loaded one token ahead.
#include "common.cuh"
#include "kernels.h"

namespace gdr2 {

namespace {

constexpr int kQedThreads = 128;
constexpr int kQedCols = 32;  // value columns per CTA

template <typename Tin, int DK>
__global__ void __launch_bounds__(kQedThreads)
qed_fwd_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
               const float *__restrict__ log_alpha, const Tin *__restrict__ b, const Tin *__restrict__ w,
               const float *__restrict__ strength, const float *__restrict__ direction, int flags,
               const float *__restrict__ init_state, const int32_t *__restrict__ cu_seqlens, int64_t T,
               int64_t H, int64_t DV, int64_t tokens, Tin *__restrict__ o, float *__restrict__ final_state)
{
    constexpr int ROWS = DK / 4;   // key rows per warp
    constexpr int CPL = DK / 32;   // channels per lane in the direction's reductions
    // per warp: alpha, e = b . k, k, u, f, q for every channel (written and read
    // by the same warp only)
    __shared__ float s_v[4][6][DK];
    __shared__ float s_rk[4][kQedCols], s_ru[4][kQedCols], s_o[4][kQedCols];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t unit = blockIdx.x, n = unit / H, h = unit % H;
    const int64_t j = (int64_t)kQedCols * blockIdx.y + lane;  // this thread's value column
    int64_t t_begin, t_end;
    if (cu_seqlens) {
        packed_bounds(cu_seqlens, n, tokens, t_begin, t_end);
    } else {
        t_begin = n * T;
        t_end = t_begin + T;
    }
    const float lambda = strength[h];
    const bool gate = (flags & GDR2_QED_GATE) != 0, project = (flags & GDR2_QED_PROJECT) != 0;
    float dirc[CPL];
#pragma unroll
    for (int m = 0; m < CPL; ++m) dirc[m] = direction ? direction[h * DK + lane + 32 * m] : 0.f;

    float s[ROWS];
    const int64_t sbase = (unit * DK + (int64_t)ROWS * warp) * DV + j;
#pragma unroll
    for (int i = 0; i < ROWS; ++i) s[i] = init_state ? init_state[sbase + (int64_t)i * DV] : 0.f;

    auto warp_sum = [&](float x) {
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
        return x;
    };

    // inputs of token t: channels lane + 32m of q, k, log_alpha, b; value
    // column j of v and w
    float nq[CPL], nk[CPL], nla[CPL], nb[CPL], nv = 0.f, nw = 0.f;
#pragma unroll
    for (int m = 0; m < CPL; ++m) nq[m] = nk[m] = nla[m] = nb[m] = 0.f;
    auto fetch = [&](int64_t t) {
        if (t >= t_end) return;
        const int64_t rk = (t * H + h) * DK, rv = (t * H + h) * DV;
#pragma unroll
        for (int m = 0; m < CPL; ++m) {
            const int c = lane + 32 * m;
            nq[m] = to_f32(q[rk + c]);
            nk[m] = to_f32(k[rk + c]);
            nla[m] = log_alpha[rk + c];
            nb[m] = to_f32(b[rk + c]);
        }
        nv = to_f32(v[rv + j]);
        nw = to_f32(w[rv + j]);
    };
    fetch(t_begin);
    float (&sv)[6][DK] = s_v[warp];
    for (int64_t t = t_begin; t < t_end; ++t) {
        float qc[CPL], kc[CPL], lac[CPL], bc[CPL];
#pragma unroll
        for (int m = 0; m < CPL; ++m) {
            qc[m] = nq[m]; kc[m] = nk[m]; lac[m] = nla[m]; bc[m] = nb[m];
        }
        const float z = nv * nw;
        fetch(t + 1);
        // the erase direction u from the query (or the fixed direction), in this warp
        float kk = 0.f, ks = 0.f, ss = 0.f;
#pragma unroll
        for (int m = 0; m < CPL; ++m) {
            const float src = direction ? dirc[m] : qc[m];
            kk = fmaf(kc[m], kc[m], kk);
            ks = fmaf(kc[m], src, ks);
            ss = fmaf(src, src, ss);
        }
        kk = warp_sum(kk);
        ks = warp_sum(ks);
        ss = warp_sum(ss);
        const float coef = (project && kk > 0.f) ? ks / kk : 0.f;
        float pc[CPL], pp = 0.f;
#pragma unroll
        for (int m = 0; m < CPL; ++m) {
            pc[m] = (direction ? dirc[m] : qc[m]) - coef * kc[m];
            pp = fmaf(pc[m], pc[m], pp);
        }
        pp = warp_sum(pp);
        const float inv = (pp > 1e-12f * ss && pp > 0.f) ? rsqrtf(pp) : 0.f;
#pragma unroll
        for (int m = 0; m < CPL; ++m) {
            const int c = lane + 32 * m;
            const float uc = pc[m] * inv;
            sv[0][c] = expf(lac[m]);
            sv[1][c] = bc[m] * kc[m];
            sv[2][c] = kc[m];
            sv[3][c] = uc;
            sv[4][c] = gate ? bc[m] * uc : uc;
            sv[5][c] = qc[m];
        }
        __syncwarp();
        // decay, then both reads of the decayed state (this warp's rows)
        float rk = 0.f, ru = 0.f;
#pragma unroll
        for (int i = 0; i < ROWS; ++i) {
            const int c = ROWS * warp + i;
            s[i] *= sv[0][c];
            rk = fmaf(sv[1][c], s[i], rk);
            ru = fmaf(sv[4][c], s[i], ru);
        }
        s_rk[warp][lane] = rk;
        s_ru[warp][lane] = ru;
        __syncthreads();
        rk = s_rk[0][lane] + s_rk[1][lane] + s_rk[2][lane] + s_rk[3][lane];
        ru = s_ru[0][lane] + s_ru[1][lane] + s_ru[2][lane] + s_ru[3][lane];
        const float resid = z - rk, lru = lambda * ru;
        // the edit and the readout partial sums
        float oq = 0.f;
#pragma unroll
        for (int i = 0; i < ROWS; ++i) {
            const int c = ROWS * warp + i;
            s[i] = fmaf(sv[2][c], resid, fmaf(-sv[3][c], lru, s[i]));
            oq = fmaf(sv[5][c], s[i], oq);
        }
        s_o[warp][lane] = oq;
        // (every thread has read s_rk / s_ru before it passes this barrier, and
        // the next token writes them only after it)
        __syncthreads();
        if (warp == 0) {
            const float oj = s_o[0][lane] + s_o[1][lane] + s_o[2][lane] + s_o[3][lane];
            o[(t * H + h) * DV + j] = from_f32<Tin>(oj);
        }
        // (warp 0's reads of s_o come before its next barrier, which the other
        // warps must also reach before they write s_o again; this warp's slice
        // of s_v is rewritten only after its own reads above)
        __syncwarp();
    }
    if (final_state) {
#pragma unroll
        for (int i = 0; i < ROWS; ++i) final_state[sbase + (int64_t)i * DV] = s[i];
    }
}

template <typename Tin, int DK>
cudaError_t launch_qed_t(const QedArgs &a, cudaStream_t stream)
{
    const dim3 grid((unsigned)(a.num_seqs * a.H), (unsigned)(a.dv / kQedCols), 1);
    qed_fwd_kernel<Tin, DK><<<grid, kQedThreads, 0, stream>>>(
        static_cast<const Tin *>(a.q), static_cast<const Tin *>(a.k), static_cast<const Tin *>(a.v), a.log_alpha,
        static_cast<const Tin *>(a.b), static_cast<const Tin *>(a.w), a.strength, a.direction, (int)a.flags,
        a.init_state, a.cu_seqlens, a.T, a.H, a.dv, a.B * a.T, static_cast<Tin *>(a.o), a.final_state);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_qed(const QedArgs &a, cudaStream_t stream)
{
    if (a.num_seqs == 0 || a.H == 0) return cudaSuccess;
    if (a.bf16)
        return a.dk == 128 ? launch_qed_t<__nv_bfloat16, 128>(a, stream) : launch_qed_t<__nv_bfloat16, 64>(a, stream);
    return a.dk == 128 ? launch_qed_t<float, 128>(a, stream) : launch_qed_t<float, 64>(a, stream);
}

}  // namespace gdr2
