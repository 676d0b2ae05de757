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
// in registers; each token costs three block reductions (the direction's
// norms, the two reads of the decayed state, the readout), and its inputs are
// loaded one token ahead.
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
    constexpr int ROWS = DK / 4;  // key rows per warp
    __shared__ float s_q[DK], s_k[DK], s_a[DK], s_e[DK], s_u[DK], s_f[DK];
    __shared__ float s_red[4][3];
    __shared__ float s_rk[4][kQedCols], s_ru[4][kQedCols];

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
    const float dirc = (direction && tid < DK) ? direction[h * DK + tid] : 0.f;

    float s[ROWS];
    const int64_t sbase = (unit * DK + (int64_t)ROWS * warp) * DV + j;
#pragma unroll
    for (int i = 0; i < ROWS; ++i) s[i] = init_state ? init_state[sbase + (int64_t)i * DV] : 0.f;

    // block sum of three values (one per thread; the result in every thread)
    auto sum3 = [&](float &x, float &y, float &z) {
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) {
            x += __shfl_xor_sync(0xffffffffu, x, m);
            y += __shfl_xor_sync(0xffffffffu, y, m);
            z += __shfl_xor_sync(0xffffffffu, z, m);
        }
        if (lane == 0) {
            s_red[warp][0] = x;
            s_red[warp][1] = y;
            s_red[warp][2] = z;
        }
        __syncthreads();
        x = s_red[0][0] + s_red[1][0] + s_red[2][0] + s_red[3][0];
        y = s_red[0][1] + s_red[1][1] + s_red[2][1] + s_red[3][1];
        z = s_red[0][2] + s_red[1][2] + s_red[2][2] + s_red[3][2];
        __syncthreads();  // (s_red is reused by the next call)
    };

    // inputs of token t: channel tid (tid < DK) of q, k, log_alpha, b; value
    // column j of v and w (every warp loads the same 32 columns)
    float nq = 0.f, nk = 0.f, nla = 0.f, nb = 0.f, nv = 0.f, nw = 0.f;
    auto fetch = [&](int64_t t) {
        if (t >= t_end) return;
        const int64_t rk = (t * H + h) * DK, rv = (t * H + h) * DV;
        if (tid < DK) {
            nq = to_f32(q[rk + tid]);
            nk = to_f32(k[rk + tid]);
            nla = log_alpha[rk + tid];
            nb = to_f32(b[rk + tid]);
        }
        nv = to_f32(v[rv + j]);
        nw = to_f32(w[rv + j]);
    };
    fetch(t_begin);
    for (int64_t t = t_begin; t < t_end; ++t) {
        const float qc = nq, kc = nk, lac = nla, bc = nb, z = nv * nw;
        fetch(t + 1);
        // the erase direction u from the query (or the fixed direction)
        const float src = direction ? dirc : qc;
        float kk = tid < DK ? kc * kc : 0.f, ks = tid < DK ? kc * src : 0.f, ss = tid < DK ? src * src : 0.f;
        sum3(kk, ks, ss);
        const float coef = (project && kk > 0.f) ? ks / kk : 0.f;
        const float pc = src - coef * kc;
        float pp = tid < DK ? pc * pc : 0.f, d1 = 0.f, d2 = 0.f;
        sum3(pp, d1, d2);
        const float inv = (pp > 1e-12f * ss && pp > 0.f) ? rsqrtf(pp) : 0.f;
        if (tid < DK) {
            const float uc = pc * inv;
            s_q[tid] = qc;
            s_k[tid] = kc;
            s_a[tid] = expf(lac);
            s_e[tid] = bc * kc;
            s_u[tid] = uc;
            s_f[tid] = gate ? bc * uc : uc;
        }
        __syncthreads();
        // decay, then both reads of the decayed state (this warp's rows)
        float rk = 0.f, ru = 0.f;
#pragma unroll
        for (int i = 0; i < ROWS; ++i) {
            const int c = ROWS * warp + i;
            s[i] *= s_a[c];
            rk = fmaf(s_e[c], s[i], rk);
            ru = fmaf(s_f[c], s[i], ru);
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
            s[i] = fmaf(s_k[c], resid, fmaf(-s_u[c], lru, s[i]));
            oq = fmaf(s_q[c], s[i], oq);
        }
        __syncthreads();  // (every read of s_rk / s_ru above is done)
        s_rk[warp][lane] = oq;
        __syncthreads();
        if (warp == 0) {
            const float oj = s_rk[0][lane] + s_rk[1][lane] + s_rk[2][lane] + s_rk[3][lane];
            o[(t * H + h) * DV + j] = from_f32<Tin>(oj);
        }
        // (the next token's first barrier orders these reads before s_rk is rewritten)
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
