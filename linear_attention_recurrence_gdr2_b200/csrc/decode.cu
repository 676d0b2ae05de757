// Single-token decode step of Gated Delta Rule-2 (bandwidth-bound).
//
// Per (sequence n, head h), with the fp32 state S (d_k x d_v, d_v contiguous)
// updated in place:
//   S' = Diag(alpha) S                  (decay before the edit)
//   r  = S'^T e,  e = b . k             (gated read along the erase direction)
//   p  = S'^T q
//   S  = S' + k (z - r)^T,  z = w . v   (delta edit with the gated write)
//   o  = S^T q = p + (k . q) (z - r)
// ("Gated Delta Rule-2" section of the zhichai.net summary of Gated
// DeltaNet-2; decay-before-edit from the "two gates instead of one" section
// of the ainews.random.gg article.)
//
// The state is the only large operand (64 KiB per head at d = 128), read once
// and written once: each CTA owns one head, each warp a set of key rows, each
// lane VEC consecutive value columns, so every warp access is one contiguous
// d_v row (512 B at d = 128). The two reductions over key channels are
// per-thread partial sums followed by one shared-memory pass across warps.
#include "common.cuh"
#include "kernels.h"

namespace gdr2 {

// kPre: the fused prologue is compiled in (the *_preact calls only).
template <typename Tin, int DK, int DV, int NWARPS, bool kPre>
__global__ void __launch_bounds__(NWARPS * 32)
decode_step_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                   const Tin *__restrict__ v, const float *__restrict__ log_alpha,
                   const Tin *__restrict__ b, const Tin *__restrict__ w,
                   float *__restrict__ state, Tin *__restrict__ o, uint32_t pre)
{
    constexpr int VEC = DV / 32;          // value columns per lane
    constexpr int ROWS = DK / NWARPS;     // key rows per warp
    static_assert(VEC == 2 || VEC == 4, "d_v must be 64 or 128");
    static_assert(DK % NWARPS == 0, "rows must split evenly across warps");

    __shared__ float s_alpha[DK], s_e[DK], s_q[DK], s_k[DK];
    __shared__ float s_z[DV];
    __shared__ float s_red[2][NWARPS][DV];

    const int64_t head = blockIdx.x;   // n * H + h
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // (with the fused prologue: gates through a sigmoid, log_alpha through
    // -softplus; q and k are normalised below where they are read)
    for (int c = threadIdx.x; c < DK; c += NWARPS * 32) {
        const int64_t i = head * DK + c;
        float kc = to_f32(k[i]);
        float la = log_alpha[i], bc = to_f32(b[i]);
        if (kPre && (pre & GDR2_PROLOGUE_DECAY_SOFTPLUS)) la = pre_neg_softplus(la);
        if (kPre && (pre & GDR2_PROLOGUE_GATE_SIGMOID)) bc = pre_sigmoid(bc);
        s_alpha[c] = expf(la);
        s_e[c] = bc * kc;
        s_q[c] = to_f32(q[i]);
        s_k[c] = kc;
    }
    for (int j = threadIdx.x; j < DV; j += NWARPS * 32) {
        const int64_t i = head * DV + j;
        float wj = to_f32(w[i]);
        if (kPre && (pre & GDR2_PROLOGUE_GATE_SIGMOID)) wj = pre_sigmoid(wj);
        s_z[j] = wj * to_f32(v[i]);
    }

    // Issue every state load of this thread before the first use.
    float *S = state + head * (int64_t)DK * DV;
    float x[ROWS][VEC];
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
        const int c = warp + i * NWARPS;
        load_vec<float, VEC>(S + (int64_t)c * DV + lane * VEC, x[i]);
    }
    __syncthreads();

    // prologue: 1 / ||q||, 1 / ||k|| (every warp reduces the shared copies itself)
    float iq = 1.f, ik = 1.f;
    if (kPre && (pre & GDR2_PROLOGUE_QK_L2NORM)) {
        float sq = 0.f, sk = 0.f;
        for (int c = lane; c < DK; c += 32) {
            sq = fmaf(s_q[c], s_q[c], sq);
            sk = fmaf(s_k[c], s_k[c], sk);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            sq += __shfl_xor_sync(0xffffffffu, sq, off);
            sk += __shfl_xor_sync(0xffffffffu, sk, off);
        }
        iq = rsqrtf(sq + 1e-6f);
        ik = rsqrtf(sk + 1e-6f);
    }

    float r[VEC], p[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) r[j] = p[j] = 0.f;
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
        const int c = warp + i * NWARPS;
        const float a = s_alpha[c], e = kPre ? s_e[c] * ik : s_e[c], qc = kPre ? s_q[c] * iq : s_q[c];
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            x[i][j] *= a;
            r[j] = fmaf(e, x[i][j], r[j]);
            p[j] = fmaf(qc, x[i][j], p[j]);
        }
    }
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
        s_red[0][warp][lane * VEC + j] = r[j];
        s_red[1][warp][lane * VEC + j] = p[j];
    }
    // k . q, reduced within every warp (no extra block barrier needed).
    float kq = 0.f;
    for (int c = lane; c < DK; c += 32) kq = fmaf(s_k[c], s_q[c], kq);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    if constexpr (kPre) kq *= ik * iq;
    __syncthreads();

    float u[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) {
        float rs = 0.f, ps = 0.f;
#pragma unroll
        for (int ww = 0; ww < NWARPS; ++ww) {
            rs += s_red[0][ww][lane * VEC + j];
            ps += s_red[1][ww][lane * VEC + j];
        }
        u[j] = s_z[lane * VEC + j] - rs;
        p[j] = ps;
    }
#pragma unroll
    for (int i = 0; i < ROWS; ++i) {
        const int c = warp + i * NWARPS;
        const float kc = kPre ? s_k[c] * ik : s_k[c];
        float *dst = S + (int64_t)c * DV + lane * VEC;
        float y[VEC];
#pragma unroll
        for (int j = 0; j < VEC; ++j) y[j] = fmaf(kc, u[j], x[i][j]);
        if constexpr (VEC == 4) {
            *reinterpret_cast<float4 *>(dst) = make_float4(y[0], y[1], y[2], y[3]);
        } else {
            *reinterpret_cast<float2 *>(dst) = make_float2(y[0], y[1]);
        }
    }
    if (warp == 0) {
#pragma unroll
        for (int j = 0; j < VEC; ++j)
            o[head * DV + lane * VEC + j] = from_f32<Tin>(fmaf(kq, u[j], p[j]));
    }
}

template <typename Tin, int D>
static cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t stream)
{
    constexpr int NWARPS = 8;
    const int64_t heads = a.N * a.H;
    if (heads == 0) return cudaSuccess;
    auto kern = a.pre ? decode_step_kernel<Tin, D, D, NWARPS, true> : decode_step_kernel<Tin, D, D, NWARPS, false>;
    kern<<<(unsigned)heads, NWARPS * 32, 0, stream>>>(
        (const Tin *)a.q, (const Tin *)a.k, (const Tin *)a.v, a.log_alpha,
        (const Tin *)a.b, (const Tin *)a.w, a.state, (Tin *)a.o, a.pre);
    return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t stream)
{
    if (a.bf16) {
        return a.dk == 128 ? launch_decode_t<__nv_bfloat16, 128>(a, stream)
                           : launch_decode_t<__nv_bfloat16, 64>(a, stream);
    }
    return a.dk == 128 ? launch_decode_t<float, 128>(a, stream)
                       : launch_decode_t<float, 64>(a, stream);
}

}  // namespace gdr2
