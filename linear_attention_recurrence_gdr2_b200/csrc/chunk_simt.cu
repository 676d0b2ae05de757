// Chunkwise forward of Gated Delta Rule-2 on CUDA cores, every product in
// fp32. This is the library's fp32 path (tensor-core formats cannot hold the
// 1e-4 relative error an fp32 caller expects); bf16 inputs run on the
// tensor-core kernel instead.
//
// Chunk form (C = 64, "Chunkwise training and gate-aware backward" section of
// the ainews.random.gg article on Gated DeltaNet-2; derivation below).
// Inside a chunk with entry state S0 let g_r = sum_{i<=r} log alpha_i
// (cumulative per key channel, relative to the chunk start) and
// Shat_r = Diag(e^{-g_r}) S_r. The token rule becomes
//     Shat_r = (I - kbar_r ebar_r^T) Shat_{r-1} + kbar_r z_r^T,
//     kbar_r = k_r . e^{-g_r},  ebar_r = b_r . k_r . e^{g_r},  z_r = w_r . v_r,
// i.e. the asymmetric rank-one erase factors of the article. Unrolling gives
// Shat_r = S0 + sum_{s<=r} kbar_s u_s^T with u_r = z_r - S0^T ebar_r -
// sum_{s<r} (ebar_r . kbar_s) u_s, so with A = strict_tril(Ebar Kbar^T):
//     U = (I + A)^{-1} (Z - Ebar S0)
//     O = Qbar S0 + tril(Qbar Kbar^T) U,           qbar_r = q_r . e^{g_r}
//     S_C = Diag(e^{g_C}) S0 + (K . e^{g_C - g})^T U.
// Range: the products ebar_r . kbar_s and qbar_r . kbar_s only need
// e^{g_r - g_s} <= 1, so they are formed about the chunk's middle row m
// (factors e^{+-(g - g_m)}), which halves the exponent range; the state-side
// products use e^{g_r} <= 1 directly. A chunk in which |g_r - g_m| passes
// kFactorRange on some channel (decay too strong for those factors) runs
// the token rule itself instead, one token at a time, exact for any alpha.
//
// One CTA owns one (sequence, head, 32-wide value tile) and walks its chunks
// in order, keeping the fp32 state tile in shared memory.
#include "common.cuh"
#include "kernels.h"

namespace gdr2 {
namespace {

constexpr int kThreads = 256;
constexpr int kDVT = 32;          // value columns per CTA
constexpr int kLD = kChunk + 4;   // padded row length of [channel][row] arrays
constexpr int kMid = 31;          // reference row for the pairwise products
// Largest |g_r - g_m| (natural log) the factors e^{+-(g_r - g_m)} may take:
// e^64 and e^-64 are normal fp32 numbers with room for the products they enter.
constexpr float kFactorRange = 64.f;

template <int DK>
struct SimtSmem {
    float qm[DK][kLD];     // q . e^{g - g_m}       (transposed: [channel][row])
    float km[DK][kLD];     // k . e^{g_m - g}
    float em[DK][kLD];     // b . k . e^{g - g_m}
    float a[kChunk][kLD];  // strict_tril(Ebar Kbar^T)
    float p[kChunk][kLD];  // tril(Qbar Kbar^T), diagonal included
    float s0[DK][kDVT];    // state tile (fp32 master)
    float sm[DK][kDVT];    // Diag(e^{g_m}) S0
    float z[kChunk][kDVT]; // z -> r = z - Ebar S0 -> u (in place)
    float la[DK][kLD];     // log alpha of the chunk (used by a token-serial chunk)
    float gC[DK];
    float gm[DK];
    int serial;            // this chunk runs token by token
    float qinv[kChunk];    // prologue: 1 / ||q_r||, 1 / ||k_r|| (1 without it)
    float kinv[kChunk];
};

// kPre: the fused prologue is compiled in (the *_preact calls only).
template <typename Tin, int DK, bool kPre>
__global__ void __launch_bounds__(kThreads, 1)
chunk_simt_kernel(ChunkArgs args)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SimtSmem<DK> &sm = *reinterpret_cast<SimtSmem<DK> *>(smem_raw);

    const int tid = threadIdx.x;
    const int j0 = blockIdx.x * kDVT;      // first value column of this tile
    const int64_t h = blockIdx.y;
    const int64_t n = args.order ? (int64_t)args.order[blockIdx.z] : (int64_t)blockIdx.z;
    const int64_t H = args.H;
    const int DV = (int)args.dv;

    const Tin *q = (const Tin *)args.q, *k = (const Tin *)args.k, *b = (const Tin *)args.b;
    const Tin *v = (const Tin *)args.v, *w = (const Tin *)args.w;
    const float *la = args.log_alpha;
    Tin *o = (Tin *)args.o;

    int64_t t_begin, t_end;
    if (args.cu_seqlens) {
        packed_bounds(args.cu_seqlens, n, args.B * args.T, t_begin, t_end);
    } else {
        t_begin = n * args.T;
        t_end = t_begin + args.T;
    }

    const int64_t state_off = (n * H + h) * (int64_t)DK * DV + j0;
    for (int i = tid; i < DK * kDVT; i += kThreads) {
        const int c = i / kDVT, j = i % kDVT;
        sm.s0[c][j] = args.init_state ? args.init_state[state_off + (int64_t)c * DV + j] : 0.f;
    }

    if (tid == 0) sm.serial = 0;
    const uint32_t pre = kPre ? args.pre : 0u;
    for (int64_t t0 = t_begin; t0 < t_end; t0 += kChunk) {
        const int L = (int)(t_end - t0 < kChunk ? t_end - t0 : kChunk);
        __syncthreads();  // previous chunk finished with every buffer

        // ---- prologue: L2 norms of the q and k rows (one warp per row) ----
        if constexpr (kPre) {
            const int wp = tid >> 5, ln = tid & 31;
            for (int r = wp; r < kChunk; r += kThreads / 32) {
                float sq = 0.f, sk = 0.f;
                if ((pre & GDR2_PROLOGUE_QK_L2NORM) && r < L) {
                    for (int c = ln; c < DK; c += 32) {
                        const int64_t i = ((t0 + r) * H + h) * DK + c;
                        const float qv = to_f32(q[i]), kv = to_f32(k[i]);
                        sq = fmaf(qv, qv, sq);
                        sk = fmaf(kv, kv, sk);
                    }
                    for (int m = 16; m >= 1; m >>= 1) {
                        sq += __shfl_xor_sync(0xffffffffu, sq, m);
                        sk += __shfl_xor_sync(0xffffffffu, sk, m);
                    }
                }
                if (ln == 0) {
                    const bool nrm = (pre & GDR2_PROLOGUE_QK_L2NORM) != 0;
                    sm.qinv[r] = nrm ? rsqrtf(sq + 1e-6f) : 1.f;
                    sm.kinv[r] = nrm ? rsqrtf(sk + 1e-6f) : 1.f;
                }
            }
        }
        if constexpr (kPre) __syncthreads();

        // ---- cumulative log-decay and decay-absorbed factors -------------
        float g[kChunk];
        if (tid < DK) {
            const int c = tid;
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < kChunk; ++r) {
                float x = r < L ? la[((t0 + r) * H + h) * DK + c] : 0.f;
                if ((pre & GDR2_PROLOGUE_DECAY_SOFTPLUS) && r < L) x = pre_neg_softplus(x);
                sm.la[c][r] = x;
                acc += x;
                g[r] = acc;
            }
            float m = 0.f;
#pragma unroll
            for (int r = 0; r < kChunk; ++r) m = fmaxf(m, fabsf(g[r] - g[kMid]));
            if (m > kFactorRange) sm.serial = 1;
        }
        __syncthreads();
        const bool serial = sm.serial != 0;
        if (tid < DK) {
            const int c = tid;
            const float gm = g[kMid];
            sm.gC[c] = g[kChunk - 1];
            sm.gm[c] = gm;
#pragma unroll
            for (int r = 0; r < kChunk; ++r) {
                float qv = 0.f, kv = 0.f, bv = 0.f;
                if (r < L) {
                    const int64_t i = ((t0 + r) * H + h) * DK + c;
                    qv = to_f32(q[i]);
                    kv = to_f32(k[i]);
                    if constexpr (kPre) {
                        qv *= sm.qinv[r];
                        kv *= sm.kinv[r];
                    }
                    bv = to_f32(b[i]);
                    if (pre & GDR2_PROLOGUE_GATE_SIGMOID) bv = pre_sigmoid(bv);
                }
                // (a token-serial chunk keeps the raw q, k and b . k)
                const float up = serial ? 1.f : expf(g[r] - gm), dn = serial ? 1.f : expf(gm - g[r]);
                sm.qm[c][r] = qv * up;
                sm.km[c][r] = kv * dn;
                sm.em[c][r] = bv * kv * up;
            }
        }
        for (int i = tid; i < kChunk * kDVT; i += kThreads) {
            const int r = i / kDVT, j = i % kDVT;
            float zv = 0.f;
            if (r < L) {
                const int64_t e = ((t0 + r) * H + h) * DV + j0 + j;
                float wv = to_f32(w[e]);
                if (pre & GDR2_PROLOGUE_GATE_SIGMOID) wv = pre_sigmoid(wv);
                zv = wv * to_f32(v[e]);
            }
            sm.z[r][j] = zv;
        }
        __syncthreads();

        if (serial) {
            // ---- the token rule, one token at a time (decay past the factor
            // range): s' = alpha . s, r = e^T s', s = s' + k (z - r),
            // o = q^T s = q^T s' + (k^T q)(z - r). Thread (jc, rg) holds key
            // channels rg * CPT .. + CPT - 1 of value column jc.
            constexpr int CPT = DK / (kThreads / kDVT);
            const int jc = tid % kDVT, rg = tid / kDVT, cb = rg * CPT;
            float *red = &sm.a[0][0];  // [2][2][8][32] partial sums, then [2][8] k^T q
            float *kqp = red + 2 * 2 * 8 * kDVT;
            float st[CPT];
#pragma unroll
            for (int i = 0; i < CPT; ++i) st[i] = sm.s0[cb + i][jc];
            int buf = 0;
            for (int r = 0; r < L; ++r) {
                float pe = 0.f, pq = 0.f, pkq = 0.f;
#pragma unroll
                for (int i = 0; i < CPT; ++i) {
                    const int c = cb + i;
                    st[i] *= expf(sm.la[c][r]);
                    pe = fmaf(sm.em[c][r], st[i], pe);
                    pq = fmaf(sm.qm[c][r], st[i], pq);
                    pkq = fmaf(sm.km[c][r], sm.qm[c][r], pkq);
                }
                float *rb = red + buf * 2 * 8 * kDVT;
                rb[rg * kDVT + jc] = pe;
                rb[8 * kDVT + rg * kDVT + jc] = pq;
                if (jc == 0) kqp[buf * 8 + rg] = pkq;
                __syncthreads();
                float rr = 0.f, pp = 0.f, kq = 0.f;
#pragma unroll
                for (int gi = 0; gi < 8; ++gi) {
                    rr += rb[gi * kDVT + jc];
                    pp += rb[8 * kDVT + gi * kDVT + jc];
                    kq += kqp[buf * 8 + gi];
                }
                const float delta = sm.z[r][jc] - rr;
#pragma unroll
                for (int i = 0; i < CPT; ++i) st[i] = fmaf(sm.km[cb + i][r], delta, st[i]);
                if (rg == 0) o[((t0 + r) * H + h) * DV + j0 + jc] = from_f32<Tin>(fmaf(kq, delta, pp));
                buf ^= 1;
            }
#pragma unroll
            for (int i = 0; i < CPT; ++i) sm.s0[cb + i][jc] = st[i];
            __syncthreads();
            if (tid == 0) sm.serial = 0;  // (read again only after the next chunk's first barrier)
            continue;
        }

        // ---- A = strict_tril(Ebar Kbar^T), P = tril(Qbar Kbar^T) ----------
        {
            const int rb = tid / 16, sb = tid % 16;
            if (sb <= rb) {
                float pa[4][4] = {}, aa[4][4] = {};
                for (int c = 0; c < DK; ++c) {
                    const float4 qv = *reinterpret_cast<const float4 *>(&sm.qm[c][4 * rb]);
                    const float4 ev = *reinterpret_cast<const float4 *>(&sm.em[c][4 * rb]);
                    const float4 kv = *reinterpret_cast<const float4 *>(&sm.km[c][4 * sb]);
                    const float qa[4] = {qv.x, qv.y, qv.z, qv.w};
                    const float ea[4] = {ev.x, ev.y, ev.z, ev.w};
                    const float ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {
                            pa[i][jj] = fmaf(qa[i], ka[jj], pa[i][jj]);
                            aa[i][jj] = fmaf(ea[i], ka[jj], aa[i][jj]);
                        }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const int r = 4 * rb + i, s = 4 * sb + jj;
                        sm.p[r][s] = s <= r ? pa[i][jj] : 0.f;
                        sm.a[r][s] = s < r ? aa[i][jj] : 0.f;
                    }
            }
        }
        for (int i = tid; i < DK * kDVT; i += kThreads) {
            const int c = i / kDVT, j = i % kDVT;
            sm.sm[c][j] = expf(sm.gm[c]) * sm.s0[c][j];
        }
        __syncthreads();

        // ---- R = Z - Ebar S0 (= Z - Em Sm) ---------------------------------
        const int jc = tid % kDVT, rg = tid / kDVT;  // 8 row groups of 8 rows
        {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = sm.z[8 * rg + i][jc];
            for (int c = 0; c < DK; ++c) {
                const float s = sm.sm[c][jc];
                const float4 e0 = *reinterpret_cast<const float4 *>(&sm.em[c][8 * rg]);
                const float4 e1 = *reinterpret_cast<const float4 *>(&sm.em[c][8 * rg + 4]);
                acc[0] = fmaf(-e0.x, s, acc[0]); acc[1] = fmaf(-e0.y, s, acc[1]);
                acc[2] = fmaf(-e0.z, s, acc[2]); acc[3] = fmaf(-e0.w, s, acc[3]);
                acc[4] = fmaf(-e1.x, s, acc[4]); acc[5] = fmaf(-e1.y, s, acc[5]);
                acc[6] = fmaf(-e1.z, s, acc[6]); acc[7] = fmaf(-e1.w, s, acc[7]);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) sm.z[8 * rg + i][jc] = acc[i];
        }
        __syncthreads();

        // ---- U = (I + A)^{-1} R by forward substitution, column-parallel ---
        {
            const int warp = tid >> 5, lane = tid & 31;
            const int col = warp * 4 + (lane >> 3), sub = lane & 7;
            for (int r = 1; r < kChunk; ++r) {
                float part = 0.f;
                for (int s = sub; s < r; s += 8) part = fmaf(sm.a[r][s], sm.z[s][col], part);
                part += __shfl_xor_sync(0xffffffffu, part, 1);
                part += __shfl_xor_sync(0xffffffffu, part, 2);
                part += __shfl_xor_sync(0xffffffffu, part, 4);
                if (sub == 0) sm.z[r][col] -= part;
                __syncwarp();
            }
        }
        __syncthreads();

        // ---- O = Qbar S0 + P U ;  S0 <- Diag(e^{g_C}) S0 + (K e^{g_C-g})^T U
        {
            float acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.f;
            for (int c = 0; c < DK; ++c) {
                const float s = sm.sm[c][jc];
                const float4 q0 = *reinterpret_cast<const float4 *>(&sm.qm[c][8 * rg]);
                const float4 q1 = *reinterpret_cast<const float4 *>(&sm.qm[c][8 * rg + 4]);
                acc[0] = fmaf(q0.x, s, acc[0]); acc[1] = fmaf(q0.y, s, acc[1]);
                acc[2] = fmaf(q0.z, s, acc[2]); acc[3] = fmaf(q0.w, s, acc[3]);
                acc[4] = fmaf(q1.x, s, acc[4]); acc[5] = fmaf(q1.y, s, acc[5]);
                acc[6] = fmaf(q1.z, s, acc[6]); acc[7] = fmaf(q1.w, s, acc[7]);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = 8 * rg + i;
                float x = acc[i];
                for (int s = 0; s <= r; ++s) x = fmaf(sm.p[r][s], sm.z[s][jc], x);
                if (r < L) o[((t0 + r) * H + h) * DV + j0 + jc] = from_f32<Tin>(x);
            }
            constexpr int CPT = DK / (kThreads / kDVT);  // key rows per thread
#pragma unroll 4
            for (int ci = 0; ci < CPT; ++ci) {
                const int c = rg * CPT + ci;
                float x = 0.f;
                for (int s = 0; s < kChunk; ++s) x = fmaf(sm.km[c][s], sm.z[s][jc], x);
                const float gc = sm.gC[c];
                sm.s0[c][jc] = fmaf(expf(gc - sm.gm[c]), x, expf(gc) * sm.s0[c][jc]);
            }
        }
    }
    __syncthreads();
    if (args.final_state) {
        for (int i = tid; i < DK * kDVT; i += kThreads) {
            const int c = i / kDVT, j = i % kDVT;
            args.final_state[state_off + (int64_t)c * DV + j] = sm.s0[c][j];
        }
    }
}

template <typename Tin, int DK>
cudaError_t launch_t(const ChunkArgs &a, cudaStream_t stream)
{
    const size_t smem = sizeof(SimtSmem<DK>);
    auto kern = a.pre ? chunk_simt_kernel<Tin, DK, true> : chunk_simt_kernel<Tin, DK, false>;
    cudaError_t e = ensure_dynamic_smem((const void *)kern, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)(a.dv / kDVT), (unsigned)a.H, (unsigned)a.num_seqs);
    kern<<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_simt(const ChunkArgs &a, cudaStream_t stream)
{
    if (a.num_seqs == 0 || a.H == 0) return cudaSuccess;
    if (a.bf16)
        return a.dk == 128 ? launch_t<__nv_bfloat16, 128>(a, stream) : launch_t<__nv_bfloat16, 64>(a, stream);
    return a.dk == 128 ? launch_t<float, 128>(a, stream) : launch_t<float, 64>(a, stream);
}

}  // namespace gdr2
