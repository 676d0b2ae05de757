// Gate-aware backward of Gated Delta Rule-2: the vector-Jacobian product of
//   S'_t = Diag(alpha_t) S_{t-1},  e_t = b_t . k_t,  z_t = w_t . v_t,
//   u_t  = z_t - S'_t^T e_t,       S_t = S'_t + k_t u_t^T,  o_t = S_t^T q_t
// for cotangents dO (per token) and dS_T (per sequence). The "Chunkwise
// training and gate-aware backward" section of the ainews.random.gg article on
// Gated DeltaNet-2 notes that with two different diagonal gates the gate
// factors must sit inside the gradient's dot products; here every gradient is
// the exact chain rule of the lines above, taken in fp32.
//
// Decomposition (three sweeps, two launches):
//   A (forward, per value column j): the rule above only mixes key rows, so
//     column j of S evolves on its own given alpha, e, k and z_{t,j}. Stores
//     u_t and the state at every chunk start (checkpoints, fp32).
//   B (reverse, per value column j): with H_t = G + q_t do_t^T,
//     du_t = H_t^T k_t and G <- Diag(alpha_t)(H_t - e_t du_t^T), starting from
//     dS_T, column j of G also evolves on its own. Stores du_t and G at every
//     chunk end; writes dv = du . w, dw = du . v and dS_0 (the last G).
//   C (per chunk and key row i): given u and du, row i of S (forward from the
//     chunk-start checkpoint) and row i of H (reverse from the chunk-end one)
//     evolve on their own, so every remaining gradient is a row-local dot
//     product over value columns:
//       dq_t = S_t do_t,  de_t = -S'_t du_t,  dkW_t = H_t u_t,
//       dk_t = dkW_t + b_t . de_t,  db_t = k_t . de_t,
//       dlog_alpha_t = sum_{s >= t in the chunk} (q.dq - k.dkW + e.de)_s
//                      + rowsum(G_end . S_end).
//     The last line replaces the per-token rowsum(dS'_t . S'_t): both
//     recurrences telescope, so the decay gradient of token t is that of
//     token t+1 plus the three per-token terms, and at a chunk end it equals
//     the row-wise product of the incoming cotangent with the state there.
//     Restarting it at every chunk end keeps its cancellation within 64 tokens.
// A and B run in one launch (blockIdx.z picks the sweep); C follows on the
// same stream. All arithmetic is fp32 on the CUDA cores.
#include "common.cuh"
#include "kernels.h"

namespace gdr2 {
namespace {

constexpr int kSub = 8;            // tokens staged per round of the column sweeps
constexpr int kScanThreads = 256;  // 8 warps; a half-warp per 4 value columns
constexpr int kTile = 64;          // value columns per column-sweep CTA
constexpr int kRowThreads = 256;   // 4 lanes per key row in the per-chunk kernel

struct BwdParams {
    const void *q, *k, *v, *b, *w, *d_o;
    const float *la, *init_state, *d_final;
    const int32_t *cu;
    void *dq, *dk, *dv, *db, *dw;
    float *dla, *d_init;
    float *ck, *gk, *U, *dU;   // workspace: checkpoints and per-token column vectors
    int64_t T, H, N, tokens;
};

// Token range of sequence n (packed offsets are clamped to the token count).
__device__ __forceinline__ void seq_bounds(const BwdParams &p, int64_t n, int64_t &start, int64_t &len)
{
    if (p.cu) {
        int64_t s = p.cu[n], e = p.cu[n + 1];
        s = s < 0 ? 0 : (s > p.tokens ? p.tokens : s);
        e = e < s ? s : (e > p.tokens ? p.tokens : e);
        start = s;
        len = e - s;
    } else {
        start = n * p.T;
        len = p.T;
    }
}

// First checkpoint slot of sequence n. start/64 + n grows by at least
// ceil(len/64) from one sequence to the next, so the slots of different
// sequences never overlap and all lie below tokens/64 + N.
__device__ __forceinline__ int64_t slot_base(int64_t start, int64_t n) { return start / kChunk + n; }

template <typename T>
__device__ __forceinline__ void store2(T *p, float a, float b);
template <>
__device__ __forceinline__ void store2<float>(float *p, float a, float b) {
    *reinterpret_cast<float2 *>(p) = make_float2(a, b);
}
template <>
__device__ __forceinline__ void store2<__nv_bfloat16>(__nv_bfloat16 *p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(a, b);
}

// ROWS floats from shared memory in groups of 4: group g at src + g * GS (each
// group one 16-byte load).
template <int ROWS, int GS>
__device__ __forceinline__ void load_row_groups(const float *src, float (&out)[ROWS])
{
    static_assert(ROWS % 4 == 0, "rows come in float4 groups");
#pragma unroll
    for (int g = 0; g < ROWS / 4; ++g) {
        const float4 v = *reinterpret_cast<const float4 *>(src + GS * g);
        out[4 * g] = v.x; out[4 * g + 1] = v.y; out[4 * g + 2] = v.z; out[4 * g + 3] = v.w;
    }
}

// 16-byte asynchronous copy global -> shared (cp.async, bypassing L1).
__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;\n" ::: "memory");
}

// Sweeps A (blockIdx.z == 0) and B (blockIdx.z == 1). CTA = (sequence, head,
// tile of 64 value columns); lane l of warp w owns the 4 columns 64*tile + 8w +
// 4*(l/16) + {0..3} and D/16 key rows in groups of 4 (group g: rows
// 64 g + 4 (l % 16) + {0..3}, read from shared memory as float4 without bank
// conflicts), so the reductions over key rows are
// four xor-shuffles inside a half-warp, four independent columns at a time. One
// CTA per 64 columns keeps both sweeps of a layer-sized batch resident at once.
// Row inputs (alpha, e, k, q) for 8 tokens are staged in shared memory, the
// next 8 prefetched into registers while the current ones are consumed.
template <typename Tin, int D>
__global__ void __launch_bounds__(kScanThreads, 2) bwd_scan_kernel(BwdParams p)
{
    constexpr int ROWS = D / 16;
    constexpr int NC = 4;                                 // value columns per lane
    constexpr int PF = kSub * D / kScanThreads;           // staged row elements per thread
    constexpr int PC = kSub * kTile / kScanThreads;       // staged column elements per thread
    static_assert(PF * kScanThreads == kSub * D && PC * kScanThreads == kSub * kTile, "staging split");
    static_assert(kTile == 8 * 2 * NC, "8 warps x 2 half-warps x NC columns");
    __shared__ __align__(16) float s_al[kSub * D], s_e[kSub * D], s_k[kSub * D], s_q[kSub * D];
    __shared__ __align__(16) float s_c[3][kSub * kTile];   // A: z | B: do, v, w

    const int64_t n = blockIdx.x / p.H;
    const int h = (int)(blockIdx.x % p.H);
    const int tile = blockIdx.y;
    const bool rev = blockIdx.z != 0;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // this lane's key rows: ROWS/4 groups of 4, group g at g * GS + 4 (lane % 16),
    // so that the 16 lanes' 16-byte reads of one group are one contiguous 256 B
    // (no shared-memory bank conflicts)
    constexpr int GS = D / (ROWS / 4);
    const int row0 = 4 * (lane & 15);
    auto row_of = [&](int m) { return GS * (m >> 2) + row0 + (m & 3); };
    const int jl = warp * 2 * NC + (lane >> 4) * NC;  // first of this lane's columns, in the tile
    const int j = tile * kTile + jl;
    const Tin *Q = static_cast<const Tin *>(p.q), *K = static_cast<const Tin *>(p.k);
    const Tin *Bg = static_cast<const Tin *>(p.b), *V = static_cast<const Tin *>(p.v);
    const Tin *Wg = static_cast<const Tin *>(p.w), *DO = static_cast<const Tin *>(p.d_o);

    int64_t start, len;
    seq_bounds(p, n, start, len);
    const int64_t base = slot_base(start, n);
    const int64_t nsub = (len + kSub - 1) / kSub;
    const int64_t head_state = (n * p.H + h) * (int64_t)D * D;

    // X: state columns (A) or cotangent columns (B), rows row_of(0 .. ROWS - 1)
    float X[NC][ROWS];
    const float *x_init = rev ? p.d_final : p.init_state;
#pragma unroll
    for (int m = 0; m < ROWS; ++m) {
        float4 v4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (x_init) v4 = *reinterpret_cast<const float4 *>(x_init + head_state + (int64_t)row_of(m) * D + j);
        X[0][m] = v4.x; X[1][m] = v4.y; X[2][m] = v4.z; X[3][m] = v4.w;
    }

    float pf_la[PF], pf_k[PF], pf_b[PF], pf_q[PF], pc0[PC], pc1[PC], pc2[PC];
    auto prefetch = [&](int64_t sb) {
        const int64_t t0 = sb * kSub;
#pragma unroll
        for (int x = 0; x < PF; ++x) {
            const int idx = tid + x * kScanThreads;
            const int tt = idx / D, i = idx % D;
            pf_la[x] = 0.f; pf_k[x] = 0.f; pf_b[x] = 0.f; pf_q[x] = 0.f;
            if (t0 + tt < len) {
                const int64_t off = ((start + t0 + tt) * p.H + h) * D + i;
                pf_la[x] = p.la[off];
                pf_k[x] = to_f32(K[off]);
                pf_b[x] = to_f32(Bg[off]);
                if (rev) pf_q[x] = to_f32(Q[off]);
            }
        }
#pragma unroll
        for (int x = 0; x < PC; ++x) {
            const int idx = tid + x * kScanThreads;
            const int tt = idx / kTile, jj = idx % kTile;
            pc0[x] = 0.f; pc1[x] = 0.f; pc2[x] = 0.f;
            if (t0 + tt < len) {
                const int64_t off = ((start + t0 + tt) * p.H + h) * D + tile * kTile + jj;
                const float vv = to_f32(V[off]), ww = to_f32(Wg[off]);
                if (rev) {
                    pc0[x] = to_f32(DO[off]);
                    pc1[x] = vv;
                    pc2[x] = ww;
                } else {
                    pc0[x] = ww * vv;
                }
            }
        }
    };

    constexpr int kSubPerChunk = kChunk / kSub;
    if (nsub > 0) prefetch(rev ? nsub - 1 : 0);
    for (int64_t it = 0; it < nsub; ++it) {
        const int64_t sb = rev ? nsub - 1 - it : it;
        __syncthreads();   // the previous round's shared reads are done
#pragma unroll
        for (int x = 0; x < PF; ++x) {
            const int idx = tid + x * kScanThreads;   // = tt * D + i
            s_al[idx] = expf(pf_la[x]);
            s_e[idx] = pf_b[x] * pf_k[x];
            s_k[idx] = pf_k[x];
            s_q[idx] = pf_q[x];
        }
#pragma unroll
        for (int x = 0; x < PC; ++x) {
            const int idx = tid + x * kScanThreads;   // = tt * kTile + jj
            s_c[0][idx] = pc0[x];
            s_c[1][idx] = pc1[x];
            s_c[2][idx] = pc2[x];
        }
        __syncthreads();
        if (rev ? sb > 0 : sb + 1 < nsub) prefetch(rev ? sb - 1 : sb + 1);

        const int L = (int)((len - sb * kSub) < kSub ? (len - sb * kSub) : kSub);
        const int64_t chunk = sb / kSubPerChunk;
        const bool at_chunk_edge = rev ? (sb % kSubPerChunk == kSubPerChunk - 1 || sb == nsub - 1)
                                       : (sb % kSubPerChunk == 0);
        if (at_chunk_edge) {
            // A: state at the chunk start; B: cotangent of the state at the chunk end
            float *dst = (rev ? p.gk : p.ck) + ((base + chunk) * p.H + h) * (int64_t)D * D;
#pragma unroll
            for (int m = 0; m < ROWS; ++m)
                *reinterpret_cast<float4 *>(dst + (int64_t)row_of(m) * D + j) =
                    make_float4(X[0][m], X[1][m], X[2][m], X[3][m]);
        }

        if (!rev) {
            for (int tt = 0; tt < L; ++tt) {
                const int64_t tok = start + sb * kSub + tt;
                float r[NC] = {0.f, 0.f, 0.f, 0.f}, al[ROWS], ee[ROWS], kk[ROWS];
                load_row_groups<ROWS, GS>(s_al + tt * D + row0, al);
                load_row_groups<ROWS, GS>(s_e + tt * D + row0, ee);
                load_row_groups<ROWS, GS>(s_k + tt * D + row0, kk);
#pragma unroll
                for (int m = 0; m < ROWS; ++m)
#pragma unroll
                    for (int c = 0; c < NC; ++c) {
                        X[c][m] *= al[m];                     // S' = Diag(alpha) S
                        r[c] = fmaf(X[c][m], ee[m], r[c]);    // r = S'^T e
                    }
#pragma unroll
                for (int off = 8; off >= 1; off >>= 1)
#pragma unroll
                    for (int c = 0; c < NC; ++c) r[c] += __shfl_xor_sync(0xffffffffu, r[c], off);
                const float4 z4 = *reinterpret_cast<const float4 *>(&s_c[0][tt * kTile + jl]);
                const float u[NC] = {z4.x - r[0], z4.y - r[1], z4.z - r[2], z4.w - r[3]};
#pragma unroll
                for (int m = 0; m < ROWS; ++m)
#pragma unroll
                    for (int c = 0; c < NC; ++c) X[c][m] = fmaf(kk[m], u[c], X[c][m]);   // S = S' + k u^T
                if ((lane & 15) == 0)
                    *reinterpret_cast<float4 *>(p.U + (tok * p.H + h) * D + j) = make_float4(u[0], u[1], u[2], u[3]);
            }
        } else {
            for (int tt = L - 1; tt >= 0; --tt) {
                const int64_t tok = start + sb * kSub + tt;
                const int cb = tt * kTile + jl;
                const float4 o4 = *reinterpret_cast<const float4 *>(&s_c[0][cb]);
                const float oo[NC] = {o4.x, o4.y, o4.z, o4.w};
                float d[NC] = {0.f, 0.f, 0.f, 0.f}, qq[ROWS], kk[ROWS], al[ROWS], ee[ROWS];
                load_row_groups<ROWS, GS>(s_q + tt * D + row0, qq);
                load_row_groups<ROWS, GS>(s_k + tt * D + row0, kk);
                load_row_groups<ROWS, GS>(s_al + tt * D + row0, al);
                load_row_groups<ROWS, GS>(s_e + tt * D + row0, ee);
#pragma unroll
                for (int m = 0; m < ROWS; ++m)
#pragma unroll
                    for (int c = 0; c < NC; ++c) {
                        X[c][m] = fmaf(qq[m], oo[c], X[c][m]);   // H = G + q do^T
                        d[c] = fmaf(X[c][m], kk[m], d[c]);       // du = H^T k
                    }
#pragma unroll
                for (int off = 8; off >= 1; off >>= 1)
#pragma unroll
                    for (int c = 0; c < NC; ++c) d[c] += __shfl_xor_sync(0xffffffffu, d[c], off);
#pragma unroll
                for (int m = 0; m < ROWS; ++m)
#pragma unroll
                    for (int c = 0; c < NC; ++c) X[c][m] = al[m] * fmaf(-ee[m], d[c], X[c][m]);  // G = Diag(alpha)(H - e du^T)
                if ((lane & 15) == 0) {
                    const int64_t off = (tok * p.H + h) * D + j;
                    const float4 v4 = *reinterpret_cast<const float4 *>(&s_c[1][cb]);
                    const float4 w4 = *reinterpret_cast<const float4 *>(&s_c[2][cb]);
                    *reinterpret_cast<float4 *>(p.dU + off) = make_float4(d[0], d[1], d[2], d[3]);
                    Tin *dvp = static_cast<Tin *>(p.dv) + off, *dwp = static_cast<Tin *>(p.dw) + off;
                    store2(dvp, d[0] * w4.x, d[1] * w4.y);       // dv = du . w
                    store2(dvp + 2, d[2] * w4.z, d[3] * w4.w);
                    store2(dwp, d[0] * v4.x, d[1] * v4.y);       // dw = du . v
                    store2(dwp + 2, d[2] * v4.z, d[3] * v4.w);
                }
            }
        }
    }
    if (rev && p.d_init) {
#pragma unroll
        for (int m = 0; m < ROWS; ++m)
            *reinterpret_cast<float4 *>(p.d_init + head_state + (int64_t)row_of(m) * D + j) =
                make_float4(X[0][m], X[1][m], X[2][m], X[3][m]);
    }
}

// Sweep C. CTA = (checkpoint slot, head); thread = (key rows rg + 64r, lane s
// of 4), lane s holding value columns 4(s + 4g) .. +3. Row reductions over
// value columns are two xor-shuffles inside each group of 4 lanes. The chunk's
// u, du and dO rows are copied to shared memory once (cp.async) and read from
// there by both passes; the per-row scalars of the next token are loaded while
// the current one is processed.
template <typename Tin, int D>
constexpr size_t rows_smem_bytes()
{
    return (size_t)kChunk * D * (3 * sizeof(float) + sizeof(Tin));
}

template <typename Tin, int D>
__global__ void __launch_bounds__(kRowThreads, 2) bwd_rows_kernel(BwdParams p)
{
    constexpr int RPT = D / 64;   // key rows per thread
    constexpr int NG = D / 16;    // float4 column groups per thread
    extern __shared__ __align__(16) unsigned char rows_smem[];
    float *s_u = reinterpret_cast<float *>(rows_smem);   // [kChunk][D] u
    float *s_du = s_u + kChunk * D;                       // [kChunk][D] du
    float *s_g = s_du + kChunk * D;                       // [kChunk][D] dkW, then the decay terms
    Tin *s_do = reinterpret_cast<Tin *>(s_g + kChunk * D);  // [kChunk][D] dO

    const int64_t slot = blockIdx.x;
    const int h = blockIdx.y;
    // the sequence that owns this slot: the last n with slot_base(n) <= slot
    int64_t lo = 0, hi = p.N - 1;
    while (lo < hi) {
        const int64_t mid = (lo + hi + 1) >> 1;
        int64_t s_mid, l_mid;
        seq_bounds(p, mid, s_mid, l_mid);
        if (slot_base(s_mid, mid) <= slot) lo = mid;
        else hi = mid - 1;
    }
    int64_t start, len;
    seq_bounds(p, lo, start, len);
    const int64_t c = slot - slot_base(start, lo);
    if (c < 0 || c * kChunk >= len) return;   // an unused slot
    const int64_t t0 = start + c * kChunk;
    const int L = (int)((len - c * kChunk) < kChunk ? (len - c * kChunk) : kChunk);

    const int tid = threadIdx.x, s = tid & 3, rg = tid >> 2;
    const Tin *Q = static_cast<const Tin *>(p.q), *K = static_cast<const Tin *>(p.k);
    const Tin *Bg = static_cast<const Tin *>(p.b), *DO = static_cast<const Tin *>(p.d_o);
    const int64_t slot_off = (slot * p.H + h) * (int64_t)D * D;

    // stage u, du (fp32) and dO (Tin) of the chunk's L tokens
    {
        constexpr int F4 = D / 4;                       // 16-byte pieces per fp32 row
        constexpr int T16 = D * (int)sizeof(Tin) / 16;  // 16-byte pieces per dO row
        for (int idx = tid; idx < L * F4; idx += kRowThreads) {
            const int tt = idx / F4, q4 = idx % F4;
            const int64_t g = ((t0 + tt) * p.H + h) * D + 4 * q4;
            cp_async16(s_u + tt * D + 4 * q4, p.U + g);
            cp_async16(s_du + tt * D + 4 * q4, p.dU + g);
        }
        for (int idx = tid; idx < L * T16; idx += kRowThreads) {
            const int tt = idx / T16, q16 = idx % T16;
            constexpr int E = 16 / (int)sizeof(Tin);    // elements per piece
            cp_async16(s_do + tt * D + E * q16, DO + ((t0 + tt) * p.H + h) * D + E * q16);
        }
        cp_async_wait_all();
        __syncthreads();
    }

    float X[RPT][NG][4];
    // pass R: H from the chunk-end cotangent, tokens in reverse
#pragma unroll
    for (int r = 0; r < RPT; ++r)
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const float4 v4 = *reinterpret_cast<const float4 *>(p.gk + slot_off + (int64_t)(rg + 64 * r) * D + 4 * (s + 4 * g));
            X[r][g][0] = v4.x; X[r][g][1] = v4.y; X[r][g][2] = v4.z; X[r][g][3] = v4.w;
        }
    // per-row scalars of the next token to process (prefetched one token ahead)
    float nq[RPT], nk[RPT], nb[RPT], nla[RPT];
    auto load_scalars = [&](int tt) {
        const int64_t row0 = ((t0 + tt) * p.H + h) * D;
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int64_t o = row0 + rg + 64 * r;
            nq[r] = to_f32(Q[o]);
            nk[r] = to_f32(K[o]);
            nb[r] = to_f32(Bg[o]);
            nla[r] = p.la[o];
        }
    };
    load_scalars(L - 1);
    for (int tt = L - 1; tt >= 0; --tt) {
        float qr[RPT], ar[RPT], er[RPT], acc[RPT];
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            qr[r] = nq[r];
            ar[r] = expf(nla[r]);
            er[r] = nb[r] * nk[r];
            acc[r] = 0.f;
        }
        if (tt > 0) load_scalars(tt - 1);
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const int col = 4 * (s + 4 * g);
            float o4[4];
            load_vec<Tin, 4>(s_do + tt * D + col, o4);
            const float4 u4 = *reinterpret_cast<const float4 *>(s_u + tt * D + col);
            const float4 d4 = *reinterpret_cast<const float4 *>(s_du + tt * D + col);
            const float uu[4] = {u4.x, u4.y, u4.z, u4.w}, dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
            for (int r = 0; r < RPT; ++r)
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    float hv = fmaf(qr[r], o4[x], X[r][g][x]);   // H = G + q do^T
                    acc[r] = fmaf(hv, uu[x], acc[r]);            // dkW = H u
                    X[r][g][x] = ar[r] * fmaf(-er[r], dd[x], hv); // G = alpha (H - e du^T)
                }
        }
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 1);
            acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], 2);
            if (s == 0) s_g[tt * D + rg + 64 * r] = acc[r];
        }
    }
    __syncwarp();

    // pass F: S from the chunk-start state, tokens in order
#pragma unroll
    for (int r = 0; r < RPT; ++r)
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const float4 v4 = *reinterpret_cast<const float4 *>(p.ck + slot_off + (int64_t)(rg + 64 * r) * D + 4 * (s + 4 * g));
            X[r][g][0] = v4.x; X[r][g][1] = v4.y; X[r][g][2] = v4.z; X[r][g][3] = v4.w;
        }
    Tin *DQ = static_cast<Tin *>(p.dq), *DK = static_cast<Tin *>(p.dk), *DB = static_cast<Tin *>(p.db);
    load_scalars(0);
    for (int tt = 0; tt < L; ++tt) {
        const int64_t row0 = ((t0 + tt) * p.H + h) * D;
        float qr[RPT], kr[RPT], br[RPT], ar[RPT], de[RPT], dq[RPT];
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            qr[r] = nq[r];
            kr[r] = nk[r];
            br[r] = nb[r];
            ar[r] = expf(nla[r]);
            de[r] = 0.f;
            dq[r] = 0.f;
        }
        if (tt + 1 < L) load_scalars(tt + 1);
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const int col = 4 * (s + 4 * g);
            float o4[4];
            load_vec<Tin, 4>(s_do + tt * D + col, o4);
            const float4 u4 = *reinterpret_cast<const float4 *>(s_u + tt * D + col);
            const float4 d4 = *reinterpret_cast<const float4 *>(s_du + tt * D + col);
            const float uu[4] = {u4.x, u4.y, u4.z, u4.w}, dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
            for (int r = 0; r < RPT; ++r)
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const float sp = ar[r] * X[r][g][x];          // S' = alpha S
                    de[r] = fmaf(sp, dd[x], de[r]);               // S' du
                    X[r][g][x] = fmaf(kr[r], uu[x], sp);          // S = S' + k u^T
                    dq[r] = fmaf(X[r][g][x], o4[x], dq[r]);       // S do
                }
        }
        float dkv[RPT], dbv[RPT], dgv[RPT];
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            de[r] += __shfl_xor_sync(0xffffffffu, de[r], 1);
            de[r] += __shfl_xor_sync(0xffffffffu, de[r], 2);
            dq[r] += __shfl_xor_sync(0xffffffffu, dq[r], 1);
            dq[r] += __shfl_xor_sync(0xffffffffu, dq[r], 2);
            const float dev = -de[r];
            const float dkw = s_g[tt * D + rg + 64 * r];
            dkv[r] = fmaf(br[r], dev, dkw);                       // dk = dkW + b . de
            dbv[r] = kr[r] * dev;                                 // db = k . de
            dgv[r] = qr[r] * dq[r] - kr[r] * dkw + br[r] * kr[r] * dev;  // q.dq - k.dkW + e.de
        }
        __syncwarp();   // every lane has read s_g[tt] before lane 3 overwrites it
#pragma unroll
        for (int r = 0; r < RPT; ++r) {
            const int64_t o = row0 + rg + 64 * r;
            if (s == 0) DQ[o] = from_f32<Tin>(dq[r]);
            else if (s == 1) DK[o] = from_f32<Tin>(dkv[r]);
            else if (s == 2) DB[o] = from_f32<Tin>(dbv[r]);
            else s_g[tt * D + rg + 64 * r] = dgv[r];
        }
    }
    // rowsum(G_end . S_end), then the reverse cumulative sum of the decay terms
    float bt[RPT];
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        bt[r] = 0.f;
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            const float4 v4 = *reinterpret_cast<const float4 *>(p.gk + slot_off + (int64_t)(rg + 64 * r) * D + 4 * (s + 4 * g));
            bt[r] = fmaf(v4.x, X[r][g][0], bt[r]);
            bt[r] = fmaf(v4.y, X[r][g][1], bt[r]);
            bt[r] = fmaf(v4.z, X[r][g][2], bt[r]);
            bt[r] = fmaf(v4.w, X[r][g][3], bt[r]);
        }
        bt[r] += __shfl_xor_sync(0xffffffffu, bt[r], 1);
        bt[r] += __shfl_xor_sync(0xffffffffu, bt[r], 2);
    }
    __syncwarp();   // lane 3's decay terms are visible to the lanes that sum them
#pragma unroll
    for (int r = 0; r < RPT; ++r) {
        if (s == r) {
            float acc = bt[r];
            for (int tt = L - 1; tt >= 0; --tt) {
                acc += s_g[tt * D + rg + 64 * r];
                p.dla[((t0 + tt) * p.H + h) * D + rg + 64 * r] = acc;
            }
        }
    }
}

template <typename Tin, int D>
cudaError_t launch_typed(const BwdParams &p, int64_t slots, cudaStream_t stream)
{
    if (p.N * p.H > 0) {
        dim3 grid((unsigned)(p.N * p.H), D / kTile, 2);
        bwd_scan_kernel<Tin, D><<<grid, kScanThreads, 0, stream>>>(p);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (p.tokens > 0) {
        constexpr size_t smem = rows_smem_bytes<Tin, D>();
        cudaError_t e = ensure_dynamic_smem((const void *)bwd_rows_kernel<Tin, D>, (int)smem);
        if (e != cudaSuccess) return e;
        dim3 grid((unsigned)slots, (unsigned)p.H);
        bwd_rows_kernel<Tin, D><<<grid, kRowThreads, smem, stream>>>(p);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

}  // namespace

int64_t bwd_slots(int64_t tokens, int64_t num_seqs) { return tokens / kChunk + num_seqs; }

size_t bwd_workspace_bytes(int64_t tokens, int64_t H, int64_t d, int64_t num_seqs)
{
    const size_t states = (size_t)bwd_slots(tokens, num_seqs) * H * d * d * sizeof(float);
    const size_t vecs = (size_t)tokens * H * d * sizeof(float);
    const size_t bytes = 2 * states + 2 * vecs;
    return (bytes + 255) & ~(size_t)255;
}

cudaError_t launch_chunk_bwd(const BwdArgs &a, cudaStream_t stream)
{
    BwdParams p;
    p.q = a.q; p.k = a.k; p.v = a.v; p.b = a.b; p.w = a.w; p.d_o = a.d_o;
    p.la = a.log_alpha; p.init_state = a.init_state; p.d_final = a.d_final;
    p.cu = a.cu_seqlens;
    p.dq = a.dq; p.dk = a.dk; p.dv = a.dv; p.db = a.db; p.dw = a.dw;
    p.dla = a.d_log_alpha; p.d_init = a.d_init_state;
    p.T = a.T; p.H = a.H; p.N = a.num_seqs; p.tokens = a.B * a.T;
    const int64_t slots = bwd_slots(p.tokens, p.N);
    const size_t states = (size_t)slots * a.H * a.d * a.d;
    float *ws = static_cast<float *>(a.workspace);
    p.ck = ws;
    p.gk = ws + states;
    p.U = ws + 2 * states;
    p.dU = p.U + (size_t)p.tokens * a.H * a.d;
    if (a.bf16)
        return a.d == 128 ? launch_typed<__nv_bfloat16, 128>(p, slots, stream)
                          : launch_typed<__nv_bfloat16, 64>(p, slots, stream);
    return a.d == 128 ? launch_typed<float, 128>(p, slots, stream) : launch_typed<float, 64>(p, slots, stream);
}

}  // namespace gdr2
