// Segment-parallel scan for few long sequences (bf16, d = 128, fixed-length
// batches): the serial chunk chain of each (sequence, head) is cut into nseg
// segments that run concurrently, and a short fix-up restores the exact
// result.
//
// The recurrence is affine in the state. Over segment p, starting from S,
//     S_t = Phi_t S + S0_t,      o_t = S0_t^T q_t + S^T psi_t,  psi_t = Phi_t^T q_t,
// where S0_t is the state reached from S = 0 and Phi_t is the product of the
// segment's transitions (I - k e^T) Diag(alpha) up to t. The chunk kernel runs,
// all at once:
//   pass A, every segment, from the true initial state (segment 0) or from 0:
//       o (partial for p >= 1) and the segment's final state S0_p;
//   pass B, every segment p >= 1, from the identity with z = 0 (so that the
//       "state" is Phi_t and the "output" is psi_t): psi into scratch and Phi_p.
// Then, per (sequence, head):
//   combine: S_start(1) = S0_0; S_start(p+1) = Phi_p S_start(p) + S0_p; the
//       last one is the final state;
//   correct: o_t += S_start(p)^T psi_t for every token of segment p >= 1 (on the
//       tensor cores, with S_start split into bf16 hi + lo parts).
// (Chunkwise form of the Gated DeltaNet-2 pages' rule; the split is the
// affine-map scan of the state, computed in fp32.)
#include "common.cuh"
#include "kernels.h"

namespace gdr2 {

namespace {

constexpr int kD = 128;
constexpr int64_t kStateElems = (int64_t)kD * kD;
// (main, helper) CTA pairs the chunk kernel keeps resident at once on a
// 148-SM B200; a split is used only while all its jobs fit in one wave.
constexpr int64_t kMaxPairs = 64;
constexpr int64_t kMinSegChunks = 8;   // no segment shorter than 8 chunks
constexpr int kMaxSegments = 16;

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Per (sequence, head): S <- S0_0, then for p = 1..nseg-1 S <- Phi_p S + S0_p,
// storing the entry state S of segment p (transposed, as bf16 hi + lo) over
// Phi_p once that is read; finally the final state. 512 threads; thread t owns row t/4 and the 32
// columns 4 (t%4) + 16 m + {0..3}, m = 0..7 (a warp's reads of one S row are
// 4 adjacent 16-byte pieces: no bank conflicts).
__global__ void __launch_bounds__(512)
seg_combine_kernel(const float *__restrict__ s0, float *__restrict__ phi_w, float *__restrict__ final_state,
                   int nseg, int64_t H)
{
    const float *phi = phi_w;
    extern __shared__ float4 S4[];  // the running state, [128][128] fp32
    float *S = reinterpret_cast<float *>(S4);
    const int tid = threadIdx.x;
    const int64_t h = blockIdx.x % H, n = blockIdx.x / H;
    auto slot = [&](int p) { return ((n * nseg + p) * H + h) * kStateElems; };
    const int r = tid >> 2, cq = 4 * (tid & 3);
    for (int i = tid; i < (int)(kStateElems / 4); i += 512)
        S4[i] = reinterpret_cast<const float4 *>(s0 + slot(0))[i];
    __syncthreads();
    for (int p = 1; p < nseg; ++p) {
        float4 acc[8];
        const float *s0p = s0 + slot(p) + r * kD + cq;
#pragma unroll
        for (int m = 0; m < 8; ++m) acc[m] = *reinterpret_cast<const float4 *>(s0p + 16 * m);
        const float *phr = phi + slot(p) + r * kD;
#pragma unroll 4
        for (int k = 0; k < kD; ++k) {
            const float a = phr[k];
            const float *srow = S + k * kD + cq;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const float4 x = *reinterpret_cast<const float4 *>(srow + 16 * m);
                acc[m].x = fmaf(a, x.x, acc[m].x);
                acc[m].y = fmaf(a, x.y, acc[m].y);
                acc[m].z = fmaf(a, x.z, acc[m].z);
                acc[m].w = fmaf(a, x.w, acc[m].w);
            }
        }
        __syncthreads();  // every read of S and of Phi_p for this step is done
        // entry state of segment p, transposed and split into bf16 hi + lo, over
        // Phi_p (no longer needed): [hi: 128 x 128][lo: 128 x 128], element (j, k) = S[k][j]
        __nv_bfloat16 *sth = reinterpret_cast<__nv_bfloat16 *>(phi_w + slot(p));
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const float4 x = *reinterpret_cast<const float4 *>(S + r * kD + cq + 16 * m);
            const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int j = cq + 16 * m + e;
                const __nv_bfloat16 hi = __float2bfloat16_rn(xs[e]);
                sth[j * kD + r] = hi;
                sth[kStateElems + j * kD + r] = __float2bfloat16_rn(xs[e] - __bfloat162float(hi));
            }
        }
        __syncthreads();
#pragma unroll
        for (int m = 0; m < 8; ++m) *reinterpret_cast<float4 *>(S + r * kD + cq + 16 * m) = acc[m];
        __syncthreads();
    }
    if (final_state) {
        float *dst = final_state + (n * H + h) * kStateElems + r * kD + cq;
#pragma unroll
        for (int m = 0; m < 8; ++m)
            *reinterpret_cast<float4 *>(dst + 16 * m) = *reinterpret_cast<const float4 *>(S + r * kD + cq + 16 * m);
    }
}

constexpr int kFixTok = 64;     // tokens per tile (4 warps x 16 rows)
constexpr int kFixTiles = 16;   // tiles per CTA (the entry state is staged once per 1024 tokens)
constexpr int kPitch = 272;     // bytes per staged 128-element bf16 row (16 B pad: ldmatrix
                                // rows of one 8x8 matrix fall in distinct bank groups)

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// o_t += S_start(p)^T psi_t for the tokens of segments p >= 1, on the tensor
// cores: O_tile (tokens x 128) += Psi_tile (tokens x 128, bf16) * S with
// S = S_hi + S_lo split into two bf16 parts (so the product keeps about 16
// mantissa bits of S) and fp32 accumulation. CTA: up to 256 tokens of one
// (sequence, head) inside one segment; warp w: 16 tokens of each 64-token
// tile, all 128 output channels (16 n-tiles of 8).
__global__ void __launch_bounds__(128)
seg_correct_kernel(__nv_bfloat16 *__restrict__ o, const __nv_bfloat16 *__restrict__ psi,
                   const float *__restrict__ sth_f, int nseg, int64_t seg_len, int64_t T, int64_t H)
{
    extern __shared__ __align__(16) unsigned char fix_smem[];
    // (each state slot holds 64 KB: the bf16 hi and lo halves of S^T)
    const __nv_bfloat16 *sth = reinterpret_cast<const __nv_bfloat16 *>(sth_f);
    unsigned char *st_hi = fix_smem;                  // S^T hi: [128 out channels][128 k] bf16, kPitch
    unsigned char *st_lo = fix_smem + kD * kPitch;    // S^T lo
    unsigned char *pt = fix_smem + 2 * kD * kPitch;   // psi tile: [64 tokens][128 k] bf16, kPitch
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t h = blockIdx.y, n = blockIdx.z;
    const int64_t per_seg = (seg_len + kFixTok * kFixTiles - 1) / (kFixTok * kFixTiles);
    const int p = 1 + (int)(blockIdx.x / per_seg);
    const int64_t tb = p * seg_len + (int64_t)(blockIdx.x % per_seg) * kFixTok * kFixTiles;  // first token
    const int64_t seg_end = (p + 1) * seg_len < T ? (p + 1) * seg_len : T;
    if (tb >= seg_end) return;
    // stage S^T hi and lo (written by the combine step, bf16 [j][k]), 16-byte pieces
    const uint4 *src = reinterpret_cast<const uint4 *>(sth + ((n * nseg + p) * H + h) * 2 * kStateElems);
    for (int i = tid; i < 2 * kD * kD / 8; i += 128) {
        const int row = i >> 4, piece = i & 15;  // rows 0-127 hi, 128-255 lo
        *reinterpret_cast<uint4 *>(fix_smem + row * kPitch + 16 * piece) = src[i];
    }
    // ldmatrix lane addresses: A (psi rows of this warp), B (S^T rows = output channels)
    const int a_row = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1), a_k = 8 * (lane >> 4);
    const int b_row = (lane & 7) + 8 * (lane >> 4), b_k = 8 * ((lane >> 3) & 1);
    const uint32_t a_base = smem_addr(pt) + a_row * kPitch + 2 * a_k;
    const uint32_t bh_base = smem_addr(st_hi) + b_row * kPitch + 2 * b_k;
    const uint32_t bl_base = smem_addr(st_lo) + b_row * kPitch + 2 * b_k;
    const int g = lane >> 2, t4 = lane & 3;
    for (int tile = 0; tile < kFixTiles; ++tile) {
        const int64_t t0 = tb + tile * kFixTok;
        if (t0 >= seg_end) break;
        __syncthreads();  // (S staged / previous tile's psi consumed)
        for (int i = tid; i < kFixTok * kD / 8; i += 128) {  // psi rows, 16 B pieces
            const int rr = i >> 4, piece = i & 15;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (t0 + rr < seg_end)
                v = *reinterpret_cast<const uint4 *>(psi + ((n * T + t0 + rr) * H + h) * kD + 8 * piece);
            *reinterpret_cast<uint4 *>(pt + rr * kPitch + 16 * piece) = v;
        }
        __syncthreads();
        float acc[16][4];
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll 2
        for (int kk = 0; kk < kD; kk += 16) {
            uint32_t a[4];
            ldmatrix_x4(a, a_base + 2 * kk);
#pragma unroll
            for (int np = 0; np < 8; ++np) {  // n-tile pairs
                uint32_t bh[4], bl[4];
                ldmatrix_x4(bh, bh_base + np * 16 * kPitch + 2 * kk);
                ldmatrix_x4(bl, bl_base + np * 16 * kPitch + 2 * kk);
                mma_bf16_16816(acc[2 * np], a, bh[0], bh[1]);
                mma_bf16_16816(acc[2 * np], a, bl[0], bl[1]);
                mma_bf16_16816(acc[2 * np + 1], a, bh[2], bh[3]);
                mma_bf16_16816(acc[2 * np + 1], a, bl[2], bl[3]);
            }
        }
        // o (rows g, g+8 of this warp's 16; channels 8 nt + 2 t4, +1) += acc
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            const int64_t t = t0 + 16 * warp + g + 8 * half;
            if (t >= seg_end) continue;
            __nv_bfloat16 *orow = o + ((n * T + t) * H + h) * kD + 2 * t4;
#pragma unroll
            for (int nt = 0; nt < 16; ++nt) {
                __nv_bfloat162 *po = reinterpret_cast<__nv_bfloat162 *>(orow + 8 * nt);
                const float2 f = __bfloat1622float2(*po);
                *po = __floats2bfloat162_rn(f.x + acc[nt][2 * half], f.y + acc[nt][2 * half + 1]);
            }
        }
    }
}

}  // namespace

size_t seg_psi_offset() { return 0; }

size_t seg_state_offset(int64_t B, int64_t T, int64_t H)
{
    return align256((size_t)B * T * H * kD * 2);
}

size_t seg_phi_offset(int64_t B, int64_t T, int64_t H, int nseg)
{
    return seg_state_offset(B, T, H) + align256((size_t)B * nseg * H * kStateElems * 4);
}

SegPlan plan_segments(int64_t B, int64_t T, int64_t H, int64_t d, bool bf16)
{
    SegPlan plan{1, 0, 0};
    if (!bf16 || d != kD || B <= 0 || T <= 0 || H <= 0) return plan;
    const int64_t units = B * H, nc = (T + 63) / 64;
    int best = 1;
    for (int P = 2; P <= kMaxSegments; ++P) {
        if (units * (2 * P - 1) > kMaxPairs || nc < kMinSegChunks * P) break;
        best = P;
    }
    if (best == 1) return plan;
    const int64_t seg_chunks = (nc + best - 1) / best;
    const int nseg = (int)((nc + seg_chunks - 1) / seg_chunks);  // every segment non-empty
    if (nseg < 2) return plan;
    plan.nseg = nseg;
    plan.seg_len = 64 * seg_chunks;
    plan.ws_bytes = seg_phi_offset(B, T, H, nseg) + align256((size_t)B * nseg * H * kStateElems * 4);
    return plan;
}

cudaError_t launch_segment_fix(const ChunkArgs &a, cudaStream_t stream)
{
    unsigned char *ws = static_cast<unsigned char *>(a.seg_ws);
    float *s0 = reinterpret_cast<float *>(ws + seg_state_offset(a.B, a.T, a.H));
    float *phi = reinterpret_cast<float *>(ws + seg_phi_offset(a.B, a.T, a.H, a.nseg));
    const __nv_bfloat16 *psi = reinterpret_cast<const __nv_bfloat16 *>(ws + seg_psi_offset());
    const int comb_smem = (int)(kStateElems * 4);
    cudaError_t e = ensure_dynamic_smem((const void *)seg_combine_kernel, comb_smem);
    if (e != cudaSuccess) return e;
    seg_combine_kernel<<<(unsigned)(a.B * a.H), 512, comb_smem, stream>>>(s0, phi, a.final_state, a.nseg, a.H);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int fix_smem = (2 * kD + kFixTok) * kPitch;
    e = ensure_dynamic_smem((const void *)seg_correct_kernel, fix_smem);
    if (e != cudaSuccess) return e;
    const int64_t per_seg = (a.seg_len + kFixTok * kFixTiles - 1) / (kFixTok * kFixTiles);
    const int64_t ntiles = per_seg * (a.nseg - 1);  // segments 1..nseg-1
    dim3 grid((unsigned)ntiles, (unsigned)a.H, (unsigned)a.B);
    seg_correct_kernel<<<grid, 128, fix_smem, stream>>>(static_cast<__nv_bfloat16 *>(a.o), psi, phi, a.nseg,
                                                       a.seg_len, a.T, a.H);
    return cudaGetLastError();
}

}  // namespace gdr2
