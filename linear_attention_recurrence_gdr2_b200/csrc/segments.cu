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
#include "sm100.cuh"

#include <mutex>

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

// One step of the chain of segment entry states, S_start(1) = S0_0 and
//     S_start(p+1) = Phi_p S_start(p) + S0_p,
// with the rows of the result split over kCombCtas CTAs per (sequence, head).
// Step p reads S_start(p) from state slot p-1 and writes S_start(p+1) over
// slot p (each CTA reads its own rows of S0_p before it writes them), or, after
// the last segment, into the final state. 256 threads; thread t owns row
// t / 16 of the CTA's 16 and the 8 columns 8 (t % 16) + {0..7}.
constexpr int kCombRows = 16;
constexpr int kCombCtas = kD / kCombRows;
__global__ void __launch_bounds__(256)
seg_combine_kernel(float *__restrict__ s0, const float *__restrict__ phi, float *__restrict__ final_state,
                   int nseg, int p, int64_t H)
{
    extern __shared__ float4 comb4[];
    float *Ss = reinterpret_cast<float *>(comb4);    // S_start(p), [128][128]
    float *Ph = Ss + kStateElems;                    // the CTA's rows of Phi_p, [16][128]
    const int tid = threadIdx.x;
    const int64_t h = blockIdx.y, n = blockIdx.z;
    const int r0 = kCombRows * (int)blockIdx.x;
    auto slot = [&](int q) { return ((n * nseg + q) * H + h) * kStateElems; };
    // (all loads of a thread are issued before its first store, so their
    // latencies overlap)
    const float4 *src = reinterpret_cast<const float4 *>(s0 + slot(p - 1));
    const float4 *prow = reinterpret_cast<const float4 *>(phi + slot(p) + (int64_t)r0 * kD);
    {
        float4 x[kStateElems / 4 / 256], y[kCombRows * kD / 4 / 256];
#pragma unroll
        for (int i = 0; i < (int)(kStateElems / 4 / 256); ++i) x[i] = src[tid + 256 * i];
#pragma unroll
        for (int i = 0; i < kCombRows * kD / 4 / 256; ++i) y[i] = prow[tid + 256 * i];
#pragma unroll
        for (int i = 0; i < (int)(kStateElems / 4 / 256); ++i) comb4[tid + 256 * i] = x[i];
#pragma unroll
        for (int i = 0; i < kCombRows * kD / 4 / 256; ++i) comb4[kStateElems / 4 + tid + 256 * i] = y[i];
    }
    __syncthreads();
    const int rr = tid >> 4, c8 = 8 * (tid & 15);
    const float *s0r = s0 + slot(p) + (int64_t)(r0 + rr) * kD + c8;
    const float4 b0 = *reinterpret_cast<const float4 *>(s0r), b1 = *reinterpret_cast<const float4 *>(s0r + 4);
    float acc[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll 8
    for (int k = 0; k < kD; ++k) {
        const float a = Ph[rr * kD + k];
        const float4 x0 = *reinterpret_cast<const float4 *>(Ss + k * kD + c8);
        const float4 x1 = *reinterpret_cast<const float4 *>(Ss + k * kD + c8 + 4);
        acc[0] = fmaf(a, x0.x, acc[0]); acc[1] = fmaf(a, x0.y, acc[1]);
        acc[2] = fmaf(a, x0.z, acc[2]); acc[3] = fmaf(a, x0.w, acc[3]);
        acc[4] = fmaf(a, x1.x, acc[4]); acc[5] = fmaf(a, x1.y, acc[5]);
        acc[6] = fmaf(a, x1.z, acc[6]); acc[7] = fmaf(a, x1.w, acc[7]);
    }
    float *dst = p + 1 < nseg ? s0 + slot(p) : (final_state ? final_state + (n * H + h) * kStateElems : nullptr);
    if (dst) {
        float *d = dst + (int64_t)(r0 + rr) * kD + c8;
        *reinterpret_cast<float4 *>(d) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        *reinterpret_cast<float4 *>(d + 4) = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

// ---- the correction o_t += S_start(p)^T psi_t on tcgen05 -------------------
// Per 128-token tile of segment p >= 1: D (tokens x 128 out channels, fp32 in
// TMEM) = Psi (tokens x 128 k, bf16) * S_start(p), with S_start(p) (fp32,
// state slot p-1 after the combine steps) split into bf16 hi and lo parts and
// staged as the MMA's B operand in its MN-major layout (rows k, output
// channels contiguous, as S is stored); both parts accumulate into the same D
// (the product keeps about 16 mantissa bits of S). One CTA stages S once and
// runs up to kCorrTiles tiles of one (sequence, head): warp 0 loads Psi tiles
// by TMA (two slots), warp 1 issues
// the 16 MMAs of a tile into one of two TMEM accumulators, warps 4-11 add the
// accumulator to o (thread = token row = TMEM lane, two warps per lane quarter
// taking 64 output channels each). The tile's o rows arrive by TMA with its
// Psi rows, so the epilogue reads them from shared memory and only stores to
// global memory. Every wait is bounded.
constexpr int kCorrRows = 128;     // tokens per tile (the MMA's M)
constexpr int kCorrTiles = 16;     // tiles per CTA: S is staged once per 2048 tokens
constexpr int kCorrThreads = 384;  // warp 0 TMA, warp 1 MMA, warp 2 TMEM, warps 4-11 epilogue
constexpr uint32_t kCB = 0;        // S [part hi, lo][j half][128 k rows x 128 B], 64 KB
constexpr uint32_t kCA = 65536;    // Psi slots [2][k half][128 rows x 128 B], 32 KB each
constexpr uint32_t kCO = 131072;   // o slots, the same layout (channel halves apart)
constexpr uint32_t kCBar = 196608;
enum { C_FULL0 = 0, C_FULL1, C_FREE0, C_FREE1, C_ACC0, C_ACC1, C_ACCFREE0, C_ACCFREE1, C_DRAIN, C_NUM };
constexpr uint32_t kCMisc = kCBar + C_NUM * 8;      // TMEM base, abort flag
constexpr uint32_t kCorrSmem = kCMisc + 16 + 1024;  // + alignment slack
constexpr uint64_t kCorrWaitNs = 1000000000ull;     // one second per wait
constexpr uint32_t kBarEpiC = 1;                    // named barrier of the epilogue warps

__device__ int g_seg_error;

// Bounded wait: one blocking probe, then the timed loop (which records `site`
// in the error word and raises the CTA's abort flag when the limit passes).
__device__ __forceinline__ bool cwait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int site) {
    if (sm100::mbar_try(bar, parity)) return true;
    sm100::WaitGuard g{kCorrWaitNs, abort_flag, &g_seg_error};
    return sm100::mbar_wait(bar, parity, g, site);
}
// Barrier over an n-thread group that ANDs one predicate across it.
__device__ __forceinline__ bool group_all(uint32_t id, uint32_t n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r) : "r"((uint32_t)v), "r"(id), "r"(n) : "memory");
    return r != 0;
}

__global__ void __launch_bounds__(kCorrThreads, 1)
seg_correct_kernel(const __grid_constant__ CUtensorMap map_psi, const __grid_constant__ CUtensorMap map_o,
                   __nv_bfloat16 *__restrict__ o,
                   const float *__restrict__ sst, int nseg, int64_t seg_len, int64_t T, int64_t H)
{
    using namespace sm100;
    extern __shared__ __align__(1024) unsigned char corr_smem_raw[];
    unsigned char *smem = corr_smem_raw + ((1024u - (smem_u32(corr_smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kCBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kCMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kCMisc + 4);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t h = blockIdx.y, n = blockIdx.z;
    const int64_t per_seg = (seg_len + kCorrRows * kCorrTiles - 1) / (kCorrRows * kCorrTiles);
    const int p = 1 + (int)(blockIdx.x / per_seg);
    const int64_t tb = p * seg_len + (int64_t)(blockIdx.x % per_seg) * kCorrRows * kCorrTiles;  // first token
    const int64_t seg_end = (p + 1) * seg_len < T ? (p + 1) * seg_len : T;
    if (p >= nseg || tb >= seg_end) return;  // (the same for every thread of the CTA)
    const int64_t left = (seg_end - tb + kCorrRows - 1) / kCorrRows;
    const int ntiles = left < kCorrTiles ? (int)left : kCorrTiles;

    // S_start(p) (fp32 [k][j]) as bf16 hi and lo into the 128B-swizzled MN-major
    // layout: rows k, 64 output channels per 128-byte row, channel halves apart
    {
        const float4 *src = reinterpret_cast<const float4 *>(sst + ((n * nseg + p - 1) * H + h) * kStateElems);
        constexpr int kPer = (int)((kStateElems / 4 + kCorrThreads - 1) / kCorrThreads);
        float4 xin[kPer];
#pragma unroll
        for (int m = 0; m < kPer; ++m) {  // (every load before the first store)
            const int i = tid + kCorrThreads * m;
            if (i < (int)(kStateElems / 4)) xin[m] = src[i];
        }
#pragma unroll
        for (int m = 0; m < kPer; ++m) {
            const int i = tid + kCorrThreads * m;
            if (i >= (int)(kStateElems / 4)) break;
            const int k = i >> 5, j = 4 * (i & 31);
            const float4 x = xin[m];
            const float xs[4] = {x.x, x.y, x.z, x.w};
            uint32_t hi[2], lo[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const __nv_bfloat16 h0 = __float2bfloat16_rn(xs[2 * e]), h1 = __float2bfloat16_rn(xs[2 * e + 1]);
                hi[e] = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
                lo[e] = pack_bf16x2(xs[2 * e] - __bfloat162float(h0), xs[2 * e + 1] - __bfloat162float(h1));
            }
            const uint32_t off = (j >> 6) * 16384 + sw128_offset(k, 2 * (j & 63));
            *reinterpret_cast<uint2 *>(smem + kCB + off) = make_uint2(hi[0], hi[1]);
            *reinterpret_cast<uint2 *>(smem + kCB + 32768 + off) = make_uint2(lo[0], lo[1]);
        }
        fence_proxy_async_smem();  // (read next by the MMAs, through the async proxy)
    }
    if (tid == 0) {
        for (int i = 0; i < C_NUM; ++i) mbar_init(&bars[i], 1);
        mbar_init(&bars[C_FREE0], 2);  // a slot is free once its MMAs and its o readers are done
        mbar_init(&bars[C_FREE1], 2);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&map_psi);
        prefetch_tensormap(&map_o);
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    if (warp == 0) {
        // ---- Psi and o tiles by TMA (two slots) ----
        if (lane == 0) {
            int issued0 = 0, issued1 = 0;
            for (int i = 0; i < ntiles; ++i) {
                const int s = i & 1;
                if (i >= 2 && !cwait(&bars[C_FREE0 + s], ((i >> 1) - 1) & 1, abort_flag, 40)) break;
                const int z = (int)(n * T + tb + (int64_t)kCorrRows * i);
                mbar_arrive_expect_tx(&bars[C_FULL0 + s], 65536);
                for (int half = 0; half < 2; ++half) {
                    tma_load_3d(smem + kCA + s * 32768 + half * 16384, &map_psi, &bars[C_FULL0 + s], 64 * half,
                                (int)h, z);
                    tma_load_3d(smem + kCO + s * 32768 + half * 16384, &map_o, &bars[C_FULL0 + s], 64 * half,
                                (int)h, z);
                }
                (s ? issued1 : issued0) = (i >> 1) + 1;
            }
            // (loads still in flight after an abort land before the CTA exits)
            if (issued0 > 0) { volatile int nf = 0; WaitGuard g{kCorrWaitNs, &nf, &g_seg_error}; mbar_wait(&bars[C_FULL0], (issued0 - 1) & 1, g, 41); }
            if (issued1 > 0) { volatile int nf = 0; WaitGuard g{kCorrWaitNs, &nf, &g_seg_error}; mbar_wait(&bars[C_FULL1], (issued1 - 1) & 1, g, 41); }
        }
    } else if (warp == 1) {
        // ---- MMA issuer: D[a] = Psi S_hi + Psi S_lo ----
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(128, 128, false, true);  // A K-major, B MN-major
            const uint64_t da = smem_desc_sw128(sbase + kCA, 16, 1024);
            const uint64_t db = smem_desc_sw128(sbase + kCB, 16384, 1024);
            for (int i = 0; i < ntiles; ++i) {
                const int s = i & 1;
                if (!cwait(&bars[C_FULL0 + s], (i >> 1) & 1, abort_flag, 42)) break;
                if (i >= 2 && !cwait(&bars[C_ACCFREE0 + s], ((i >> 1) - 1) & 1, abort_flag, 43)) break;
                tc_fence_after();
#pragma unroll
                for (int part = 0; part < 2; ++part)
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        // A: 16 k columns = 32 bytes of a row (k halves 16 KB apart);
                        // B: 16 k rows = 2 KB
                        const uint32_t ka = (kk >> 2) * 16384 + (kk & 3) * 32;
                        mma_ss(tbase + 128 * s, da + ((s * 32768 + ka) >> 4), db + ((part * 32768 + kk * 2048) >> 4),
                               idesc, (part | kk) != 0);
                    }
                tc_commit(&bars[C_FREE0 + s]);
                tc_commit(&bars[C_ACC0 + s]);
            }
            tc_commit(&bars[C_DRAIN]);
            volatile int nf = 0;
            WaitGuard g{kCorrWaitNs, &nf, &g_seg_error};
            mbar_wait(&bars[C_DRAIN], 0, g, 44);
        }
    } else if (warp >= 4) {
        // ---- o rows += D rows (thread = token row = TMEM lane; 64 channels) ----
        const int q4 = warp & 3, half = (warp - 4) >> 2, row = 32 * q4 + lane, te = tid - 128;
        const uint32_t lane_off = (uint32_t)(32 * q4) << 16;
        for (int i = 0; i < ntiles; ++i) {
            const int s = i & 1;
            // (the FULL wait makes the TMA-written o rows visible to these threads)
            if (!group_all(kBarEpiC, 256, cwait(&bars[C_ACC0 + s], (i >> 1) & 1, abort_flag, 45) &&
                                              cwait(&bars[C_FULL0 + s], (i >> 1) & 1, abort_flag, 46)))
                break;
            tc_fence_after();
            const int64_t t = tb + (int64_t)kCorrRows * i + row;
            const bool mine = t < seg_end;
            uint4 *po = reinterpret_cast<uint4 *>(o + ((n * T + t) * H + h) * kD + 64 * half);
            const unsigned char *so = smem + kCO + s * 32768 + half * 16384;
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {
                uint32_t v[32];
                tmem_ld32(tbase + 128 * s + 64 * half + 32 * qq + lane_off, v);
                tc_wait_ld();
                if (mine) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const uint4 x = *reinterpret_cast<const uint4 *>(so + sw128_offset(row, 16 * (4 * qq + e)));
                        uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&w4[c]));
                            w4[c] = pack_bf16x2(f.x + __uint_as_float(v[8 * e + 2 * c]),
                                                f.y + __uint_as_float(v[8 * e + 2 * c + 1]));
                        }
                        po[4 * qq + e] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(kBarEpiC, 256);
            if (te == 0) {
                mbar_arrive(&bars[C_ACCFREE0 + s]);
                mbar_arrive(&bars[C_FREE0 + s]);  // (its o rows have been read)
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) tmem_dealloc(tbase, 256);
}

}  // namespace

typedef CUresult (*EncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                             const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

cudaError_t seg_read_and_clear_error(int *code)
{
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(code, g_seg_error, sizeof(int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_seg_error, &zero, sizeof(int));
}

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
    const int comb_smem = (int)((kStateElems + kCombRows * kD) * 4);
    cudaError_t e = ensure_dynamic_smem((const void *)seg_combine_kernel, comb_smem);
    if (e != cudaSuccess) return e;
    for (int p = 1; p < a.nseg; ++p) {  // (each step reads the previous one's result)
        seg_combine_kernel<<<dim3(kCombCtas, (unsigned)a.H, (unsigned)a.B), 256, comb_smem, stream>>>(
            s0, phi, a.final_state, a.nseg, p, a.H);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // Psi [B*T tokens, H, 128] bf16 as a 3-D map; box = 128 tokens x 1 head x 64 channels
    static std::once_flag once;
    static EncodeFn enc = nullptr;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *fp = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fp, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            enc = reinterpret_cast<EncodeFn>(fp);
    });
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap map_psi;
    const int64_t tokens = a.B * a.T;
    if (tokens > 0x7fffffffLL) return cudaErrorInvalidValue;
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)a.H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)kD * 2, (cuuint64_t)(a.H * kD * 2)};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kCorrRows};
    cuuint32_t es[3] = {1, 1, 1};
    CUtensorMap map_o;  // o, the same shape and box
    if (enc(&map_psi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16 *>(psi), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        enc(&map_o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.o, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    e = ensure_dynamic_smem((const void *)seg_correct_kernel, (int)kCorrSmem);
    if (e != cudaSuccess) return e;
    const int64_t per_seg = (a.seg_len + kCorrRows * kCorrTiles - 1) / (kCorrRows * kCorrTiles);
    const int64_t nblk = per_seg * (a.nseg - 1);  // segments 1..nseg-1
    dim3 grid((unsigned)nblk, (unsigned)a.H, (unsigned)a.B);
    seg_correct_kernel<<<grid, kCorrThreads, kCorrSmem, stream>>>(map_psi, map_o, static_cast<__nv_bfloat16 *>(a.o), s0,
                                                                 a.nseg, a.seg_len, a.T, a.H);
    return cudaGetLastError();
}

}  // namespace gdr2
