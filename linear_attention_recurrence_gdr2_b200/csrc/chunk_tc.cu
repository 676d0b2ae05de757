// Chunkwise forward of Gated Delta Rule-2 for bf16 inputs, d_k = d_v = 128,
// on the sm_100a tensor cores (tcgen05 + TMEM, operands staged by TMA).
//
// Chunk form (C = 64; "Chunkwise training and gate-aware backward" section
// of the ainews.random.gg article on Gated DeltaNet-2). Per chunk with entry
// state S0 and cumulative log-decay g (per key channel, from the chunk
// start), the asymmetric erase factors give, with A = strict_tril(Ebar Kbar^T)
// and T = (I + A)^{-1}:
//     W = T Ebar,  U = T Z - W S0,  O = Qbar S0 + tril(Qbar Kbar^T) U,
//     S_C = Diag(e^{g_C}) S0 + (K . e^{g_C - g})^T U.
// All decay factors are taken about the chunk's middle (after row 31):
// with d_r = g_r - g_31,
//     Qm = q . e^{d}, Km = k . e^{-d}, Em = b . k . e^{d}
// so that every pairwise product carries e^{g_r - g_s} <= 1 and each half of
// the chunk needs only its own partial sums. The state enters as
// Sm = Diag(e^{g_31}) S0, which makes Qm Sm = Qbar S0 and (T Em) Sm = W S0,
// and the state update becomes S_C = Diag(e^{g_C - g_31}) (Sm + Km^T U).
//
// One CTA owns one (sequence, head) and walks its chunks in order. Everything
// is computed transposed so that the value dimension (128) sits on the MMA's
// M axis and on the 128 TMEM lanes (P = tril(Qm Km^T), M = the TMEM state):
//     [A; P]        = [Em; Qm] Km^T                 M=128 N=64  K=128
//     W^T, U0^T     = Em^T T^T, Z^T T^T             M=128 N=64  K=64 (x2)
//     [U^T | O^T]  += Sm^T [-W; Qm]^T               M=128 N=128 K=128, A in TMEM
//     [O^T | M^T]  += U^T [P^T | Km]                M=128 N=192 K=64,  A in TMEM
// Merging the products that share an A operand into one wide-N chain keeps
// the number of tcgen05.mma instructions per chunk at 28 (each costs a fixed
// issue time whatever its N). -W is written K-major over Em (dead by then) so
// that it sits right before Qm; P^T is written MN-major right before Km; the
// O columns sit between U and the state in TMEM.
// The fp32 state lives in TMEM (as M = Diag(e^{g_31}) S plus the chunk's
// update); once per chunk the epilogue scales it by e^{g_C - g_31 + g'_31}
// (g'_31: the next chunk's half sum) and writes its bf16 copy back to TMEM as
// the next chunk's MMA operand.
//
// Warp roles (16 warps; the first warpgroup gives registers to the others):
//   0      TMA producer of q, k, b tiles (double-buffered slots)
//   1      tcgen05.mma issuer of the prep pipeline ([A;P], W^T, U0^T)
//   2      TMEM allocator; TMA producer of v tiles, L2 prefetch of w
//   3      tcgen05.mma issuer of the state chain
//   4..7   prep A: cumulative decay, decay-absorbed factors, Z, P^T
//   8..11  prep B: (I + A)^{-1}, -W
//   12..15 epilogue: U^T to bf16, o stores, state scaling, final state
// The two prep warpgroups work on consecutive chunks concurrently, and both
// run ahead of the state chain. Every wait is bounded: after about a second
// without progress the CTA records the site in the device error word and
// winds down (drains its TMA loads and MMAs, frees TMEM, returns).
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

#include <mutex>

namespace gdr2 {

__device__ int g_chunk_tc_error;

// Optional per-phase SM-clock timestamps for the first CTAs (compiled in only
// with -DGDR2_TRACE; the tracing driver points g_chunk_tc_trace at a buffer
// of [4 CTAs][1024 chunks][32 events] uint64).
#ifdef GDR2_TRACE
__device__ unsigned long long *g_chunk_tc_trace;
#define GDR2_TRACE_AT(chunk, ev)                                                           \
    do {                                                                                   \
        if (blockIdx.x < 4 && g_chunk_tc_trace && (chunk) < 1024)                          \
            g_chunk_tc_trace[((size_t)blockIdx.x * 1024 + (chunk)) * 32 + (ev)] = clock64(); \
    } while (0)
#else
#define GDR2_TRACE_AT(chunk, ev) do { } while (0)
#endif

namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kThreadsTC = 512;
constexpr uint64_t kWaitNs = 1000000000ull;  // one second per wait

// ---- shared memory map (bytes from the 1024-aligned base) ----------------
constexpr uint32_t kEQ0 = 0;             // per 64-channel block kb: [Em -> -W 8K | Qm 8K]
constexpr uint32_t kEQ1 = 32768;
constexpr uint32_t kKB0 = 65536;         // [P^T 8K | Km kb0 8K | Km kb1 8K]
constexpr uint32_t kKB1 = 90112;
constexpr uint32_t kKmOff = 8192;        // Km after the P^T block
constexpr uint32_t kZB0 = 114688;        // v -> Z: [dv block 0 8K][dv block 1 8K]
constexpr uint32_t kZB1 = 131072;
constexpr uint32_t kTB = 147456;         // T bf16, 64 rows x 128 B
constexpr uint32_t kLA = 155648;         // staged log_alpha, fp32 [64][128]
constexpr int kLD = 68;                  // fp32 scratch row pitch (16-byte aligned rows)
constexpr uint32_t kSA = 188416;         // fp32 A^T, 64 x kLD
constexpr uint32_t kST = kSA + 64 * kLD * 4;  // fp32 T, 64 x kLD
constexpr uint32_t kVEC = kST + 64 * kLD * 4; // half sums: T0[4][128], T1[4][128], f[128]
constexpr uint32_t kBSUM = kVEC + (8 * 128 + 128) * 4;  // per-row-block log-decay sums [4][128]
constexpr uint32_t kBAR = kBSUM + 4 * 128 * 4;
constexpr int kNumBars = 28;
constexpr uint32_t kMISC = kBAR + kNumBars * 8;
constexpr uint32_t kSmemBytes = kMISC + 64 + 1024;  // + alignment slack

// barrier indices
enum {
    B_FULL0 = 0, B_FULL1, B_SLOTFREE0, B_SLOTFREE1, B_VFULL0, B_VFULL1, B_VFREE0, B_VFREE1,
    B_LAFULL, B_PREP, B_VEC0, B_VEC1, B_AP, B_AFREE, B_ZREADY0, B_ZREADY1, B_T, B_WDONE, B_WREADY0,
    B_WREADY1, B_PREADY0, B_PREADY1, B_SREADY, B_UDONE, B_UCONV, B_SDONE, B_DRAIN, B_DRAIN2
};

// ---- TMEM column map (512 columns allocated) -------------------------------
constexpr uint32_t kTmU = 0;         // U^T fp32, 64      } one N=128 accumulator
constexpr uint32_t kTmO = 64;        // O^T fp32, 64      }        } one N=192
constexpr uint32_t kTmMaster = 128;  // state (transposed) fp32, 128 } accumulator
constexpr uint32_t kTmX = 256;       // 128 columns shared by two M=64 accumulators:
                                     //   lanes 0-15 of each quarter: [A^T | P^T] (rows s)
                                     //   lanes 16-31 of each quarter: W (rows r)
constexpr uint32_t kTmSB = 384;      // Sm^T bf16 pairs, 64 words
constexpr uint32_t kTmUB = 448;      // U^T bf16 pairs, 32 words

// group (named) barriers
constexpr uint32_t kBarPrepA = 1, kBarEpi = 2, kBarPrepB = 3;

struct TcParams {
    const float *la;
    const __nv_bfloat16 *w;
    const float *init_state;
    const int32_t *cu_seqlens;
    const int32_t *order;
    __nv_bfloat16 *o;
    float *final_state;
    int64_t T, H;
};

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         int site) {
    WaitGuard g{globaltimer_ns() + kWaitNs, abort_flag, &g_chunk_tc_error};
    return mbar_wait(bar, parity, g, site);
}

// Barrier over a 128-thread group that also ANDs one predicate across it, so
// every thread of the group takes the same continue / abort decision.
__device__ __forceinline__ bool group_and(uint32_t id, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, 128, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r) : "r"((uint32_t)v), "r"(id) : "memory");
    return r != 0;
}

// Bounded spin on a barrier phase without suspending (for the MMA issuers,
// whose reaction time is on the chunk-to-chunk path).
__device__ __forceinline__ bool spin_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         int site) {
    uint64_t deadline = 0;
    for (uint32_t it = 0;; ++it) {
        if (mbar_test(bar, parity)) return true;
        if ((it & 1023u) == 1023u) {
            if (*abort_flag) return false;
            const uint64_t now = globaltimer_ns();
            if (deadline == 0) deadline = now + kWaitNs;
            else if (now > deadline) {
                *abort_flag = 1;
                atomicCAS(&g_chunk_tc_error, 0, 0x100 | site);
                return false;
            }
        }
    }
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
// Warp-level D (16x8, fp32) += A (16x8, tf32) * B (8x8, tf32).
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}
// One 16x8 output tile of C = X * Y over K (multiple of 8) on the tensor
// cores in tf32 with fp32 accumulation; X(i, k) and Y(k, j) are fp32 values in
// shared memory addressed as x[i * xsi + k * xsk] and y[k * ysk + j].
template <int K>
__device__ __forceinline__ void tile_tf32(float (&d)[4], const float *x, int xsi, int xsk,
                                          const float *y, int ysk, int lane) {
    const int ar = lane >> 2, ac = lane & 3;
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 8) {
        uint32_t a[4], b[2];
        a[0] = to_tf32(x[ar * xsi + (k0 + ac) * xsk]);
        a[1] = to_tf32(x[(ar + 8) * xsi + (k0 + ac) * xsk]);
        a[2] = to_tf32(x[ar * xsi + (k0 + ac + 4) * xsk]);
        a[3] = to_tf32(x[(ar + 8) * xsi + (k0 + ac + 4) * xsk]);
        b[0] = to_tf32(y[(k0 + ac) * ysk + ar]);
        b[1] = to_tf32(y[(k0 + ac + 4) * ysk + ar]);
        mma_tf32_16x8x8(d, a, b);
    }
}
// Stores a 16x8 fp32 tile (times `scale`) at out[i * osi + j].
__device__ __forceinline__ void store_tile(const float (&d)[4], float *out, int osi, int lane,
                                           float scale) {
    const int r = lane >> 2, c2 = 2 * (lane & 3);
    *reinterpret_cast<float2 *>(out + r * osi + c2) = make_float2(scale * d[0], scale * d[1]);
    *reinterpret_cast<float2 *>(out + (r + 8) * osi + c2) = make_float2(scale * d[2], scale * d[3]);
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float2 bf2_to_f2(uint32_t v) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&v));
}

// Writes 64 fp32 values as one 128-byte bf16 row of a 128B-swizzled tile.
__device__ __forceinline__ void store_row_bf16_sw128(unsigned char *tile, uint32_t row, const float *x) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        uint4 u;
        u.x = pack_bf16x2(x[8 * q + 0], x[8 * q + 1]);
        u.y = pack_bf16x2(x[8 * q + 2], x[8 * q + 3]);
        u.z = pack_bf16x2(x[8 * q + 4], x[8 * q + 5]);
        u.w = pack_bf16x2(x[8 * q + 6], x[8 * q + 7]);
        *reinterpret_cast<uint4 *>(tile + sw128_offset(row, 16 * q)) = u;
    }
}

__device__ __forceinline__ void setmaxnreg_dec40() { asm volatile("setmaxnreg.dec.sync.aligned.u32 40;" ::: "memory"); }
__device__ __forceinline__ void setmaxnreg_inc152() { asm volatile("setmaxnreg.inc.sync.aligned.u32 152;" ::: "memory"); }

__global__ void __launch_bounds__(kThreadsTC, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_v,
                const __grid_constant__ CUtensorMap map_la, const __grid_constant__ CUtensorMap map_w,
                TcParams prm)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // Align to 1024 B by offsetting the __shared__ array itself (not through an
    // integer round trip), so every access below stays a shared-space access.
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kMISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kMISC + 4);
    float *sA = reinterpret_cast<float *>(smem + kSA);
    float *sT = reinterpret_cast<float *>(smem + kST);
    float *vecT0 = reinterpret_cast<float *>(smem + kVEC);         // [4][128]
    float *vecT1 = vecT0 + 4 * 128;                                 // [4][128]
    float *vecF = vecT1 + 4 * 128;                                  // [128]
    float *vecBS = reinterpret_cast<float *>(smem + kBSUM);         // [4][128]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = prm.H;
    const int64_t h = blockIdx.x % H;
    const int64_t n = prm.order ? (int64_t)prm.order[blockIdx.x / H] : (int64_t)(blockIdx.x / H);
    int64_t t_begin, t_end;
    if (prm.cu_seqlens) {
        t_begin = prm.cu_seqlens[n];
        t_end = prm.cu_seqlens[n + 1];
    } else {
        t_begin = n * prm.T;
        t_end = t_begin + prm.T;
    }
    const int nc = (int)((t_end - t_begin + 63) / 64);
    const int64_t state_base = (n * H + h) * (int64_t)kD * kD;

    if (nc == 0) {  // empty sequence: the final state is the initial state
        if (prm.final_state)
            for (int i = tid; i < kD * kD; i += kThreadsTC)
                prm.final_state[state_base + i] = prm.init_state ? prm.init_state[state_base + i] : 0.f;
        return;
    }

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(&bars[i], 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&map_q); prefetch_tensormap(&map_k); prefetch_tensormap(&map_b);
    }
    if (warp == 2) {
        if (lane == 0) {
            prefetch_tensormap(&map_v); prefetch_tensormap(&map_la); prefetch_tensormap(&map_w);
        }
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tmem_slot;

    // =====================================================================
    if (warp < 4) {
    setmaxnreg_dec40();
    if (warp == 0) {
        // ---------------- producer: q, k, b tiles ----------------------------
        if (lane == 0) {
            int issued[2] = {0, 0};
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1;
                if (c >= 2 && !wait_bar(&bars[B_SLOTFREE0 + s], ((c >> 1) - 1) & 1, abort_flag, 1)) break;
                const int z = (int)(t_begin + 64 * c);
                unsigned char *eq = smem + (s ? kEQ1 : kEQ0), *kq = smem + (s ? kKB1 : kKB0) + kKmOff;
                GDR2_TRACE_AT(c, 0);
                mbar_arrive_expect_tx(&bars[B_FULL0 + s], 3 * 16384);
                for (int blk = 0; blk < 2; ++blk) {
                    tma_load_3d(eq + blk * 16384, &map_b, &bars[B_FULL0 + s], 64 * blk, (int)h, z);
                    tma_load_3d(eq + blk * 16384 + 8192, &map_q, &bars[B_FULL0 + s], 64 * blk, (int)h, z);
                    tma_load_3d(kq + blk * 8192, &map_k, &bars[B_FULL0 + s], 64 * blk, (int)h, z);
                }
                issued[s] = (c >> 1) + 1;
            }
            // drain: wait (bounded) for every load issued into each slot
            for (int s = 0; s < 2; ++s)
                if (issued[s] > 0) {
                    volatile int dummy = 0;
                    WaitGuard g2{globaltimer_ns() + kWaitNs, &dummy, &g_chunk_tc_error};
                    mbar_wait(&bars[B_FULL0 + s], (issued[s] - 1) & 1, g2, 20);
                }
        }
    } else if (warp == 2) {
        // ---------------- producer: v tiles, L2 prefetch of w ------------------
        if (lane == 0) {
            tma_prefetch_3d(&map_w, 0, (int)h, (int)t_begin);
            int vissued[2] = {0, 0};
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1;
                if (c >= 2 && !wait_bar(&bars[B_VFREE0 + s], ((c >> 1) - 1) & 1, abort_flag, 2)) break;
                const int z = (int)(t_begin + 64 * c);
                GDR2_TRACE_AT(c, 1);
                mbar_arrive_expect_tx(&bars[B_VFULL0 + s], 16384);
                for (int blk = 0; blk < 2; ++blk)
                    tma_load_3d(smem + (s ? kZB1 : kZB0) + blk * 8192, &map_v, &bars[B_VFULL0 + s], 64 * blk,
                                (int)h, z);
                vissued[s] = (c >> 1) + 1;
                if (c + 1 < nc) tma_prefetch_3d(&map_w, 0, (int)h, z + 64);
            }
            for (int s = 0; s < 2; ++s)
                if (vissued[s] > 0) {
                    volatile int dummy = 0;
                    WaitGuard g2{globaltimer_ns() + kWaitNs, &dummy, &g_chunk_tc_error};
                    mbar_wait(&bars[B_VFULL0 + s], (vissued[s] - 1) & 1, g2, 21);
                }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer for the prep pipeline --------------------
        if (lane == 0) {
            const uint32_t i_ap = idesc_bf16_f32(64, 128, false, false);
            const uint32_t i_w = idesc_bf16_f32(64, 128, false, true);
            const uint32_t i_u = idesc_bf16_f32(128, 64, true, false);
            for (int cp = 0; cp < nc; ++cp) {
                const int s = cp & 1;
                const uint32_t eq = sbase + (s ? kEQ1 : kEQ0);
                const uint32_t km = sbase + (s ? kKB1 : kKB0) + kKmOff;
                if (!wait_bar(&bars[B_PREP], cp & 1, abort_flag, 12)) break;
                if (cp >= 1 && !wait_bar(&bars[B_AFREE], (cp - 1) & 1, abort_flag, 13)) break;
                tc_fence_after();
                // [A^T | P^T] = Km [Em; Qm]^T   (M = 64 rows s, N = 128, lanes 0-15)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t a = smem_desc_sw128(km + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
                    const uint64_t b = smem_desc_sw128(eq + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    mma_ss(tb + kTmX, a, b, i_ap, kk > 0);
                }
                tc_commit(&bars[B_AP]);
                GDR2_TRACE_AT(cp, 2);
                if (!wait_bar(&bars[B_T], cp & 1, abort_flag, 14)) break;
                // P^T read out of the shared columns (implies Z is ready): the W
                // accumulator below shares those TMEM columns (other lanes)
                if (!wait_bar(&bars[B_PREADY0 + s], (cp >> 1) & 1, abort_flag, 15)) break;
                // the single U region is free once the epilogue has read chunk cp-1's U
                if (cp >= 1 && !wait_bar(&bars[B_UCONV], (cp - 1) & 1, abort_flag, 16)) break;
                tc_fence_after();
                // W = T Em (M = 64 rows r, N = 128, lanes 16-31); U0^T = Z^T T^T (M = 128)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t at = smem_desc_sw128(sbase + kTB + kk * 32, 16, 1024);
                    const uint64_t be = smem_desc_sw128(eq + kk * 2048, 16384, 1024);
                    mma_ss(tb + kTmX + (16u << 16), at, be, i_w, kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bt = smem_desc_sw128(sbase + kTB + kk * 32, 16, 1024);
                    const uint64_t az = smem_desc_sw128(sbase + (s ? kZB1 : kZB0) + kk * 2048, 8192, 1024);
                    mma_ss(tb + kTmU, az, bt, i_u, kk > 0);
                }
                tc_commit(&bars[B_WDONE]);
                GDR2_TRACE_AT(cp, 3);
                tc_commit(&bars[B_VFREE0 + s]);
            }
            // drain every MMA this thread issued before TMEM is released
            tc_commit(&bars[B_DRAIN]);
            volatile int dummy = 0;
            WaitGuard g2{globaltimer_ns() + kWaitNs, &dummy, &g_chunk_tc_error};
            mbar_wait(&bars[B_DRAIN], 0, g2, 22);
        }
    } else if (warp == 3) {
        // ---------------- MMA issuer for the state chain -----------------------
        if (lane == 0) {
            const uint32_t i_uo = idesc_bf16_f32(128, 128, false, false);
            const uint32_t i_os = idesc_bf16_f32(128, 192, false, true);
            for (int cc = 0; cc < nc; ++cc) {
                const int s = cc & 1;
                const uint32_t eq = sbase + (s ? kEQ1 : kEQ0);
                const uint32_t kbs = sbase + (s ? kKB1 : kKB0);
                if (!wait_bar(&bars[B_WREADY0 + s], (cc >> 1) & 1, abort_flag, 17)) break;
                if (!wait_bar(&bars[B_SREADY], cc & 1, abort_flag, 18)) break;
                GDR2_TRACE_AT(cc, 7);
                tc_fence_after();
                // [U^T | O^T] += Sm^T [-W ; Qm]^T   (N = 128: -W rows then Qm rows)
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t b = smem_desc_sw128(eq + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    mma_ts(tb + kTmU, tb + kTmSB + kk * 8, b, i_uo, 1);
                }
                tc_commit(&bars[B_UDONE]);
                GDR2_TRACE_AT(cc, 4);
                if (!wait_bar(&bars[B_UCONV], cc & 1, abort_flag, 19)) break;
                if (!wait_bar(&bars[B_PREADY0 + s], (cc >> 1) & 1, abort_flag, 25)) break;
                GDR2_TRACE_AT(cc, 6);
                tc_fence_after();
                // [O^T | M^T] += U^T [P^T | Km]   (N = 192, B MN-major: P^T atom, two Km atoms)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t b = smem_desc_sw128(kbs + kk * 2048, 8192, 1024);
                    mma_ts(tb + kTmO, tb + kTmUB + kk * 8, b, i_os, 1);
                }
                tc_commit(&bars[B_SDONE]);
                GDR2_TRACE_AT(cc, 5);
                tc_commit(&bars[B_SLOTFREE0 + s]);
            }
            tc_commit(&bars[B_DRAIN2]);
            volatile int dummy = 0;
            WaitGuard g2{globaltimer_ns() + kWaitNs, &dummy, &g_chunk_tc_error};
            mbar_wait(&bars[B_DRAIN2], 0, g2, 23);
        }
    }
    } else if (warp < 8) {
        setmaxnreg_inc152();
        // ---------------- prep A: decay factors, Z, P^T ------------------------
        // Element-wise layout: lane g owns key channels 4g..4g+3 (64-channel
        // block kb = g / 16), warp rb owns rows 16rb..16rb+15. Loads are
        // unconditional (rows clamped to the valid range) and rows past the
        // chunk end are zeroed with selects, so many loads stay in flight.
        const int pw = warp - 4, tp = tid - 128;
        const int g = lane, rb = pw, kb = g >> 4;
        const uint32_t cbyte = 8 * (g & 15);
        constexpr float kLog2e = 1.4426950408889634f;
        const float *la_s = reinterpret_cast<const float *>(smem + kLA);  // staged log_alpha [64][128]
        int la_issued = 0;  // log_alpha tiles staged so far (thread tp == 0)
        if (tp == 0) {
            ++la_issued;
            mbar_arrive_expect_tx(&bars[B_LAFULL], 32768);
            tma_load_3d(smem + kLA, &map_la, &bars[B_LAFULL], 0, (int)h, (int)t_begin);
        }
        for (int c = 0; c < nc; ++c) {
            const int s = c & 1;
            const int64_t t0 = t_begin + 64 * c;
            const int L = (int)(t_end - t0 < 64 ? t_end - t0 : 64);
            unsigned char *e_tile = smem + (s ? kEQ1 : kEQ0) + kb * 16384;
            unsigned char *q_tile = e_tile + 8192;
            unsigned char *k_tile = smem + (s ? kKB1 : kKB0) + kKmOff + kb * 8192;

            if (tp == 0) GDR2_TRACE_AT(c, 8);
            // write-gate rows of this chunk, consumed in the Z step (L2-prefetched)
            uint2 wv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = 16 * rb + i;
                const int rr = r < L ? r : L - 1;
                wv[i] = *reinterpret_cast<const uint2 *>(prm.w + ((t0 + rr) * H + h) * kD + 4 * g);
            }
            if (!group_and(kBarPrepA, wait_bar(&bars[B_LAFULL], c & 1, abort_flag, 3))) break;
            float4 la[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = 16 * rb + i;
                const float4 x = *reinterpret_cast<const float4 *>(la_s + r * 128 + 4 * g);
                la[i] = r < L ? x : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            float4 bs = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                bs.x += la[i].x; bs.y += la[i].y; bs.z += la[i].z; bs.w += la[i].w;
            }
            *reinterpret_cast<float4 *>(vecBS + rb * 128 + 4 * g) = bs;
            if (tp == 0) GDR2_TRACE_AT(c, 9);
            // (this group barrier also publishes the block sums and frees the staging tile)
            fence_proxy_async_smem();
            if (!group_and(kBarPrepA, wait_bar(&bars[B_FULL0 + s], (c >> 1) & 1, abort_flag, 4))) break;
            if (tp == 0) {
                GDR2_TRACE_AT(c, 10);
                if (c + 1 < nc) {  // stage the next chunk's log_alpha
                    ++la_issued;
                    mbar_arrive_expect_tx(&bars[B_LAFULL], 32768);
                    tma_load_3d(smem + kLA, &map_la, &bars[B_LAFULL], 0, (int)h, (int)(t0 + 64));
                }
            }
            // d_r = g_r - g_31 in log2 units: suffix sums for rows < 32, prefix
            // sums for rows >= 32; half sums T0 = g_31, T1 = g_63 - g_31.
            {
                float4 run = make_float4(0.f, 0.f, 0.f, 0.f);
                if (rb == 0) run = *reinterpret_cast<const float4 *>(vecBS + 1 * 128 + 4 * g);
                if (rb == 3) run = *reinterpret_cast<const float4 *>(vecBS + 2 * 128 + 4 * g);
                if (rb == 1 || rb == 2) {
                    const float4 o4 = *reinterpret_cast<const float4 *>(vecBS + (rb == 1 ? 0 : 3) * 128 + 4 * g);
                    float *vt = (rb == 1 ? vecT0 : vecT1) + (c & 3) * 128 + 4 * g;
                    *reinterpret_cast<float4 *>(vt) =
                        make_float4(bs.x + o4.x, bs.y + o4.y, bs.z + o4.z, bs.w + o4.w);
                }
                if (rb < 2) {
#pragma unroll
                    for (int i = 15; i >= 0; --i) {
                        const float4 x = la[i];
                        la[i] = make_float4(-run.x * kLog2e, -run.y * kLog2e, -run.z * kLog2e, -run.w * kLog2e);
                        run.x += x.x; run.y += x.y; run.z += x.z; run.w += x.w;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        run.x += la[i].x; run.y += la[i].y; run.z += la[i].z; run.w += la[i].w;
                        la[i] = make_float4(run.x * kLog2e, run.y * kLog2e, run.z * kLog2e, run.w * kLog2e);
                    }
                }
            }
            // factors, in place: b -> Em, q -> Qm, k -> Km
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = 16 * rb + i;
                const uint32_t off = sw128_offset(r, cbyte);
                const uint2 qr = *reinterpret_cast<const uint2 *>(q_tile + off);
                const uint2 kr = *reinterpret_cast<const uint2 *>(k_tile + off);
                const uint2 br = *reinterpret_cast<const uint2 *>(e_tile + off);
                const float2 q0 = bf2_to_f2(qr.x), q1 = bf2_to_f2(qr.y);
                const float2 k0 = bf2_to_f2(kr.x), k1 = bf2_to_f2(kr.y);
                const float2 b0 = bf2_to_f2(br.x), b1 = bf2_to_f2(br.y);
                const float u0 = ex2_approx(la[i].x), u1 = ex2_approx(la[i].y);
                const float u2 = ex2_approx(la[i].z), u3 = ex2_approx(la[i].w);
                const float v0 = ex2_approx(-la[i].x), v1 = ex2_approx(-la[i].y);
                const float v2 = ex2_approx(-la[i].z), v3 = ex2_approx(-la[i].w);
                const bool ok = r < L;
                uint2 oq, okk, oe;
                oq.x = ok ? pack_bf16x2(q0.x * u0, q0.y * u1) : 0u;
                oq.y = ok ? pack_bf16x2(q1.x * u2, q1.y * u3) : 0u;
                okk.x = ok ? pack_bf16x2(k0.x * v0, k0.y * v1) : 0u;
                okk.y = ok ? pack_bf16x2(k1.x * v2, k1.y * v3) : 0u;
                oe.x = ok ? pack_bf16x2(b0.x * k0.x * u0, b0.y * k0.y * u1) : 0u;
                oe.y = ok ? pack_bf16x2(b1.x * k1.x * u2, b1.y * k1.y * u3) : 0u;
                *reinterpret_cast<uint2 *>(q_tile + off) = oq;
                *reinterpret_cast<uint2 *>(k_tile + off) = okk;
                *reinterpret_cast<uint2 *>(e_tile + off) = oe;
            }
            fence_proxy_async_smem();
            named_bar_sync(kBarPrepA, 128);
            if (tp == 0) {
                GDR2_TRACE_AT(c, 11);
                mbar_arrive(&bars[B_PREP]);
                mbar_arrive(&bars[B_VEC0 + s]);
            }

            // Z = w . v in place (v tile from TMA, w loaded at the chunk start)
            {
                if (!group_and(kBarPrepA, wait_bar(&bars[B_VFULL0 + s], (c >> 1) & 1, abort_flag, 5))) break;
                unsigned char *z_tile = smem + (s ? kZB1 : kZB0) + kb * 8192;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int r = 16 * rb + i;
                    const uint32_t off = sw128_offset(r, cbyte);
                    const uint2 vr = *reinterpret_cast<const uint2 *>(z_tile + off);
                    const float2 v0 = bf2_to_f2(vr.x), v1 = bf2_to_f2(vr.y);
                    const float2 w0 = bf2_to_f2(wv[i].x), w1 = bf2_to_f2(wv[i].y);
                    const bool ok = r < L;
                    uint2 oz;
                    oz.x = ok ? pack_bf16x2(v0.x * w0.x, v0.y * w0.y) : 0u;
                    oz.y = ok ? pack_bf16x2(v1.x * w1.x, v1.y * w1.y) : 0u;
                    *reinterpret_cast<uint2 *>(z_tile + off) = oz;
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(kBarPrepA, 128);
            if (tp == 0) {
                GDR2_TRACE_AT(c, 12);
                mbar_arrive(&bars[B_ZREADY0 + s]);
            }

            // P^T[s][r] = P[r][s] (kept for s <= r) from the M=64 accumulator: lane
            // i < 16 of warp pw holds row s = 16 pw + i -> MN-major rows before Km
            if (!group_and(kBarPrepA, wait_bar(&bars[B_AP], c & 1, abort_flag, 6))) break;
            if (tp == 0) GDR2_TRACE_AT(c, 13);
            tc_fence_after();
            {
                const uint32_t taddr = tb + kTmX + 64 + ((uint32_t)(32 * pw) << 16);
                uint32_t v0[32], v1[32];
                tmem_ld32(taddr, v0);
                tmem_ld32(taddr + 32, v1);
                tc_wait_ld();
                if (lane < 16) {
                    const int srow = 16 * pw + lane;
                    float x[64];
#pragma unroll
                    for (int j2 = 0; j2 < 32; ++j2) {
                        x[j2] = j2 >= srow ? __uint_as_float(v0[j2]) : 0.f;
                        x[32 + j2] = 32 + j2 >= srow ? __uint_as_float(v1[j2]) : 0.f;
                    }
                    store_row_bf16_sw128(smem + (s ? kKB1 : kKB0), srow, x);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(kBarPrepA, 128);
            if (tp == 0) {
                GDR2_TRACE_AT(c, 14);
                mbar_arrive(&bars[B_PREADY0 + s]);
            }
        }
        if (tp == 0 && la_issued > 0) {  // drain a staged log_alpha load still in flight
            volatile int dummy = 0;
            WaitGuard g2{globaltimer_ns() + kWaitNs, &dummy, &g_chunk_tc_error};
            mbar_wait(&bars[B_LAFULL], (la_issued - 1) & 1, g2, 24);
        }
    } else if (warp < 12) {
        setmaxnreg_inc152();
        // ---------------- prep B: (I + A)^{-1}, -W ------------------------------
        const int pw = warp - 8, tp = tid - 256;
        for (int c = 0; c < nc; ++c) {
            const int s = c & 1;
            if (!group_and(kBarPrepB, wait_bar(&bars[B_AP], c & 1, abort_flag, 7))) break;
            if (tp == 0) GDR2_TRACE_AT(c, 15);
            tc_fence_after();
            {   // A^T rows from the M=64 accumulator (lane i < 16 of warp pw: row s = 16 pw + i):
                // A^T[s][r] = A[r][s], kept for r > s
                const uint32_t taddr = tb + kTmX + ((uint32_t)(32 * pw) << 16);
                uint32_t v0[32], v1[32];
                tmem_ld32(taddr, v0);
                tmem_ld32(taddr + 32, v1);
                tc_wait_ld();
                if (lane < 16) {
                    const int srow = 16 * pw + lane;
                    float *row = sA + srow * kLD;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float4 a0, a1;
                        a0.x = 4 * q + 0 > srow ? __uint_as_float(v0[4 * q + 0]) : 0.f;
                        a0.y = 4 * q + 1 > srow ? __uint_as_float(v0[4 * q + 1]) : 0.f;
                        a0.z = 4 * q + 2 > srow ? __uint_as_float(v0[4 * q + 2]) : 0.f;
                        a0.w = 4 * q + 3 > srow ? __uint_as_float(v0[4 * q + 3]) : 0.f;
                        a1.x = 32 + 4 * q + 0 > srow ? __uint_as_float(v1[4 * q + 0]) : 0.f;
                        a1.y = 32 + 4 * q + 1 > srow ? __uint_as_float(v1[4 * q + 1]) : 0.f;
                        a1.z = 32 + 4 * q + 2 > srow ? __uint_as_float(v1[4 * q + 2]) : 0.f;
                        a1.w = 32 + 4 * q + 3 > srow ? __uint_as_float(v1[4 * q + 3]) : 0.f;
                        *reinterpret_cast<float4 *>(row + 4 * q) = a0;
                        *reinterpret_cast<float4 *>(row + 32 + 4 * q) = a1;
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(kBarPrepB, 128);
            if (tp == 0) {
                GDR2_TRACE_AT(c, 25);
                // lanes 0-15 of the shared columns may now take the next [A^T | P^T]
                // (prep A has read its P^T: that precedes PREP of the next chunk).
                // The W readout below still loads all 32 lanes of each quarter,
                // but it only uses lanes 16-31, which that MMA does not write.
                mbar_arrive(&bars[B_AFREE]);
            }

            // T = (I + A)^{-1} by doubling on 16-row blocks (A held transposed,
            // sA = A^T; T in sT, both fp32 with row pitch kLD):
            //   1. T_ii = (I + A_ii)^{-1} for the four 16x16 diagonal blocks,
            //      right-looking forward substitution, one column per thread;
            //   2. inside each 32-block: T_10 = -T_11 (A_10 T_00);
            //   3. across the two 32-blocks: T_10 = -T_11 (A_10 T_00).
            // Steps 2 and 3 are small dense products run as warp-level tensor-core
            // MMAs in tf32 with fp32 accumulation (T itself is consumed in bf16),
            // their intermediate Y parked in the upper-right (zero) part of T,
            // which the bf16 writer masks out.
            if (tp < 64) {
                const int blk = tp >> 4, jj = tp & 15, base = 16 * blk;
                float x[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) x[i] = (i == jj) ? 1.f : 0.f;
#pragma unroll
                for (int i = 0; i < 15; ++i) {
                    const float xi = x[i];
                    const float *at = sA + (base + i) * kLD + base;
                    float a16[16];
#pragma unroll
                    for (int q4 = (i + 1) >> 2; q4 < 4; ++q4) {
                        const float4 v = *reinterpret_cast<const float4 *>(at + 4 * q4);
                        a16[4 * q4] = v.x; a16[4 * q4 + 1] = v.y; a16[4 * q4 + 2] = v.z; a16[4 * q4 + 3] = v.w;
                    }
#pragma unroll
                    for (int k2 = i + 1; k2 < 16; ++k2) x[k2] = fmaf(-a16[k2], xi, x[k2]);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) sT[(base + i) * kLD + base + jj] = x[i];
                if ((blk & 1) == 0) {  // the upper-right 16x16 of each 32-block is zero
#pragma unroll
                    for (int i = 0; i < 16; ++i) sT[(base + i) * kLD + base + 16 + jj] = 0.f;
                }
            }
            named_bar_sync(kBarPrepB, 128);
            if (tp == 0) GDR2_TRACE_AT(c, 26);
            {   // step 2a: Y = A_10 T_00 inside 32-block pb (warp: pb = pw >> 1, n-tile pw & 1)
                const int pb = pw >> 1, nt = pw & 1, b0 = 32 * pb;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                tile_tf32<16>(d, sA + b0 * kLD + b0 + 16, 1, kLD, sT + b0 * kLD + b0 + 8 * nt, kLD, lane);
                store_tile(d, sT + (16 * pb) * kLD + 32 + 16 * pb + 8 * nt, kLD, lane, 1.f);
            }
            named_bar_sync(kBarPrepB, 128);
            {   // step 2b: T_10 = -T_11 Y inside 32-block pb
                const int pb = pw >> 1, nt = pw & 1, b0 = 32 * pb;
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                tile_tf32<16>(d, sT + (b0 + 16) * kLD + b0 + 16, kLD, 1,
                              sT + (16 * pb) * kLD + 32 + 16 * pb + 8 * nt, kLD, lane);
                store_tile(d, sT + (b0 + 16) * kLD + b0 + 8 * nt, kLD, lane, -1.f);
            }
            named_bar_sync(kBarPrepB, 128);
            {   // step 3a: Y = A_10 T_00 across the 32-blocks -> upper-right 32x32 of sT
                const int mt = pw >> 1;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int nt = 2 * (pw & 1) + q;
                    float d[4] = {0.f, 0.f, 0.f, 0.f};
                    tile_tf32<32>(d, sA + 32 + 16 * mt, 1, kLD, sT + 8 * nt, kLD, lane);
                    store_tile(d, sT + (16 * mt) * kLD + 32 + 8 * nt, kLD, lane, 1.f);
                }
            }
            named_bar_sync(kBarPrepB, 128);
            {   // step 3b: T_10 = -T_11 Y
                const int mt = pw >> 1;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    const int nt = 2 * (pw & 1) + q;
                    float d[4] = {0.f, 0.f, 0.f, 0.f};
                    tile_tf32<32>(d, sT + (32 + 16 * mt) * kLD + 32, kLD, 1, sT + 32 + 8 * nt, kLD, lane);
                    store_tile(d, sT + (32 + 16 * mt) * kLD + 8 * nt, kLD, lane, -1.f);
                }
            }
            named_bar_sync(kBarPrepB, 128);
            if (tp == 0) GDR2_TRACE_AT(c, 27);
            {   // T (lower triangle incl. diagonal) -> bf16 MMA operand
                const int r = tp >> 1, half = tp & 1;
                const float *trow = sT + r * kLD + 32 * half;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t ue[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s0 = 32 * half + 8 * q + 2 * e;
                        ue[e] = pack_bf16x2(s0 <= r ? trow[8 * q + 2 * e] : 0.f,
                                            s0 + 1 <= r ? trow[8 * q + 2 * e + 1] : 0.f);
                    }
                    *reinterpret_cast<uint4 *>(smem + kTB + sw128_offset(r, 64 * half + 16 * q)) =
                        make_uint4(ue[0], ue[1], ue[2], ue[3]);
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(kBarPrepB, 128);
            if (tp == 0) {
                GDR2_TRACE_AT(c, 16);
                mbar_arrive(&bars[B_T]);
            }

            // W^T (lanes = key channels) -> -W, K-major, into the Em half of the slot
            if (!group_and(kBarPrepB, wait_bar(&bars[B_WDONE], c & 1, abort_flag, 8))) break;
            if (tp == 0) GDR2_TRACE_AT(c, 17);
            tc_fence_after();
            {   // W rows from the M=64 accumulator (lane 16 + i of warp pw: row r = 16 pw + i)
                // -> -W, K-major, over the Em half of the slot (two 64-channel blocks)
                const uint32_t taddr = tb + kTmX + ((uint32_t)(32 * pw) << 16);
                const int rrow = 16 * pw + (lane & 15);
#pragma unroll 1
                for (int hb = 0; hb < 2; ++hb) {
                    uint32_t v0[32], v1[32];
                    tmem_ld32(taddr + 64 * hb, v0);
                    tmem_ld32(taddr + 64 * hb + 32, v1);
                    tc_wait_ld();
                    if (lane >= 16) {
                        float x[64];
#pragma unroll
                        for (int j2 = 0; j2 < 32; ++j2) {
                            x[j2] = -__uint_as_float(v0[j2]);
                            x[32 + j2] = -__uint_as_float(v1[j2]);
                        }
                        store_row_bf16_sw128(smem + (s ? kEQ1 : kEQ0) + hb * 16384, rrow, x);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(kBarPrepB, 128);
            if (tp == 0) {
                GDR2_TRACE_AT(c, 18);
                mbar_arrive(&bars[B_WREADY0 + s]);
            }
        }
    } else {
        setmaxnreg_inc152();
        // ---------------- epilogue warpgroup -----------------------------------
        const int ew = warp - 12, te = tid - 384;
        const int j = 32 * ew + lane;                       // value channel = TMEM lane
        const uint32_t lane_off = (uint32_t)(32 * ew) << 16;
        const uint32_t zeros[32] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u,
                                    0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        bool ok = true;
        // master = Diag(e^{g_31 of chunk 0}) S0  (transposed: row j over key channels); O = 0
        ok = group_and(kBarEpi, wait_bar(&bars[B_VEC0], 0, abort_flag, 9));
        if (ok) {
            vecF[j] = expf(vecT0[j]);
            named_bar_sync(kBarEpi, 128);
#pragma unroll
            for (int g4 = 0; g4 < 4; ++g4) {
                uint32_t m[32], sbf[16];
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const int ch = 32 * g4 + q;
                    const float s0 = prm.init_state ? prm.init_state[state_base + (int64_t)ch * kD + j] : 0.f;
                    m[q] = __float_as_uint(vecF[ch] * s0);
                }
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    sbf[q] = pack_bf16x2(__uint_as_float(m[2 * q]), __uint_as_float(m[2 * q + 1]));
                tmem_st32(tb + kTmMaster + lane_off + 32 * g4, m);
                tmem_st16(tb + kTmSB + lane_off + 16 * g4, sbf);
            }
            tmem_st32(tb + kTmO + lane_off, zeros);
            tmem_st32(tb + kTmO + lane_off + 32, zeros);
            tc_wait_st();
            tc_fence_before();
            named_bar_sync(kBarEpi, 128);
            if (te == 0) mbar_arrive(&bars[B_SREADY]);
        }
        for (int c = 0; ok && c < nc; ++c) {
            const int64_t t0 = t_begin + 64 * c;
            const int L = (int)(t_end - t0 < 64 ? t_end - t0 : 64);
            // U^T (fp32) -> bf16 pairs in TMEM for the update MMAs
            if (!group_and(kBarEpi, wait_bar(&bars[B_UDONE], c & 1, abort_flag, 10))) break;
            if (te == 0) GDR2_TRACE_AT(c, 20);
            tc_fence_after();
            {
                uint32_t v0[32], v1[32], ub[16];
                tmem_ld32(tb + kTmU + lane_off, v0);
                tmem_ld32(tb + kTmU + lane_off + 32, v1);
                tc_wait_ld();
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    ub[q] = pack_bf16x2(__uint_as_float(v0[2 * q]), __uint_as_float(v0[2 * q + 1]));
                tmem_st16(tb + kTmUB + lane_off, ub);
#pragma unroll
                for (int q = 0; q < 16; ++q)
                    ub[q] = pack_bf16x2(__uint_as_float(v1[2 * q]), __uint_as_float(v1[2 * q + 1]));
                tmem_st16(tb + kTmUB + lane_off + 16, ub);
                tc_wait_st();
            }
            tc_fence_before();
            named_bar_sync(kBarEpi, 128);
            if (te == 0) {
                GDR2_TRACE_AT(c, 21);
                mbar_arrive(&bars[B_UCONV]);
            }

            if (!group_and(kBarEpi, wait_bar(&bars[B_SDONE], c & 1, abort_flag, 11))) break;
            if (te == 0) GDR2_TRACE_AT(c, 22);
            tc_fence_after();
            // O^T row j -> registers as bf16 pairs (rows r, r+1), then the O region
            // is zeroed for the next chunk; o is stored after the state hand-off
            uint32_t opk[32];
            {
                uint32_t v0[32], v1[32];
                tmem_ld32(tb + kTmO + lane_off, v0);
                tmem_ld32(tb + kTmO + lane_off + 32, v1);
                tc_wait_ld();
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    opk[q] = pack_bf16x2(__uint_as_float(v0[2 * q]), __uint_as_float(v0[2 * q + 1]));
                    opk[16 + q] = pack_bf16x2(__uint_as_float(v1[2 * q]), __uint_as_float(v1[2 * q + 1]));
                }
            }
            const bool last = (c + 1 == nc);
            if (!last) {
                tmem_st32(tb + kTmO + lane_off, zeros);
                tmem_st32(tb + kTmO + lane_off + 32, zeros);
            }
            if (te == 0) GDR2_TRACE_AT(c, 23);
            // state scale: e^{g_C - g_31} and, unless last, e^{g'_31} of the next chunk
            // (the group barrier also means everyone is done reading vecF)
            if (!group_and(kBarEpi, last || wait_bar(&bars[B_VEC0 + ((c + 1) & 1)], ((c + 1) >> 1) & 1,
                                                      abort_flag, 26)))
                break;
            vecF[j] = expf(vecT1[(c & 3) * 128 + j] + (last ? 0.f : vecT0[((c + 1) & 3) * 128 + j]));
            named_bar_sync(kBarEpi, 128);
#pragma unroll 1
            for (int hh = 0; hh < 2; ++hh) {
                uint32_t m0[32], m1[32];
                tmem_ld32(tb + kTmMaster + lane_off + 64 * hh, m0);
                tmem_ld32(tb + kTmMaster + lane_off + 64 * hh + 32, m1);
                tc_wait_ld();
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 f0 = *reinterpret_cast<const float4 *>(vecF + 64 * hh + 4 * q);
                    const float4 f1 = *reinterpret_cast<const float4 *>(vecF + 64 * hh + 32 + 4 * q);
                    m0[4 * q + 0] = __float_as_uint(__uint_as_float(m0[4 * q + 0]) * f0.x);
                    m0[4 * q + 1] = __float_as_uint(__uint_as_float(m0[4 * q + 1]) * f0.y);
                    m0[4 * q + 2] = __float_as_uint(__uint_as_float(m0[4 * q + 2]) * f0.z);
                    m0[4 * q + 3] = __float_as_uint(__uint_as_float(m0[4 * q + 3]) * f0.w);
                    m1[4 * q + 0] = __float_as_uint(__uint_as_float(m1[4 * q + 0]) * f1.x);
                    m1[4 * q + 1] = __float_as_uint(__uint_as_float(m1[4 * q + 1]) * f1.y);
                    m1[4 * q + 2] = __float_as_uint(__uint_as_float(m1[4 * q + 2]) * f1.z);
                    m1[4 * q + 3] = __float_as_uint(__uint_as_float(m1[4 * q + 3]) * f1.w);
                }
                if (!last) {
                    uint32_t s0b[16], s1b[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        s0b[q] = pack_bf16x2(__uint_as_float(m0[2 * q]), __uint_as_float(m0[2 * q + 1]));
                        s1b[q] = pack_bf16x2(__uint_as_float(m1[2 * q]), __uint_as_float(m1[2 * q + 1]));
                    }
                    tmem_st32(tb + kTmMaster + lane_off + 64 * hh, m0);
                    tmem_st32(tb + kTmMaster + lane_off + 64 * hh + 32, m1);
                    tmem_st16(tb + kTmSB + lane_off + 32 * hh, s0b);
                    tmem_st16(tb + kTmSB + lane_off + 32 * hh + 16, s1b);
                } else if (prm.final_state) {
#pragma unroll
                    for (int q = 0; q < 32; ++q) {
                        prm.final_state[state_base + (int64_t)(64 * hh + q) * kD + j] = __uint_as_float(m0[q]);
                        prm.final_state[state_base + (int64_t)(64 * hh + 32 + q) * kD + j] = __uint_as_float(m1[q]);
                    }
                }
            }
            tc_wait_st();
            tc_fence_before();
            named_bar_sync(kBarEpi, 128);
            if (te == 0) GDR2_TRACE_AT(c, 24);
            if (!last && te == 0) mbar_arrive(&bars[B_SREADY]);
            {   // o rows of this chunk: adjacent lanes (channels j, j+1) trade halves so
                // that the even lane stores rows 2q and the odd lane rows 2q+1 as
                // 4-byte (j, j+1) pairs
                const bool odd = (lane & 1) != 0;
                __nv_bfloat16 *obase = prm.o + (t0 * H + h) * kD + (j & ~1);
                const int64_t rstride = H * kD;
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const uint32_t mine = opk[q];                       // rows (2q, 2q+1) of channel j
                    const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
                    // even lane: (row 2q: j, j+1); odd lane: (row 2q+1: j-1, j)
                    const uint32_t pr = odd ? __byte_perm(other, mine, 0x7632) : __byte_perm(mine, other, 0x5410);
                    const int r = 2 * q + (odd ? 1 : 0);
                    if (r < L) *reinterpret_cast<uint32_t *>(obase + r * rstride) = pr;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2) tmem_dealloc(tb, 512);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Token tensor [tokens, H, 128] as a 3-D map; box = 64 tokens x 1 head x box_x channels.
bool make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int elem, int64_t tokens,
              int64_t H, int box_x, CUtensorMapSwizzle sw)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)kD * elem, (cuuint64_t)(H * kD * elem)};
    cuuint32_t box[3] = {(cuuint32_t)box_x, 1, 64};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, dt, 3, const_cast<void *>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
               sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool chunk_tc_supported(const ChunkArgs &a)
{
    return a.bf16 && a.dk == 128 && a.dv == 128;
}

cudaError_t launch_chunk_tc(const ChunkArgs &a, cudaStream_t stream)
{
    const int64_t tokens = a.B * a.T;
    const int64_t grid = a.num_seqs * a.H;
    if (grid == 0) return cudaSuccess;
    if (tokens > 0x7fffffffLL || grid > 0x7fffffffLL) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mb, mv, mla, mw;
    const int64_t tk = tokens > 0 ? tokens : 1;
    const void *dummy = a.q ? a.q : (const void *)a.o;
    bool ok = make_map(&mq, a.q ? a.q : dummy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tk, a.H, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&mk, a.k ? a.k : dummy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tk, a.H, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&mb, a.b ? a.b : dummy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tk, a.H, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&mv, a.v ? a.v : dummy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tk, a.H, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&mla, a.log_alpha ? (const void *)a.log_alpha : dummy, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, tk, a.H, 128, CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map(&mw, a.w ? a.w : dummy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tk, a.H, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (!ok) return cudaErrorInvalidValue;
    TcParams p;
    p.la = a.log_alpha;
    p.w = (const __nv_bfloat16 *)a.w;
    p.init_state = a.init_state;
    p.cu_seqlens = a.cu_seqlens;
    p.order = a.order;
    p.o = (__nv_bfloat16 *)a.o;
    p.final_state = a.final_state;
    p.T = a.T;
    p.H = a.H;
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    chunk_tc_kernel<<<(unsigned)grid, kThreadsTC, kSmemBytes, stream>>>(mq, mk, mb, mv, mla, mw, p);
    return cudaGetLastError();
}

namespace {
// One CTA waiting on a barrier that nothing arrives on, through the kernel's
// bounded wait with a caller-chosen limit (failure-detection self-test).
__global__ void wait_selftest_kernel(uint64_t timeout_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        WaitGuard g{globaltimer_ns() + timeout_ns, &abort_flag, &g_chunk_tc_error};
        mbar_wait(&bar, 0, g, 31);
    }
}
}  // namespace

cudaError_t chunk_tc_wait_selftest(uint32_t timeout_us, cudaStream_t stream)
{
    wait_selftest_kernel<<<1, 32, 0, stream>>>((uint64_t)timeout_us * 1000ull);
    return cudaGetLastError();
}

cudaError_t chunk_tc_read_and_clear_error(int *code)
{
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(code, g_chunk_tc_error, sizeof(int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_chunk_tc_error, &zero, sizeof(int));
}

}  // namespace gdr2
