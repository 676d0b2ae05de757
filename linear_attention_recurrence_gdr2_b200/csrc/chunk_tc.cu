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
// M axis and on the 128 TMEM lanes:
//     [A; P]    = [Em; Qm] Km^T                      (M=128, N=64,  K=128)
//     W^T       = Em^T T^T,   U0^T = Z^T T^T         (M=128, N=64,  K=64)
//     U^T       = U0^T - Sm^T W^T,  O^T = Sm^T Qm^T  (A = Sm^T from TMEM)
//     O^T      += U^T P^T,  M^T += U^T Km            (A = U^T from TMEM)
// The fp32 state lives in TMEM (as M = Diag(e^{g_31}) S plus the chunk's
// update); once per chunk the epilogue scales it by e^{g_C - g_31 + g'_31}
// (g'_31: the next chunk's half sum) and writes its bf16 copy back to TMEM as
// the next chunk's MMA operand.
//
// Warp roles (12 warps):
//   0      TMA producer of q, k, b tiles (double-buffered slots)
//   1      tcgen05.mma issuer (one thread, polls both pipelines)
//   2      TMEM allocator; TMA producer of v tiles and L2 prefetch of
//          log_alpha and w
//   3      idle
//   4..7   prep: cumulative decay, factors, Z, (I + A)^{-1}, W^T to smem
//   8..11  epilogue: U^T to bf16, o stores, state scaling, final state
// Every wait is bounded: after about a second without progress the CTA
// records the site in the device error word and winds down (drains its TMA
// loads and MMAs, frees TMEM, returns).
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

#include <mutex>

namespace gdr2 {

__device__ int g_chunk_tc_error;

namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kThreadsTC = 384;
constexpr uint64_t kWaitNs = 1000000000ull;  // one second per wait

// ---- shared memory map (bytes from the 1024-aligned base) ----------------
constexpr uint32_t kEQ0 = 0;             // [kb0: Em 8K | Qm 8K][kb1: Em 8K | Qm 8K]
constexpr uint32_t kEQ1 = 32768;
constexpr uint32_t kKB0 = 65536;         // Km: [kb0 8K][kb1 8K]
constexpr uint32_t kKB1 = 81920;
constexpr uint32_t kZB = 98304;          // v -> Z: [dv block 0 8K][dv block 1 8K]
constexpr uint32_t kTB = 114688;         // T bf16, 64 rows x 128 B
constexpr uint32_t kPB0 = 122880;        // P bf16, 64 rows x 128 B
constexpr uint32_t kPB1 = 131072;
constexpr uint32_t kWB0 = 139264;        // W^T bf16, 128 rows x 128 B
constexpr uint32_t kWB1 = 155648;
constexpr uint32_t kSA = 172032;         // fp32 A, 64 x 65
constexpr uint32_t kST = kSA + 64 * 65 * 4;  // fp32 T, 64 x 65
constexpr uint32_t kVEC = kST + 64 * 65 * 4; // half sums: T0[4][128], T1[4][128], f[128]
constexpr uint32_t kBAR = kVEC + (8 * 128 + 128) * 4;
constexpr int kNumBars = 20;
constexpr uint32_t kMISC = kBAR + kNumBars * 8;
constexpr uint32_t kSmemBytes = kMISC + 64 + 1024;  // + alignment slack

// barrier indices
enum {
    B_FULL0 = 0, B_FULL1, B_SLOTFREE0, B_SLOTFREE1, B_VFULL, B_VFREE, B_PREP, B_AP, B_T,
    B_WDONE, B_WREADY0, B_WREADY1, B_SREADY, B_UDONE, B_UCONV, B_SDONE, B_VEC0, B_VEC1,
    B_DRAIN, B_SPARE
};

// ---- TMEM column map ------------------------------------------------------
constexpr uint32_t kTmMaster = 0;    // fp32 state (transposed), 128 columns
constexpr uint32_t kTmO = 128;       // O^T fp32, 64
constexpr uint32_t kTmU0 = 192;      // U^T fp32 slots, 64 each
constexpr uint32_t kTmU1 = 256;
constexpr uint32_t kTmAPW = 320;     // [A;P] then W^T, fp32, 64
constexpr uint32_t kTmSB = 384;      // Sm^T bf16 pairs, 64 words
constexpr uint32_t kTmUB = 448;      // U^T bf16 pairs, 32 words

// prep / epilogue named barriers
constexpr uint32_t kBarPrep = 1, kBarEpi = 2;

struct TcParams {
    const float *la;
    const __nv_bfloat16 *w;
    const float *init_state;
    const int32_t *cu_seqlens;
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

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d) : "memory");
}
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void st_shared_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ float2 bf2_to_f2(uint32_t v) {
    return __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&v));
}

// Writes 64 fp32 values as one 128-byte bf16 row of a 128B-swizzled tile.
__device__ __forceinline__ void store_row_bf16_sw128(uint32_t tile, uint32_t row, const float *x) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const uint32_t a = pack_bf16x2(x[8 * q + 0], x[8 * q + 1]);
        const uint32_t b = pack_bf16x2(x[8 * q + 2], x[8 * q + 3]);
        const uint32_t c = pack_bf16x2(x[8 * q + 4], x[8 * q + 5]);
        const uint32_t d = pack_bf16x2(x[8 * q + 6], x[8 * q + 7]);
        st_shared_v4(tile + sw128_offset(row, 16 * q), a, b, c, d);
    }
}

__global__ void __launch_bounds__(kThreadsTC, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_v,
                const __grid_constant__ CUtensorMap map_la, const __grid_constant__ CUtensorMap map_w,
                TcParams prm)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kMISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kMISC + 4);
    float *sA = reinterpret_cast<float *>(smem + kSA);
    float *sT = reinterpret_cast<float *>(smem + kST);
    float *vecT0 = reinterpret_cast<float *>(smem + kVEC);         // [4][128]
    float *vecT1 = vecT0 + 4 * 128;                                 // [4][128]
    float *vecF = vecT1 + 4 * 128;                                  // [128]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = prm.H;
    const int64_t n = blockIdx.x / H, h = blockIdx.x % H;
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
    if (warp == 0) {
        // ---------------- producer: q, k, b tiles ----------------------------
        if (lane == 0) {
            int issued[2] = {0, 0};
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1;
                if (c >= 2 && !wait_bar(&bars[B_SLOTFREE0 + s], ((c >> 1) - 1) & 1, abort_flag, 1)) break;
                const int z = (int)(t_begin + 64 * c);
                const uint32_t eq = sbase + (s ? kEQ1 : kEQ0), kb = sbase + (s ? kKB1 : kKB0);
                mbar_arrive_expect_tx(&bars[B_FULL0 + s], 3 * 16384);
                for (int blk = 0; blk < 2; ++blk) {
                    void *dst_e = smem + (eq - sbase) + blk * 16384;
                    void *dst_q = smem + (eq - sbase) + blk * 16384 + 8192;
                    void *dst_k = smem + (kb - sbase) + blk * 8192;
                    tma_load_3d(dst_e, &map_b, &bars[B_FULL0 + s], 64 * blk, (int)h, z);
                    tma_load_3d(dst_q, &map_q, &bars[B_FULL0 + s], 64 * blk, (int)h, z);
                    tma_load_3d(dst_k, &map_k, &bars[B_FULL0 + s], 64 * blk, (int)h, z);
                }
                issued[s] = (c >> 1) + 1;
            }
            // drain: wait (bounded) for every load issued into each slot
            for (int s = 0; s < 2; ++s)
                if (issued[s] > 0) {
                    WaitGuard g{globaltimer_ns() + kWaitNs, abort_flag, &g_chunk_tc_error};
                    volatile int dummy = 0;
                    WaitGuard g2{g.deadline_ns, &dummy, &g_chunk_tc_error};
                    mbar_wait(&bars[B_FULL0 + s], (issued[s] - 1) & 1, g2, 20);
                }
        }
    } else if (warp == 2) {
        // ---------------- producer: v tiles, L2 prefetch of log_alpha, w -----
        if (lane == 0) {
            int issued = 0;
            tma_prefetch_3d(&map_la, 0, (int)h, (int)t_begin);
            tma_prefetch_3d(&map_w, 0, (int)h, (int)t_begin);
            for (int c = 0; c < nc; ++c) {
                if (c >= 1 && !wait_bar(&bars[B_VFREE], (c - 1) & 1, abort_flag, 2)) break;
                const int z = (int)(t_begin + 64 * c);
                mbar_arrive_expect_tx(&bars[B_VFULL], 16384);
                for (int blk = 0; blk < 2; ++blk)
                    tma_load_3d(smem + kZB + blk * 8192, &map_v, &bars[B_VFULL], 64 * blk, (int)h, z);
                issued = c + 1;
                if (c + 1 < nc) {
                    tma_prefetch_3d(&map_la, 0, (int)h, z + 64);
                    tma_prefetch_3d(&map_w, 0, (int)h, z + 64);
                }
            }
            if (issued > 0) {
                volatile int dummy = 0;
                WaitGuard g2{globaltimer_ns() + kWaitNs, &dummy, &g_chunk_tc_error};
                mbar_wait(&bars[B_VFULL], (issued - 1) & 1, g2, 21);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ------------------------------------------
        if (lane == 0) {
            const uint32_t i_ap = idesc_bf16_f32(128, 64, false, false);
            const uint32_t i_w = idesc_bf16_f32(128, 64, true, false);
            const uint32_t i_us = idesc_bf16_f32(128, 64, false, true, true);
            const uint32_t i_os = idesc_bf16_f32(128, 64, false, false);
            const uint32_t i_su = idesc_bf16_f32(128, 128, false, true);
            int cp = 0, pstep = 0, cc = 0, cstep = 0;
            uint64_t last_progress = globaltimer_ns();
            while (cc < nc) {
                bool progress = false;
                if (cp < nc) {
                    const int s = cp & 1;
                    const uint32_t eq = sbase + (s ? kEQ1 : kEQ0), kbb = sbase + (s ? kKB1 : kKB0);
                    if (pstep == 0 && mbar_test(&bars[B_PREP], cp & 1)) {
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t a = smem_desc_sw128(eq + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                            const uint64_t b = smem_desc_sw128(kbb + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
                            mma_ss(tb + kTmAPW, a, b, i_ap, kk > 0);
                        }
                        tc_commit(&bars[B_AP]);
                        pstep = 1;
                        progress = true;
                    } else if (pstep == 1 && cc > cp - 2 && mbar_test(&bars[B_T], cp & 1)) {
                        tc_fence_after();
                        const uint32_t ucol = s ? kTmU1 : kTmU0;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t bt = smem_desc_sw128(sbase + kTB + kk * 32, 16, 1024);
                            const uint64_t ae = smem_desc_sw128(eq + kk * 2048, 16384, 1024);
                            const uint64_t az = smem_desc_sw128(sbase + kZB + kk * 2048, 8192, 1024);
                            mma_ss(tb + kTmAPW, ae, bt, i_w, kk > 0);
                            mma_ss(tb + ucol, az, bt, i_w, kk > 0);
                        }
                        tc_commit(&bars[B_WDONE]);
                        tc_commit(&bars[B_VFREE]);
                        pstep = 0;
                        ++cp;
                        progress = true;
                    }
                }
                if (cc < cp) {
                    const int s = cc & 1;
                    const uint32_t eq = sbase + (s ? kEQ1 : kEQ0), kbb = sbase + (s ? kKB1 : kKB0);
                    const uint32_t ucol = s ? kTmU1 : kTmU0;
                    if (cstep == 0 && mbar_test(&bars[B_WREADY0 + s], (cc >> 1) & 1) &&
                        mbar_test(&bars[B_SREADY], cc & 1)) {
                        tc_fence_after();
                        const uint32_t wb = sbase + (s ? kWB1 : kWB0);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t bw = smem_desc_sw128(wb + kk * 2048, 8192, 1024);
                            mma_ts(tb + ucol, tb + kTmSB + kk * 8, bw, i_us, 1);
                        }
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t bq = smem_desc_sw128(eq + (kk >> 2) * 16384 + 8192 + (kk & 3) * 32, 16, 1024);
                            mma_ts(tb + kTmO, tb + kTmSB + kk * 8, bq, i_os, kk > 0);
                        }
                        tc_commit(&bars[B_UDONE]);
                        cstep = 1;
                        progress = true;
                    } else if (cstep == 1 && mbar_test(&bars[B_UCONV], cc & 1)) {
                        tc_fence_after();
                        const uint32_t pb = sbase + (s ? kPB1 : kPB0);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t bp = smem_desc_sw128(pb + kk * 32, 16, 1024);
                            mma_ts(tb + kTmO, tb + kTmUB + kk * 8, bp, i_os, 1);
                        }
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t bk = smem_desc_sw128(kbb + kk * 2048, 8192, 1024);
                            mma_ts(tb + kTmMaster, tb + kTmUB + kk * 8, bk, i_su, 1);
                        }
                        tc_commit(&bars[B_SDONE]);
                        tc_commit(&bars[B_SLOTFREE0 + s]);
                        cstep = 0;
                        ++cc;
                        progress = true;
                    }
                }
                if (progress) {
                    last_progress = globaltimer_ns();
                } else {
                    if (*abort_flag) break;
                    if (globaltimer_ns() - last_progress > kWaitNs) {
                        *abort_flag = 1;
                        atomicCAS(&g_chunk_tc_error, 0, 0x100 | 3);
                        break;
                    }
                }
            }
            // drain every MMA this thread issued before TMEM is released
            tc_commit(&bars[B_DRAIN]);
            volatile int dummy = 0;
            WaitGuard g2{globaltimer_ns() + kWaitNs, &dummy, &g_chunk_tc_error};
            mbar_wait(&bars[B_DRAIN], 0, g2, 22);
        }
    } else if (warp >= 4 && warp < 8) {
        // ---------------- prep warpgroup ---------------------------------------
        const int pw = warp - 4, tp = tid - 128;
        const int kb = pw & 1, hf = pw >> 1;
        const int p = kb * 32 + lane;          // column pair: channels 2p, 2p+1
        const int r0 = 32 * hf;
        for (int c = 0; c < nc; ++c) {
            const int s = c & 1;
            const int64_t t0 = t_begin + 64 * c;
            const int L = (int)(t_end - t0 < 64 ? t_end - t0 : 64);
            const uint32_t eq = sbase + (s ? kEQ1 : kEQ0), kbb = sbase + (s ? kKB1 : kKB0);

            // log-decay of this thread's 32 rows and 2 channels (L2-prefetched)
            float2 la[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int r = r0 + i;
                la[i] = r < L ? *reinterpret_cast<const float2 *>(prm.la + ((t0 + r) * H + h) * kD + 2 * p)
                              : make_float2(0.f, 0.f);
            }
            // d_r = g_r - g_31: suffix sums (first half), prefix sums (second half)
            float2 tot = make_float2(0.f, 0.f);
            if (hf == 0) {
#pragma unroll
                for (int i = 31; i >= 0; --i) {
                    const float2 x = la[i];
                    la[i] = make_float2(-tot.x, -tot.y);
                    tot.x += x.x;
                    tot.y += x.y;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    tot.x += la[i].x;
                    tot.y += la[i].y;
                    la[i] = tot;
                }
            }
            float *vt = (hf == 0 ? vecT0 : vecT1) + (c & 3) * 128;
            vt[2 * p] = tot.x;
            vt[2 * p + 1] = tot.y;

            if (!group_and(kBarPrep, wait_bar(&bars[B_FULL0 + s], (c >> 1) & 1, abort_flag, 4))) break;
            // factors, in place: b -> Em, q -> Qm, k -> Km
            {
                const uint32_t e_tile = eq + kb * 16384, q_tile = e_tile + 8192;
                const uint32_t k_tile = kbb + kb * 8192;
                const uint32_t byte = 4 * lane;  // channel pair within the 64-wide block
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int r = r0 + i;
                    const uint32_t off = sw128_offset(r, byte);
                    uint32_t oq = 0, ok = 0, oe = 0;
                    if (r < L) {
                        const float2 qv = bf2_to_f2(ld_shared_u32(q_tile + off));
                        const float2 kv = bf2_to_f2(ld_shared_u32(k_tile + off));
                        const float2 bv = bf2_to_f2(ld_shared_u32(e_tile + off));
                        const float ux = __expf(la[i].x), uy = __expf(la[i].y);
                        const float dx = __expf(-la[i].x), dy = __expf(-la[i].y);
                        oq = pack_bf16x2(qv.x * ux, qv.y * uy);
                        ok = pack_bf16x2(kv.x * dx, kv.y * dy);
                        oe = pack_bf16x2(bv.x * kv.x * ux, bv.y * kv.y * uy);
                    }
                    st_shared_u32(q_tile + off, oq);
                    st_shared_u32(k_tile + off, ok);
                    st_shared_u32(e_tile + off, oe);
                }
            }
            fence_proxy_async_smem();
            named_bar_sync(kBarPrep, 128);
            if (tp == 0) {
                mbar_arrive(&bars[B_PREP]);
                mbar_arrive(&bars[B_VEC0 + s]);
            }

            // Z = w . v in place (v tile from TMA, w from global / L2)
            {
                uint32_t wv[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int r = r0 + i;
                    wv[i] = r < L ? *reinterpret_cast<const uint32_t *>(prm.w + ((t0 + r) * H + h) * kD + 2 * p)
                                  : 0u;
                }
                if (!group_and(kBarPrep, wait_bar(&bars[B_VFULL], c & 1, abort_flag, 5))) break;
                const uint32_t z_tile = sbase + kZB + kb * 8192;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int r = r0 + i;
                    const uint32_t off = sw128_offset(r, 4 * lane);
                    uint32_t oz = 0;
                    if (r < L) {
                        const float2 vv = bf2_to_f2(ld_shared_u32(z_tile + off));
                        const float2 ww = bf2_to_f2(wv[i]);
                        oz = pack_bf16x2(vv.x * ww.x, vv.y * ww.y);
                    }
                    st_shared_u32(z_tile + off, oz);
                }
            }
            fence_proxy_async_smem();

            // [A; P] from TMEM: lanes 0-63 rows of A, lanes 64-127 rows of P
            if (!group_and(kBarPrep, wait_bar(&bars[B_AP], c & 1, abort_flag, 6))) break;
            tc_fence_after();
            {
                const uint32_t taddr = tb + kTmAPW + ((uint32_t)(32 * pw) << 16);
                uint32_t v0[32], v1[32];
                tmem_ld32(taddr, v0);
                tmem_ld32(taddr + 32, v1);
                tc_wait_ld();
                if (pw < 2) {
                    const int r = 32 * pw + lane;
                    float *row = sA + r * 65;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        row[j] = j < r ? __uint_as_float(v0[j]) : 0.f;
                        row[32 + j] = 32 + j < r ? __uint_as_float(v1[j]) : 0.f;
                    }
                } else {
                    const int r = 32 * (pw - 2) + lane;
                    float x[64];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        x[j] = j <= r ? __uint_as_float(v0[j]) : 0.f;
                        x[32 + j] = 32 + j <= r ? __uint_as_float(v1[j]) : 0.f;
                    }
                    store_row_bf16_sw128(sbase + (s ? kPB1 : kPB0), r, x);
                }
            }
            named_bar_sync(kBarPrep, 128);

            // T = (I + A)^{-1}: two 32x32 diagonal blocks by column-wise forward
            // substitution, then T10 = -T11 (A10 T00).
            if (tp < 64) {
                const int j = tp, base = (j >> 5) * 32, jj = j & 31;
                float x[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float *arow = sA + (base + i) * 65 + base;
                    float acc = (i == jj) ? 1.f : 0.f;
#pragma unroll
                    for (int s2 = 0; s2 < i; ++s2) acc = fmaf(-arow[s2], x[s2], acc);
                    x[i] = acc;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) sT[(base + i) * 65 + j] = x[i];
            }
            named_bar_sync(kBarPrep, 128);
            {   // Y = A10 T00 -> scratch in the (unused) upper-right block of sT
                const int i = tp >> 2, j0 = (tp & 3) * 8;
                float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                const float *arow = sA + (32 + i) * 65;
#pragma unroll 4
                for (int kx = 0; kx < 32; ++kx) {
                    const float a = arow[kx];
                    const float *trow = sT + kx * 65 + j0;
#pragma unroll
                    for (int q = 0; q < 8; ++q) y[q] = fmaf(a, trow[q], y[q]);
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) sT[i * 65 + 32 + j0 + q] = y[q];
            }
            named_bar_sync(kBarPrep, 128);
            {   // T10 = -T11 Y
                const int i = tp >> 2, j0 = (tp & 3) * 8;
                float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                const float *trow = sT + (32 + i) * 65 + 32;
#pragma unroll 4
                for (int kx = 0; kx < 32; ++kx) {
                    const float t = trow[kx];
                    const float *yrow = sT + kx * 65 + 32 + j0;
#pragma unroll
                    for (int q = 0; q < 8; ++q) y[q] = fmaf(-t, yrow[q], y[q]);
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) sT[(32 + i) * 65 + j0 + q] = y[q];
            }
            named_bar_sync(kBarPrep, 128);
            {   // T (lower triangle incl. diagonal) -> bf16 MMA operand
                const int r = tp >> 1, half = tp & 1;
                const float *trow = sT + r * 65 + 32 * half;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t u[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int s0 = 32 * half + 8 * q + 2 * e;
                        u[e] = pack_bf16x2(s0 <= r ? trow[8 * q + 2 * e] : 0.f,
                                           s0 + 1 <= r ? trow[8 * q + 2 * e + 1] : 0.f);
                    }
                    st_shared_v4(sbase + kTB + sw128_offset(r, 64 * half + 16 * q), u[0], u[1], u[2], u[3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(kBarPrep, 128);
            if (tp == 0) mbar_arrive(&bars[B_T]);

            // W^T (lanes = key channels) -> bf16 smem operand, MN-major rows
            if (!group_and(kBarPrep, wait_bar(&bars[B_WDONE], c & 1, abort_flag, 7))) break;
            tc_fence_after();
            {
                const uint32_t taddr = tb + kTmAPW + ((uint32_t)(32 * pw) << 16);
                uint32_t v0[32], v1[32];
                tmem_ld32(taddr, v0);
                tmem_ld32(taddr + 32, v1);
                tc_wait_ld();
                float x[64];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    x[j] = __uint_as_float(v0[j]);
                    x[32 + j] = __uint_as_float(v1[j]);
                }
                store_row_bf16_sw128(sbase + (s ? kWB1 : kWB0), 32 * pw + lane, x);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(kBarPrep, 128);
            if (tp == 0) mbar_arrive(&bars[B_WREADY0 + s]);
        }
    } else if (warp >= 8) {
        // ---------------- epilogue warpgroup -----------------------------------
        const int ew = warp - 8, te = tid - 256;
        const int j = 32 * ew + lane;                       // value channel = TMEM lane
        const uint32_t lane_off = (uint32_t)(32 * ew) << 16;
        bool ok = true;
        // master = Diag(e^{g_31 of chunk 0}) S0  (transposed: row j over key channels)
        ok = group_and(kBarEpi, wait_bar(&bars[B_VEC0], 0, abort_flag, 8));
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
            tc_wait_st();
            tc_fence_before();
            named_bar_sync(kBarEpi, 128);
            if (te == 0) mbar_arrive(&bars[B_SREADY]);
        }
        for (int c = 0; ok && c < nc; ++c) {
            const int s = c & 1;
            const int64_t t0 = t_begin + 64 * c;
            const int L = (int)(t_end - t0 < 64 ? t_end - t0 : 64);
            // U^T (fp32) -> bf16 pairs in TMEM for the second MMA group
            if (!group_and(kBarEpi, wait_bar(&bars[B_UDONE], c & 1, abort_flag, 9))) break;
            tc_fence_after();
            {
                uint32_t v0[32], v1[32], ub[16];
                const uint32_t ucol = s ? kTmU1 : kTmU0;
                tmem_ld32(tb + ucol + lane_off, v0);
                tmem_ld32(tb + ucol + lane_off + 32, v1);
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
            if (te == 0) mbar_arrive(&bars[B_UCONV]);

            if (!group_and(kBarEpi, wait_bar(&bars[B_SDONE], c & 1, abort_flag, 10))) break;
            tc_fence_after();
            {   // o rows of this chunk
                uint32_t v0[32], v1[32];
                tmem_ld32(tb + kTmO + lane_off, v0);
                tmem_ld32(tb + kTmO + lane_off + 32, v1);
                tc_wait_ld();
                __nv_bfloat16 *orow = prm.o + (t0 * H + h) * kD + j;
                const int64_t rstride = H * kD;
#pragma unroll
                for (int r = 0; r < 32; ++r)
                    if (r < L) orow[r * rstride] = __float2bfloat16_rn(__uint_as_float(v0[r]));
#pragma unroll
                for (int r = 0; r < 32; ++r)
                    if (32 + r < L) orow[(32 + r) * rstride] = __float2bfloat16_rn(__uint_as_float(v1[r]));
            }
            // state scale: e^{g_C - g_31} and, unless last, e^{g'_31} of the next chunk
            const bool last = (c + 1 == nc);
            // (the group barrier also means everyone is done reading vecF)
            if (!group_and(kBarEpi, last || wait_bar(&bars[B_VEC0 + ((c + 1) & 1)], ((c + 1) >> 1) & 1,
                                                      abort_flag, 11)))
                break;
            vecF[j] = expf(vecT1[(c & 3) * 128 + j] + (last ? 0.f : vecT0[((c + 1) & 3) * 128 + j]));
            named_bar_sync(kBarEpi, 128);
#pragma unroll 1
            for (int g4 = 0; g4 < 4; ++g4) {
                uint32_t m[32];
                tmem_ld32(tb + kTmMaster + lane_off + 32 * g4, m);
                tc_wait_ld();
#pragma unroll
                for (int q = 0; q < 32; ++q)
                    m[q] = __float_as_uint(__uint_as_float(m[q]) * vecF[32 * g4 + q]);
                if (!last) {
                    uint32_t sbf[16];
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        sbf[q] = pack_bf16x2(__uint_as_float(m[2 * q]), __uint_as_float(m[2 * q + 1]));
                    tmem_st32(tb + kTmMaster + lane_off + 32 * g4, m);
                    tmem_st16(tb + kTmSB + lane_off + 16 * g4, sbf);
                } else if (prm.final_state) {
#pragma unroll
                    for (int q = 0; q < 32; ++q)
                        prm.final_state[state_base + (int64_t)(32 * g4 + q) * kD + j] = __uint_as_float(m[q]);
                }
            }
            tc_wait_st();
            tc_fence_before();
            named_bar_sync(kBarEpi, 128);
            if (!last && te == 0) mbar_arrive(&bars[B_SREADY]);
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

cudaError_t chunk_tc_read_and_clear_error(int *code)
{
    int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbol(code, g_chunk_tc_error, sizeof(int));
    if (e != cudaSuccess) return e;
    return cudaMemcpyToSymbol(g_chunk_tc_error, &zero, sizeof(int));
}

}  // namespace gdr2
