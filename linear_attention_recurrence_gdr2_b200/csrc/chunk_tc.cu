// Chunkwise forward of Gated Delta Rule-2 for bf16 inputs, d_k = d_v = 128,
// on the sm_100a tensor cores (tcgen05 + TMEM, operands staged by TMA), two
// CTAs per (sequence, head) (a main and a helper; two such pairs per cluster).
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
// Work split. Only the state chain is serial across chunks; everything that
// depends on one chunk's inputs alone runs ahead of it on a second SM:
//   helper CTA (cluster ranks 2, 3), per chunk:
//     decay sums and factors Qm, Km, Em (in place over the q, k, b tiles),
//     [A^T | P^T] = Km [Em; Qm]^T       M=64  N=128 K=128 (tcgen05),
//     T = (I + A)^{-1} (tf32 mma.sync doubling) as bf16,
//     bulk copies of Em, Qm, Km, P^T and the half sums, and remote 16-byte
//     stores of T, into the main CTA's shared memory (distributed shared
//     memory inside the cluster);
//   main CTA (cluster ranks 0, 1), per chunk:
//     Z = w . v; -W = -(T Em) (two M=64 halves); U0^T = Z^T T^T;
//     [U^T | O^T]  += Sm^T [-W; Qm]^T   M=128 N=128 K=128, A in TMEM
//     [O^T | M^T]  += U^T [P^T | Km]    M=128 N=192 K=64,  A in TMEM
//     the epilogue (U^T to bf16, state scaling, final state), and O^T out of
//     TMEM into o (16-byte stores through a staging tile).
// Everything is computed transposed so that the value dimension (128) sits
// on the MMA's M axis and on the 128 TMEM lanes. The fp32 state lives in the
// main CTA's TMEM (as M = Diag(e^{g_31}) S plus the chunk's update); once per
// chunk the epilogue scales it by e^{g_C - g_31 + g'_31} (g'_31: the next
// chunk's half sum) and writes its bf16 copy back to TMEM as the next chunk's
// MMA operand. Both CTAs double-buffer their chunk slots; the main CTA tells
// the helper when a slot has been consumed (remote mbarrier arrives), the
// helper's copies complete on the main CTA's barriers.
//
// Warp roles (16 warps per CTA; the first warpgroup gives registers away):
//   main:   0 v and w TMA producer, slot-free relay
//           1 tcgen05.mma issuer: W, U0      2 TMEM allocator, copy-landed relay
//           3 tcgen05.mma issuer: state chain
//           4..7 Z, O^T readout and o stores   8..11 -W from TMEM   12..15 epilogue
//   helper: 0 q, k, b TMA producer           1 tcgen05.mma issuer: [A^T | P^T]
//           2 TMEM allocator, factor sender   4..11 decay factors, P^T
//           12..15 (I + A)^{-1}
// With few long sequences one launch also runs the jobs of the segment-parallel
// scan (segments.cu); a template flag compiles in the fused input prologue.
// Every wait is bounded: after about a second without progress the CTA
// records the site in the device error word, tells its peer to wind down,
// drains its own TMA loads and MMAs, frees TMEM, and returns.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

#include <mutex>

namespace gdr2 {

__device__ int g_chunk_tc_error;

namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kThreadsTC = 512;
constexpr uint64_t kWaitNs = 1000000000ull;  // one second per wait
constexpr int kPairs = 2;                     // (sequence, head) units per cluster
// Largest |g_r - g_31| (natural log) the chunk form's factors e^{+-(g_r - g_31)}
// may take: e^64 and e^-64 are normal fp32 / bf16 numbers with room for the
// products and sums they enter.
constexpr float kFactorRange = 64.f;
// Largest decay (natural log) over the 64 tokens from one chunk's middle row
// to the next one's: the epilogue moves the state between those two frames
// with the single factor e^{-that}, which must stay a normal fp32 number.
constexpr float kWindowRange = 80.f;

// ---- main CTA shared memory (bytes from the 1024-aligned base) -------------
__host__ __device__ constexpr uint32_t mEQ(int s) { return s ? 32768 : 0; }          // per key block kb: [Em -> -W 8K | Qm 8K]
__host__ __device__ constexpr uint32_t mKB(int s) { return s ? 90112 : 65536; }      // [P^T 8K | Km kb0 8K | Km kb1 8K]
constexpr uint32_t kKmOff = 8192;                  // Km after the P^T block
__host__ __device__ constexpr uint32_t mZ(int s) { return s ? 131072 : 114688; }     // v -> Z: [dv block 0 8K][dv block 1 8K]
__host__ __device__ constexpr uint32_t mT(int s) { return s ? 155648 : 147456; }     // T bf16, 64 rows x 128 B
__host__ __device__ constexpr uint32_t mVEC(int s) { return s ? 164864 : 163840; }   // half sums [T0 | T1], fp32 128 + 128
constexpr uint32_t kM_VECF = 165888;               // state scale factors, fp32 128
constexpr uint32_t kM_OST = 166400;                // o staging: 64 rows of 256 B at a 320 B pitch
constexpr uint32_t kOPitch = 320;                  // (row r+1 sits 16 banks after row r)
constexpr uint32_t kM_WT = 187392;                 // w tile (same layout as a v tile), 16 KB
// ---- helper CTA shared memory ----------------------------------------------
__host__ __device__ constexpr uint32_t hEQ(int s) { return s ? 49152 : 0; }          // [b -> Em | q -> Qm] per key block, then k -> Km
constexpr uint32_t kH_KmOff = 32768;
__host__ __device__ constexpr uint32_t hPT(int s) { return s ? 106496 : 98304; }     // P^T bf16 (MN-major operand rows s)
__host__ __device__ constexpr uint32_t hT(int s) { return s ? 122880 : 114688; }     // T bf16
constexpr uint32_t kH_LA = 131072;                 // staged log_alpha, fp32 [64][128]
constexpr int kLD = 68;                            // fp32 scratch row pitch (16-byte aligned rows)
constexpr uint32_t kH_SA = 163840;                 // fp32 A^T, 64 x kLD
constexpr uint32_t kH_ST = kH_SA + 64 * kLD * 4;   // fp32 T, 64 x kLD
__host__ __device__ constexpr uint32_t hVEC(int s) { return s ? kH_ST + 64 * kLD * 4 + 1024 : kH_ST + 64 * kLD * 4; }
constexpr uint32_t kH_BSUM = hVEC(1) + 1024;     // per-row-block log-decay sums [8][128]
// ---- both ------------------------------------------------------------------
constexpr uint32_t kBAR = kH_BSUM + 8 * 128 * 4;   // same offset in both CTAs
constexpr int kNumBars = 32;
constexpr uint32_t kMISC = kBAR + kNumBars * 8;    // TMEM slot, abort flag, copy counters, range flag
constexpr uint32_t kRangeFlagOff = 32;             // (within kMISC)
constexpr uint32_t kSmemBytes = kMISC + 64 + 1024; // + alignment slack
static_assert(kM_OST + 64 * kOPitch <= kM_WT && kM_WT + 16384 <= kBAR,
              "main shared-memory map overlaps the barriers");
static_assert(kSmemBytes <= 232448, "shared memory above the per-CTA limit");

constexpr uint32_t kFBytes = 32768 + 16384 + 1024;  // Em|Qm, Km, half sums

// barriers of the main CTA
enum {
    M_F0 = 0, M_F1, M_P0, M_P1, M_T0, M_T1, M_VFULL0, M_VFULL1, M_VFREE0, M_VFREE1, M_ZREADY0, M_ZREADY1,
    M_WDONE, M_WFREE, M_WREADY0, M_WREADY1, M_SREADY_LO, M_SREADY_HI, M_UDONE, M_UCONV, M_SDONE,
    M_OZERO,
    M_WTFULL, M_WTFREE,
    M_SLOTFREE0,
    M_SLOTFREE1, M_DRAIN, M_DRAIN2, M_NUM
};
// barriers of the helper CTA
enum {
    H_FULL0 = 0, H_FULL1, H_SLOTFREE0, H_SLOTFREE1, H_LAFULL, H_FDONE, H_AP0, H_AP1, H_XFREE0,
    H_XFREE1, H_MFREE0, H_MFREE1, H_TFREE0, H_TFREE1, H_DRAIN, H_NUM
};
static_assert(M_NUM <= kNumBars && H_NUM <= kNumBars, "barrier area too small");

// ---- TMEM column maps -------------------------------------------------------
// main (512 columns allocated)
constexpr uint32_t kTmU = 0;         // U^T fp32, 64      } one N=128 accumulator
constexpr uint32_t kTmO = 64;        // O^T fp32, 64      }        } one N=192
constexpr uint32_t kTmMaster = 128;  // state (transposed) fp32, 128 } accumulator
constexpr uint32_t kTmW = 256;       // W (M=64): lanes 0-15 of each quarter key channels 0-63,
                                     //           lanes 16-31 key channels 64-127; 64 columns
constexpr uint32_t kTmSB = 320;      // Sm^T bf16 pairs, 64 words
constexpr uint32_t kTmUB = 384;      // U^T bf16 pairs, 32 words
// helper (256 columns): [A^T | P^T] (M=64, lanes 0-15 of each quarter) for slot s at 128 s

// group (named) barriers, per CTA
constexpr uint32_t kBarZ = 1, kBarEpi = 2, kBarW = 3;   // main
constexpr uint32_t kBarPrepA = 1, kBarPrepB = 3;        // helper

struct TcParams {
    const __nv_bfloat16 *q, *k, *b, *v;  // (read directly only by the serial path)
    const float *la;
    const __nv_bfloat16 *w;
    const float *init_state;
    const int32_t *cu_seqlens;
    const int32_t *order;
    __nv_bfloat16 *o;
    float *final_state;
    int64_t T, H, units;
    int64_t tokens;  // B * T: every token range lies inside [0, tokens)
    // segment-parallel scan (nseg > 1): per sequence, jobs 0..nseg-1 run the
    // segments from their entry state (the true one for segment 0, else 0) and
    // write o and seg_s0; jobs nseg..2 nseg-2 run segments 1..nseg-1 from the
    // identity with z = 0 and write psi and seg_phi
    int nseg;
    int64_t seg_len;
    __nv_bfloat16 *psi;
    float *seg_s0, *seg_phi;
    uint32_t pre;  // GDR2_PROLOGUE_* flags (activations applied on load)
};

// Bounded wait on a barrier of this CTA (CTA-scope acquire: the peer's
// arrives only signal, and its data arrives by bulk copies that complete on
// this CTA's barriers). A wait that fails also raises the peer CTA's abort
// flag, so that the whole cluster winds down. Only the first (blocking)
// probe is inlined at each wait site; the bounded loop behind it is one
// shared function, which keeps the role loops short in instruction memory
// (their per-chunk code is fetched again every chunk) and leaves their
// registers to the hot path.
__device__ __noinline__ bool wait_bar_slow(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          uint32_t peer_abort, int site) {
    WaitGuard g{kWaitNs, abort_flag, &g_chunk_tc_error};
    const bool ok = mbar_wait(bar, parity, g, site);
    if (!ok) st_cluster_u32(peer_abort, 1u);
    return ok;
}
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         uint32_t peer_abort, int site) {
    if (mbar_try(bar, parity)) return true;
    return wait_bar_slow(bar, parity, abort_flag, peer_abort, site);
}

// Descriptor of the operand `bytes` further on in the same tile (the start
// address field is the low 14 bits in 16-byte units and shared addresses stay
// below 256 KB, so this adds without a carry out of the field).
__device__ __forceinline__ uint64_t desc_at(uint64_t d, uint32_t bytes) { return d + (bytes >> 4); }

// Bounded wait that polls without suspending, for the state-chain MMA issuer
// (a suspended wait adds its wake-up time to every chunk).
__device__ __forceinline__ bool spin_bar(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                         uint32_t peer_abort, int site) {
    uint64_t deadline = 0;
    for (uint32_t it = 0;; ++it) {
        if (mbar_test(bar, parity)) return true;
        if ((it & 255u) == 255u) {
            if (*abort_flag) break;
            const uint64_t now = globaltimer_ns();
            if (deadline == 0) {
                deadline = now + kWaitNs;
            } else if (now > deadline) {
                *abort_flag = 1;
                atomicCAS(&g_chunk_tc_error, 0, 0x100 | site);
                break;
            }
        }
    }
    st_cluster_u32(peer_abort, 1u);
    return false;
}

// Bounded wait used only while winding down (never raises the abort flag).
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity, int site) {
    volatile int dummy = 0;
    WaitGuard g{kWaitNs, &dummy, &g_chunk_tc_error};
    mbar_wait(bar, parity, g, site);
}

// Barrier over an n-thread group that also ANDs one predicate across it, so
// every thread of the group takes the same continue / abort decision.
__device__ __forceinline__ bool group_and(uint32_t id, uint32_t n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r) : "r"((uint32_t)v), "r"(id), "r"(n) : "memory");
    return r != 0;
}

// An fp32 value as a tf32 MMA operand: the tensor core reads only the tf32
// bits (sign, exponent, 10 mantissa bits), i.e. the value truncated toward
// zero (relative error below 2^-10; T is consumed in bf16, 2^-9).
__device__ __forceinline__ uint32_t to_tf32(float x) { return __float_as_uint(x); }
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
#pragma unroll 2
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

// The work of one CTA pair: its (sequence, head) unit, token range and
// states. Unit u = (cluster, position in it); with a segment split, each
// (sequence, head) has 2 nseg - 1 jobs: segments 0..nseg-1 from their entry
// state (the true one for segment 0, else zero), then segments 1..nseg-1 from
// the identity with z = 0.
struct UnitJob {
    bool valid;             // false for the padding pair of the last cluster
    bool zero_v;            // identity-state run with z = 0 (writes psi and Phi)
    int64_t h, t_begin, t_end;
    const float *init_ptr;  // entry state, or null (zero, or the identity if zero_v)
    float *final_ptr;       // where the exit state goes, or null
};

__device__ __forceinline__ UnitJob unit_job(const TcParams &prm, uint32_t cta, uint32_t rank)
{
    UnitJob u{false, false, 0, 0, 0, nullptr, nullptr};
    const int64_t H = prm.H;
    // (32-bit index arithmetic: the launch keeps units below 2^30 and H below 2^16)
    const uint32_t unit = (cta / (2 * kPairs)) * kPairs + (rank % kPairs);
    if ((int64_t)unit >= prm.units) return u;
    u.valid = true;
    const uint32_t jobs = 2 * (uint32_t)prm.nseg - 1, H32 = (uint32_t)H;
    const uint32_t nj = unit / H32;
    u.h = unit % H32;
    const int job = (int)(nj % jobs);
    const int64_t n = prm.order ? (int64_t)prm.order[nj / jobs] : (int64_t)(nj / jobs);
    if (prm.cu_seqlens) {
        packed_bounds(prm.cu_seqlens, n, prm.tokens, u.t_begin, u.t_end);
    } else {
        u.t_begin = n * prm.T;
        u.t_end = u.t_begin + prm.T;
    }
    u.zero_v = job >= prm.nseg;
    const int seg = u.zero_v ? job - prm.nseg + 1 : job;
    if (prm.nseg > 1) {
        const int64_t sb = u.t_begin + seg * prm.seg_len;
        u.t_end = sb + prm.seg_len < u.t_end ? sb + prm.seg_len : u.t_end;
        u.t_begin = sb;
    }
    const int64_t state_base = (n * H + u.h) * (int64_t)kD * kD;
    if (prm.nseg == 1) {
        u.init_ptr = prm.init_state ? prm.init_state + state_base : nullptr;
        u.final_ptr = prm.final_state ? prm.final_state + state_base : nullptr;
    } else {
        const int64_t seg_base = ((n * prm.nseg + seg) * H + u.h) * (int64_t)kD * kD;
        u.init_ptr = (!u.zero_v && seg == 0 && prm.init_state) ? prm.init_state + state_base : nullptr;
        u.final_ptr = (u.zero_v ? prm.seg_phi : prm.seg_s0) + seg_base;
    }
    return u;
}

// Exact fp32 recurrence of one (sequence, head) unit, token by token, for the
// value columns [j0, j0 + 64). A unit takes this path, after its chunk pass,
// when some chunk's decay leaves the chunk form's factor range (kFactorRange):
// it runs the token rule as the article states it ("Gated Delta Rule-2: two
// gates instead of one", ainews.random.gg): decay, erase read e^T S', delta
// write, readout with the post-update state, so any alpha in (0, 1] is exact
// to fp32 rounding. Columns of S evolve independently of each other, so each
// CTA of the pair takes half of them. All 512 threads: thread t holds key
// channels 16 (t >> 6) .. +15 of column j0 + (t & 63) in registers (the code
// runs after the role split, where the first warpgroup keeps 40 registers).
constexpr int kSerTok = 16;  // tokens staged in shared memory per batch
template <bool kPre>
__device__ __forceinline__ void serial_unit(const TcParams &prm, const UnitJob &u, int j0,
                                           unsigned char *smem, int t)
{
    const int64_t H = prm.H, h = u.h;
    const bool zero_v = u.zero_v;
    const int j = t & 63, kg = t >> 6, c0 = 16 * kg;
    float *vec = reinterpret_cast<float *>(smem);  // [kSerTok][4][128]: alpha, e = b.k, k, q
    float *zt = vec + kSerTok * 4 * kD;            // [kSerTok][64]: z = w.v of this CTA's columns
    float *red = zt + kSerTok * 64;                // [2][2][8][64]: partial e^T S', q^T S'
    float *kqp = red + 2 * 2 * 8 * 64;             // [2][8]: partial k^T q
    float st[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int c = c0 + i;
        st[i] = u.init_ptr ? u.init_ptr[(int64_t)c * kD + j0 + j] : ((zero_v && c == j0 + j) ? 1.f : 0.f);
    }
    int buf = 0;
    for (int64_t tb = u.t_begin; tb < u.t_end; tb += kSerTok) {
        const int nb = (int)(u.t_end - tb < kSerTok ? u.t_end - tb : kSerTok);
        __syncthreads();  // the previous batch has been consumed
        {   // staging: token r = t >> 5, key channels 4 (t & 31) .. +3, two of z
            const int r = t >> 5, cb = 4 * (t & 31);
            float qf[4] = {0.f, 0.f, 0.f, 0.f}, kf[4] = {0.f, 0.f, 0.f, 0.f};
            float bf[4] = {0.f, 0.f, 0.f, 0.f}, lf[4] = {0.f, 0.f, 0.f, 0.f};
            if (r < nb) {
                const int64_t base = ((tb + r) * H + h) * kD + cb;
                const uint2 qr = *reinterpret_cast<const uint2 *>(prm.q + base);
                const uint2 kr = *reinterpret_cast<const uint2 *>(prm.k + base);
                const uint2 br = *reinterpret_cast<const uint2 *>(prm.b + base);
                const float4 l4 = *reinterpret_cast<const float4 *>(prm.la + base);
                float2 x = bf2_to_f2(qr.x), y = bf2_to_f2(qr.y);
                qf[0] = x.x; qf[1] = x.y; qf[2] = y.x; qf[3] = y.y;
                x = bf2_to_f2(kr.x); y = bf2_to_f2(kr.y);
                kf[0] = x.x; kf[1] = x.y; kf[2] = y.x; kf[3] = y.y;
                x = bf2_to_f2(br.x); y = bf2_to_f2(br.y);
                bf[0] = x.x; bf[1] = x.y; bf[2] = y.x; bf[3] = y.y;
                lf[0] = l4.x; lf[1] = l4.y; lf[2] = l4.z; lf[3] = l4.w;
            }
            if (kPre && (prm.pre & GDR2_PROLOGUE_QK_L2NORM)) {  // a warp holds one token's row
                float sq = 0.f, sk = 0.f;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    sq = fmaf(qf[i], qf[i], sq);
                    sk = fmaf(kf[i], kf[i], sk);
                }
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1) {
                    sq += __shfl_xor_sync(0xffffffffu, sq, m);
                    sk += __shfl_xor_sync(0xffffffffu, sk, m);
                }
                sq = rsqrtf(sq + 1e-6f);
                sk = rsqrtf(sk + 1e-6f);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    qf[i] *= sq;
                    kf[i] *= sk;
                }
            }
            if (r < nb) {
                const bool sig = kPre && (prm.pre & GDR2_PROLOGUE_GATE_SIGMOID) != 0;
                const bool spl = kPre && (prm.pre & GDR2_PROLOGUE_DECAY_SOFTPLUS) != 0;
                float *vr = vec + r * 4 * kD + cb;
                float4 al, ev;
                // (alpha by the hardware exponential: relative error a few 1e-6 at
                // |log alpha| = 20, far inside the fp32 bound)
                al.x = __expf(spl ? pre_neg_softplus(lf[0]) : lf[0]);
                al.y = __expf(spl ? pre_neg_softplus(lf[1]) : lf[1]);
                al.z = __expf(spl ? pre_neg_softplus(lf[2]) : lf[2]);
                al.w = __expf(spl ? pre_neg_softplus(lf[3]) : lf[3]);
                ev.x = (sig ? pre_sigmoid(bf[0]) : bf[0]) * kf[0];
                ev.y = (sig ? pre_sigmoid(bf[1]) : bf[1]) * kf[1];
                ev.z = (sig ? pre_sigmoid(bf[2]) : bf[2]) * kf[2];
                ev.w = (sig ? pre_sigmoid(bf[3]) : bf[3]) * kf[3];
                *reinterpret_cast<float4 *>(vr) = al;
                *reinterpret_cast<float4 *>(vr + kD) = ev;
                *reinterpret_cast<float4 *>(vr + 2 * kD) = make_float4(kf[0], kf[1], kf[2], kf[3]);
                *reinterpret_cast<float4 *>(vr + 3 * kD) = make_float4(qf[0], qf[1], qf[2], qf[3]);
                if (!zero_v) {
                    const int cz = 2 * (t & 31);
                    const int64_t vb = ((tb + r) * H + h) * kD + j0 + cz;
                    const float2 vv = bf2_to_f2(*reinterpret_cast<const uint32_t *>(prm.v + vb));
                    float2 ww = bf2_to_f2(*reinterpret_cast<const uint32_t *>(prm.w + vb));
                    if (sig) ww = make_float2(pre_sigmoid(ww.x), pre_sigmoid(ww.y));
                    *reinterpret_cast<float2 *>(zt + r * 64 + cz) = make_float2(ww.x * vv.x, ww.y * vv.y);
                }
            }
        }
        __syncthreads();
        for (int r = 0; r < nb; ++r) {
            const float *vr = vec + r * 4 * kD + c0;
            float pe = 0.f, pq = 0.f, pkq = 0.f;
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
                const float4 a = *reinterpret_cast<const float4 *>(vr + 4 * i4);
                st[4 * i4 + 0] *= a.x; st[4 * i4 + 1] *= a.y; st[4 * i4 + 2] *= a.z; st[4 * i4 + 3] *= a.w;
                const float4 e = *reinterpret_cast<const float4 *>(vr + kD + 4 * i4);
                pe = fmaf(e.x, st[4 * i4 + 0], pe); pe = fmaf(e.y, st[4 * i4 + 1], pe);
                pe = fmaf(e.z, st[4 * i4 + 2], pe); pe = fmaf(e.w, st[4 * i4 + 3], pe);
                const float4 q = *reinterpret_cast<const float4 *>(vr + 3 * kD + 4 * i4);
                pq = fmaf(q.x, st[4 * i4 + 0], pq); pq = fmaf(q.y, st[4 * i4 + 1], pq);
                pq = fmaf(q.z, st[4 * i4 + 2], pq); pq = fmaf(q.w, st[4 * i4 + 3], pq);
                const float4 k = *reinterpret_cast<const float4 *>(vr + 2 * kD + 4 * i4);
                pkq = fmaf(k.x, q.x, pkq); pkq = fmaf(k.y, q.y, pkq);
                pkq = fmaf(k.z, q.z, pkq); pkq = fmaf(k.w, q.w, pkq);
            }
            float *rb = red + buf * 2 * 8 * 64;
            rb[kg * 64 + j] = pe;
            rb[8 * 64 + kg * 64 + j] = pq;
            if (j == 0) kqp[buf * 8 + kg] = pkq;
            __syncthreads();
            float rr = 0.f, pp = 0.f, kq = 0.f;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
                rr += rb[g * 64 + j];
                pp += rb[8 * 64 + g * 64 + j];
                kq += kqp[buf * 8 + g];
            }
            const float delta = (zero_v ? 0.f : zt[r * 64 + j]) - rr;
#pragma unroll
            for (int i4 = 0; i4 < 4; ++i4) {
                const float4 k = *reinterpret_cast<const float4 *>(vr + 2 * kD + 4 * i4);
                st[4 * i4 + 0] = fmaf(k.x, delta, st[4 * i4 + 0]);
                st[4 * i4 + 1] = fmaf(k.y, delta, st[4 * i4 + 1]);
                st[4 * i4 + 2] = fmaf(k.z, delta, st[4 * i4 + 2]);
                st[4 * i4 + 3] = fmaf(k.w, delta, st[4 * i4 + 3]);
            }
            if (kg == 0)
                (zero_v ? prm.psi : prm.o)[((tb + r) * H + h) * kD + j0 + j] = __float2bfloat16_rn(fmaf(kq, delta, pp));
            buf ^= 1;
        }
    }
    if (u.final_ptr) {
#pragma unroll
        for (int i = 0; i < 16; ++i) u.final_ptr[(int64_t)(c0 + i) * kD + j0 + j] = st[i];
    }
}

// kPre: the fused prologue is compiled in (only the *_preact calls launch it;
// the plain kernel carries none of its code, which matters for instruction
// fetch).
template <bool kPre>
__global__ void __launch_bounds__(kThreadsTC, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                const __grid_constant__ CUtensorMap map_b, const __grid_constant__ CUtensorMap map_v,
                const __grid_constant__ CUtensorMap map_la, const __grid_constant__ CUtensorMap map_w,
                TcParams prm)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    // Align to 1024 B by offsetting the __shared__ array itself (not through an
    // integer round trip), so every access below stays a shared-space access.
    // Both CTAs of the cluster get the same offsets.
    unsigned char *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBAR);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kMISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kMISC + 4);
    uint32_t *copy_count = reinterpret_cast<uint32_t *>(smem + kMISC + 8);  // helper: [F0 F1 P0 P1 T0 T1]
    // set (in both CTAs of the pair) once a chunk's decay leaves the factors' range
    volatile int *range_flag = reinterpret_cast<volatile int *>(smem + kMISC + kRangeFlagOff);

    // Cluster ranks [0, kPairs) are the main CTAs of kPairs units, ranks
    // [kPairs, 2 kPairs) their helpers (so that CTAs running the same code
    // share a TPC); unit sub of the cluster is served by ranks sub, kPairs + sub.
    const uint32_t rank = cluster_ctarank();
    const bool is_main = rank < (uint32_t)kPairs;
    const uint32_t peer = is_main ? rank + kPairs : rank - kPairs;
    const uint32_t peer_abort = mapa_shared(sbase + kMISC + 4, peer);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t H = prm.H;
    const UnitJob job = unit_job(prm, blockIdx.x, rank);
    const bool valid = job.valid;
    const int64_t h = job.h, t_begin = job.t_begin, t_end = job.t_end;
    const bool zero_v = job.zero_v;
    const float *init_ptr = job.init_ptr;
    float *final_ptr = job.final_ptr;
    const int nc = (int)((t_end - t_begin + 63) / 64);

    if (nc == 0) {
        // empty sequence (both CTAs of the pair are here): the final state is
        // the initial state; then only the cluster's three barriers are joined
        if (valid && is_main && final_ptr)
            for (int i = tid; i < kD * kD; i += kThreadsTC)
                final_ptr[i] = init_ptr ? init_ptr[i] : 0.f;
        cluster_sync_all();
        cluster_sync_all();
        cluster_sync_all();
        return;
    }

    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(&bars[i], 1);
        if (!is_main) {
            // q, k, b slot: freed by the [A^T | P^T] MMAs and by the main CTA having
            // received the factors; X columns: freed by both readout groups
            mbar_init(&bars[H_SLOTFREE0], 2);
            mbar_init(&bars[H_SLOTFREE1], 2);
            mbar_init(&bars[H_XFREE0], 2);
            mbar_init(&bars[H_XFREE1], 2);
        }
        *abort_flag = 0;
        *range_flag = 0;
        for (int i = 0; i < 6; ++i) copy_count[i] = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        if (is_main) {
            prefetch_tensormap(&map_v); prefetch_tensormap(&map_w);
        } else {
            prefetch_tensormap(&map_q); prefetch_tensormap(&map_k); prefetch_tensormap(&map_b);
            prefetch_tensormap(&map_la);
        }
    }
    if (warp == 2) {
        tmem_alloc(tmem_slot, is_main ? 512 : 256);
        tmem_relinquish();
    }
    tc_fence_before();
    cluster_sync_all();  // barriers of both CTAs initialised before any remote access
    tc_fence_after();
    const uint32_t tb = *tmem_slot;

    if (is_main) {
    // =========================================================================
    //                               main CTA
    // =========================================================================
    if (warp < 4) {
    setmaxnreg_dec40();
    if (warp == 0) {
        // ------------- v and w tiles, slot-free relay ------------------------
        if (lane == 0) {
            const uint32_t h_mfree = mapa_shared(smem_u32(&bars[H_MFREE0]), peer);
            int vissued0 = 0, vissued1 = 0;  // loads issued into each slot
            int wissued = 0;
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1;
                if (!zero_v) {  // (an identity run with z = 0 loads neither)
                    if (c >= 2 && !wait_bar(&bars[M_VFREE0 + s], ((c >> 1) - 1) & 1, abort_flag, peer_abort, 1))
                        break;
                    const int z = (int)(t_begin + 64 * c);
                    mbar_arrive_expect_tx(&bars[M_VFULL0 + s], 16384);
                    for (int blk = 0; blk < 2; ++blk)
                        tma_load_3d(smem + mZ(s) + blk * 8192, &map_v, &bars[M_VFULL0 + s], 64 * blk, (int)h, z);
                    (s ? vissued1 : vissued0) = (c >> 1) + 1;
                    // the single w buffer: free once Z of chunk c-1 is done
                    if (c >= 1 && !wait_bar(&bars[M_WTFREE], (c - 1) & 1, abort_flag, peer_abort, 4)) break;
                    mbar_arrive_expect_tx(&bars[M_WTFULL], 16384);
                    for (int blk = 0; blk < 2; ++blk)
                        tma_load_3d(smem + kM_WT + blk * 8192, &map_w, &bars[M_WTFULL], 64 * blk, (int)h, z);
                    ++wissued;
                }
                // slot s of chunk c - 2 fully consumed (its last MMA is done):
                // the helper may copy chunk c into it
                if (c >= 2) {
                    if (!wait_bar(&bars[M_SLOTFREE0 + s], ((c >> 1) - 1) & 1, abort_flag, peer_abort, 2)) break;
                    mbar_remote_arrive(h_mfree + 8 * s);
                }
            }
            if (vissued0 > 0) drain_wait(&bars[M_VFULL0], (vissued0 - 1) & 1, 20);
            if (vissued1 > 0) drain_wait(&bars[M_VFULL1], (vissued1 - 1) & 1, 20);
            if (wissued > 0) drain_wait(&bars[M_WTFULL], (wissued - 1) & 1, 21);
        }
    } else if (warp == 1) {
        // ------------- MMA issuer: W = T Em, U0^T = Z^T T^T --------------------
        if (lane == 0) {
            const uint32_t i_w = idesc_bf16_f32(64, 64, false, true, true);  // -(T Em)
            const uint32_t i_u = idesc_bf16_f32(128, 64, true, false);
            const uint64_t d_t = smem_desc_sw128(sbase + mT(0), 16, 1024);
            const uint64_t d_em = smem_desc_sw128(sbase + mEQ(0), 16384, 1024);
            const uint64_t d_z = smem_desc_sw128(sbase + mZ(0), 8192, 1024);
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1;
                const uint64_t dt = desc_at(d_t, mT(s) - mT(0)), dem = desc_at(d_em, mEQ(s) - mEQ(0));
                const uint64_t dz = desc_at(d_z, mZ(s) - mZ(0));
                if (!wait_bar(&bars[M_F0 + s], (c >> 1) & 1, abort_flag, peer_abort, 12)) break;
                if (!wait_bar(&bars[M_T0 + s], (c >> 1) & 1, abort_flag, peer_abort, 13)) break;
                if (!wait_bar(&bars[M_ZREADY0 + s], (c >> 1) & 1, abort_flag, peer_abort, 14)) break;
                // the U columns are free once the epilogue has converted chunk c-1's U;
                // the W columns once chunk c-1's -W has been read out
                if (c >= 1 && !wait_bar(&bars[M_UCONV], (c - 1) & 1, abort_flag, peer_abort, 15)) break;
                if (c >= 1 && !wait_bar(&bars[M_WFREE], (c - 1) & 1, abort_flag, peer_abort, 16)) break;
                // (T arrived by the helper's generic-proxy stores; the MMAs read it through
                // the async proxy)
                fence_proxy_async_smem();
                tc_fence_after();
                // -W rows r (M = 64, A negated): key channels of block kb -> lanes 16 kb .. 16 kb + 15
#pragma unroll
                for (int kb = 0; kb < 2; ++kb)
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ss(tb + kTmW + ((uint32_t)(16 * kb) << 16), desc_at(dt, kk * 32),
                               desc_at(dem, kb * 16384 + kk * 2048), i_w, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ss(tb + kTmU, desc_at(dz, kk * 2048), desc_at(dt, kk * 32), i_u, kk > 0);
                tc_commit(&bars[M_WDONE]);
                tc_commit(&bars[M_VFREE0 + s]);
            }
            tc_commit(&bars[M_DRAIN]);
            drain_wait(&bars[M_DRAIN], 0, 22);
        }
    } else if (warp == 2) {
        // ------------- relay: the helper's q, k, b slot may be reloaded ---------
        // (its factors have landed here; only chunks the helper reloads after)
        if (lane == 0) {
            const uint32_t h_slotfree = mapa_shared(smem_u32(&bars[H_SLOTFREE0]), peer);
            for (int c = 0; c + 2 < nc; ++c) {
                const int s = c & 1;
                if (!wait_bar(&bars[M_F0 + s], (c >> 1) & 1, abort_flag, peer_abort, 3)) break;
                mbar_remote_arrive(h_slotfree + 8 * s);
            }
        }
    } else {
        // ------------- MMA issuer: the state chain -----------------------------
        if (lane == 0) {
            const uint32_t i_uo = idesc_bf16_f32(128, 128, false, false);
            const uint32_t i_os = idesc_bf16_f32(128, 192, false, true);
            const uint64_t d_wq = smem_desc_sw128(sbase + mEQ(0), 16, 1024);
            const uint64_t d_pk = smem_desc_sw128(sbase + mKB(0), 8192, 1024);
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1;
                const uint64_t dwq = desc_at(d_wq, mEQ(s) - mEQ(0)), dpk = desc_at(d_pk, mKB(s) - mKB(0));
                if (!spin_bar(&bars[M_WREADY0 + s], (c >> 1) & 1, abort_flag, peer_abort, 17)) break;
                if (!spin_bar(&bars[M_SREADY_LO], c & 1, abort_flag, peer_abort, 18)) break;
                // (the O^T columns have been read out and cleared after chunk c-1)
                if (c >= 1 && !spin_bar(&bars[M_OZERO], (c - 1) & 1, abort_flag, peer_abort, 29)) break;
                tc_fence_after();
                // [U^T | O^T] += Sm^T [-W ; Qm]^T   (N = 128: -W rows then Qm rows); the
                // state arrives in two halves of 64 key channels (K steps 0-3, 4-7)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tb + kTmU, tb + kTmSB + kk * 8, desc_at(dwq, (kk & 3) * 32), i_uo, 1);
                if (!spin_bar(&bars[M_SREADY_HI], c & 1, abort_flag, peer_abort, 24)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 4; kk < 8; ++kk)
                    mma_ts(tb + kTmU, tb + kTmSB + kk * 8, desc_at(dwq, 16384 + (kk & 3) * 32), i_uo, 1);
                tc_commit(&bars[M_UDONE]);
                if (!spin_bar(&bars[M_UCONV], c & 1, abort_flag, peer_abort, 19)) break;
                if (!spin_bar(&bars[M_P0 + s], (c >> 1) & 1, abort_flag, peer_abort, 25)) break;
                tc_fence_after();
                // [O^T | M^T] += U^T [P^T | Km]   (N = 192, B MN-major: P^T atom, two Km atoms)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_ts(tb + kTmO, tb + kTmUB + kk * 8, desc_at(dpk, kk * 2048), i_os, 1);
                tc_commit(&bars[M_SDONE]);
                tc_commit(&bars[M_SLOTFREE0 + s]);
            }
            tc_commit(&bars[M_DRAIN2]);
            drain_wait(&bars[M_DRAIN2], 0, 23);
        }
    }
    } else if (warp < 8) {
        setmaxnreg_inc152();
        // ------------- Z = w . v, in place over the v tile ---------------------
        // Lane g owns value channels 4g..4g+3 (64-channel block g / 16), warp pw
        // rows 16pw..16pw+15; rows past the chunk end are zeroed. Iteration c also
        // takes chunk c-1's O^T out of TMEM (below), one chunk behind the Z tiles,
        // which run far ahead of the state chain.
        const int pw = warp - 4, tp = tid - 128;
        const int g = lane, kb = g >> 4;
        const uint32_t cbyte = 8 * (g & 15);
        const int jo = 32 * pw + lane;                        // value channel = TMEM lane
        const uint32_t lane_o = (uint32_t)(32 * pw) << 16;
        __nv_bfloat16 *obase = zero_v ? prm.psi : prm.o;  // (an identity run writes psi)
        // O^T of chunk cc: rows (tokens) of value channel jo as bf16 pairs, the
        // columns cleared for the next chunk (M_OZERO), then o through the staging
        // tile: adjacent lanes (channels j, j+1) trade halves so that the even
        // lane writes rows 2q and the odd lane rows 2q+1 as 4-byte (j, j+1)
        // pairs, and every row leaves in 16-byte pieces; rows past the sequence
        // end are not written
        auto o_out = [&](int cc) -> bool {
            if (!group_and(kBarZ, 128, wait_bar(&bars[M_SDONE], cc & 1, abort_flag, peer_abort, 30))) return false;
            tc_fence_after();
            uint32_t opk[32];
            {
                uint32_t v0[32], v1[32];
                tmem_ld32(tb + kTmO + lane_o, v0);
                tmem_ld32(tb + kTmO + lane_o + 32, v1);
                tc_wait_ld();
#pragma unroll
                for (int q = 0; q < 16; ++q) {
                    opk[q] = pack_bf16x2(__uint_as_float(v0[2 * q]), __uint_as_float(v0[2 * q + 1]));
                    opk[16 + q] = pack_bf16x2(__uint_as_float(v1[2 * q]), __uint_as_float(v1[2 * q + 1]));
                }
            }
            if (cc + 1 < nc) {
                const uint32_t zeros[32] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u,
                                            0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
                tmem_st32(tb + kTmO + lane_o, zeros);
                tmem_st32(tb + kTmO + lane_o + 32, zeros);
                tc_wait_st();
            }
            tc_fence_before();
            named_bar_sync(kBarZ, 128);
            if (tp == 0) mbar_arrive(&bars[M_OZERO]);
            {
                const bool odd = (lane & 1) != 0;
                unsigned char *ost = smem + kM_OST + 2 * (jo & ~1);
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const uint32_t mine = opk[q];                       // rows (2q, 2q+1) of channel jo
                    const uint32_t other = __shfl_xor_sync(0xffffffffu, mine, 1);
                    // even lane: (row 2q: j, j+1); odd lane: (row 2q+1: j-1, j)
                    const uint32_t pr = odd ? __byte_perm(other, mine, 0x7632) : __byte_perm(mine, other, 0x5410);
                    const int r = 2 * q + (odd ? 1 : 0);
                    *reinterpret_cast<uint32_t *>(ost + r * kOPitch) = pr;
                }
            }
            named_bar_sync(kBarZ, 128);
            const int64_t t0 = t_begin + 64 * cc;
            const int L = (int)(t_end - t0 < 64 ? t_end - t0 : 64);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int idx = tp + 128 * i, r = idx >> 4, piece = idx & 15;
                if (r < L) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(smem + kM_OST + r * kOPitch + 16 * piece);
                    *reinterpret_cast<uint4 *>(obase + ((t0 + r) * H + h) * kD + 8 * piece) = v;
                }
            }
            // (the staging tile is written again only after the group barrier of
            // the next SDONE wait)
            return true;
        };
        for (int c = 0; c <= nc; ++c) {
            const int s = c & 1;
            if (c < nc && zero_v) {
                // Z = 0: clear the slot once its previous U0 MMA is done (that wait
                // also paces the hand-offs, one phase per chunk and slot)
                if (!group_and(kBarZ, 128, c < 2 || wait_bar(&bars[M_VFREE0 + s], ((c >> 1) - 1) & 1, abort_flag,
                                                               peer_abort, 5)))
                    break;
                if (c < 2) {
                    uint4 *zt = reinterpret_cast<uint4 *>(smem + mZ(s));
                    for (int i = tp; i < 16384 / 16; i += 128) zt[i] = make_uint4(0u, 0u, 0u, 0u);
                    fence_proxy_async_smem();
                }
                named_bar_sync(kBarZ, 128);
                if (tp == 0) mbar_arrive(&bars[M_ZREADY0 + s]);
            } else if (c < nc) {
                const int64_t t0 = t_begin + 64 * c;
                const int L = (int)(t_end - t0 < 64 ? t_end - t0 : 64);
                if (!group_and(kBarZ, 128, wait_bar(&bars[M_VFULL0 + s], (c >> 1) & 1, abort_flag, peer_abort, 5) &&
                                               wait_bar(&bars[M_WTFULL], c & 1, abort_flag, peer_abort, 6)))
                    break;
                unsigned char *z_tile = smem + mZ(s) + kb * 8192;
                const unsigned char *w_tile = smem + kM_WT + kb * 8192;
#pragma unroll 4
                for (int i = 0; i < 16; ++i) {
                    const int r = 16 * pw + i;
                    const uint32_t off = sw128_offset(r, cbyte);
                    const uint2 vr = *reinterpret_cast<const uint2 *>(z_tile + off);
                    const uint2 wr = *reinterpret_cast<const uint2 *>(w_tile + off);
                    const float2 v0 = bf2_to_f2(vr.x), v1 = bf2_to_f2(vr.y);
                    float2 w0 = bf2_to_f2(wr.x), w1 = bf2_to_f2(wr.y);
                    if (kPre && (prm.pre & GDR2_PROLOGUE_GATE_SIGMOID)) {
                        w0 = make_float2(pre_sigmoid(w0.x), pre_sigmoid(w0.y));
                        w1 = make_float2(pre_sigmoid(w1.x), pre_sigmoid(w1.y));
                    }
                    const bool ok = r < L;
                    uint2 oz;
                    oz.x = ok ? pack_bf16x2(v0.x * w0.x, v0.y * w0.y) : 0u;
                    oz.y = ok ? pack_bf16x2(v1.x * w1.x, v1.y * w1.y) : 0u;
                    *reinterpret_cast<uint2 *>(z_tile + off) = oz;
                }
                fence_proxy_async_smem();
                named_bar_sync(kBarZ, 128);
                if (tp == 0) {
                    mbar_arrive(&bars[M_ZREADY0 + s]);
                    mbar_arrive(&bars[M_WTFREE]);
                }
            }
            if (c >= 1 && !o_out(c - 1)) break;
        }
    } else if (warp < 12) {
        setmaxnreg_inc152();
        // ------------- -W, K-major, over the Em half of the slot -------------
        // Warp pw reads its lane quarter of the -W columns: lane i < 16 holds row
        // r = 16 pw + i for key channels 0-63, lane 16 + i the same row for 64-127.
        const int pw = warp - 8, tp = tid - 256;
        const int rrow = 16 * pw + (lane & 15), kb = lane >> 4;
        const uint32_t h_tfree = mapa_shared(smem_u32(&bars[H_TFREE0]), peer);
        for (int c = 0; c < nc; ++c) {
            const int s = c & 1;
            if (!group_and(kBarW, 128, wait_bar(&bars[M_WDONE], c & 1, abort_flag, peer_abort, 8))) break;
            // the W and U0 MMAs have read T: the helper may send chunk c + 2's T
            // (only chunks the helper still sends wait for this)
            if (tp == 0 && c + 2 < nc) mbar_remote_arrive(h_tfree + 8 * s);
            tc_fence_after();
            uint32_t v0[32], v1[32];
            const uint32_t taddr = tb + kTmW + ((uint32_t)(32 * pw) << 16);
            tmem_ld32(taddr, v0);
            tmem_ld32(taddr + 32, v1);
            tc_wait_ld();
            tc_fence_before();
            float x[64];
#pragma unroll
            for (int j2 = 0; j2 < 32; ++j2) {
                x[j2] = __uint_as_float(v0[j2]);
                x[32 + j2] = __uint_as_float(v1[j2]);
            }
            store_row_bf16_sw128(smem + mEQ(s) + kb * 16384, rrow, x);
            fence_proxy_async_smem();
            named_bar_sync(kBarW, 128);
            if (tp == 0) {
                mbar_arrive(&bars[M_WFREE]);
                mbar_arrive(&bars[M_WREADY0 + s]);
            }
        }
    } else {
        setmaxnreg_inc152();
        // ------------- epilogue ---------------------------------------------
        const int ew = warp - 12, te = tid - 384;
        const int j = 32 * ew + lane;                       // value channel = TMEM lane
        const uint32_t lane_off = (uint32_t)(32 * ew) << 16;
        float *vecF = reinterpret_cast<float *>(smem + kM_VECF);
        // Range of the chunk form on key channel j, checked on the half sums that
        // also give the state's chunk-to-chunk factor (log alpha <= 0, so g falls
        // monotonically and T0 = g_31, T1 = g_63 - g_31 bound every |g_r - g_31|):
        // each half within kFactorRange, and T1(c) + T0(c+1), the exponent of
        // that factor, within kWindowRange. Past either, the pair recomputes the
        // whole unit exactly, token by token, after this pass (serial_unit).
        const uint32_t peer_range_flag = mapa_shared(sbase + kMISC + kRangeFlagOff, peer);
        auto out_of_range = [&]() {
            *range_flag = 1;
            st_cluster_u32(peer_range_flag, 1u);
        };
        const uint32_t zeros[32] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u,
                                    0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        bool ok = true;
        // master = Diag(e^{g_31 of chunk 0}) S0  (transposed: row j over key channels); O = 0
        ok = group_and(kBarEpi, 128, wait_bar(&bars[M_F0], 0, abort_flag, peer_abort, 9));
        if (ok) {
            const float t00 = reinterpret_cast<const float *>(smem + mVEC(0))[j];
            vecF[j] = expf(t00);
            if (t00 < -kFactorRange) out_of_range();
            named_bar_sync(kBarEpi, 128);
#pragma unroll
            for (int g4 = 0; g4 < 4; ++g4) {
                uint32_t m[32], sbf[16];
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const int ch = 32 * g4 + q;
                    const float s0 = init_ptr ? init_ptr[(int64_t)ch * kD + j] : (zero_v && ch == j ? 1.f : 0.f);
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
            if (te == 0) {
                mbar_arrive(&bars[M_SREADY_LO]);
                mbar_arrive(&bars[M_SREADY_HI]);
            }
        }
        bool chain_done = false;  // the last chunk's hand-off has completed
        for (int c = 0; ok && c < nc; ++c) {
            const int s = c & 1;
            const int64_t t0 = t_begin + 64 * c;
            const int L = (int)(t_end - t0 < 64 ? t_end - t0 : 64);
            // this chunk's second half sum (read now: the slot is refilled once
            // the chunk's last MMA is done; the asm below makes the load complete
            // before this thread passes the U hand-off that precedes that MMA)
            float t1c = reinterpret_cast<const float *>(smem + mVEC(s))[128 + j];
            asm volatile("mov.b32 %0, %0;" : "+f"(t1c));
            const bool last = (c + 1 == nc);
            // U^T (fp32) -> bf16 pairs in TMEM for the update MMAs
            if (!group_and(kBarEpi, 128, wait_bar(&bars[M_UDONE], c & 1, abort_flag, peer_abort, 10))) break;
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
                mbar_arrive(&bars[M_UCONV]);
            }
            // state scale for this chunk's hand-off, e^{g_C - g_31} and, unless last,
            // e^{g'_31} of the next chunk (its slot is not refilled before this
            // chunk's state has been handed off); the last readers of vecF finished
            // before the previous chunk's final group barrier, and the group
            // barrier of the SDONE wait below publishes the new factors
            if (!group_and(kBarEpi, 128,
                           last || wait_bar(&bars[M_F0 + (s ^ 1)], ((c + 1) >> 1) & 1, abort_flag, peer_abort, 26)))
                break;
            const float t0n = last ? 0.f : reinterpret_cast<const float *>(smem + mVEC(s ^ 1))[j];
            vecF[j] = expf(t1c + t0n);
            if (t1c < -kFactorRange || t0n < -kFactorRange || t1c + t0n < -kWindowRange) out_of_range();

            if (!group_and(kBarEpi, 128, wait_bar(&bars[M_SDONE], c & 1, abort_flag, peer_abort, 11))) break;
            tc_fence_after();
            // the state, scaled, in two halves of 64 key channels: each half is
            // handed to the chain as soon as its bf16 copy is in TMEM
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
                    tmem_st16(tb + kTmSB + lane_off + 32 * hh, s0b);
                    tmem_st16(tb + kTmSB + lane_off + 32 * hh + 16, s1b);
                    tc_wait_st();
                    tc_fence_before();
                    named_bar_sync(kBarEpi, 128);
                    if (te == 0) mbar_arrive(&bars[hh ? M_SREADY_HI : M_SREADY_LO]);
                    // (the master below is first read again by the next chunk's update
                    // MMAs, which wait for the U hand-off, whose tc_wait_st covers it)
                }
                // the fp32 master: after the last chunk it is the final state, which
                // is written out after the loop (off the per-chunk code)
                tmem_st32(tb + kTmMaster + lane_off + 64 * hh, m0);
                tmem_st32(tb + kTmMaster + lane_off + 64 * hh + 32, m1);
            }
            if (last) chain_done = true;
        }
        tc_wait_st();  // (a master write-back may still be in flight after an abort)
        if (chain_done && final_ptr) {
            // final state, key channel ch (row) x value channel j: 32 key channels
            // per TMEM load, each store coalesced over the warp's value channels
#pragma unroll 1
            for (int g4 = 0; g4 < 4; ++g4) {
                uint32_t m[32];
                tmem_ld32(tb + kTmMaster + lane_off + 32 * g4, m);
                tc_wait_ld();
#pragma unroll
                for (int q = 0; q < 32; ++q) final_ptr[(int64_t)(32 * g4 + q) * kD + j] = __uint_as_float(m[q]);
            }
        }
    }
    } else {
    // =========================================================================
    //                              helper CTA
    // =========================================================================
    if (warp < 4) {
    setmaxnreg_dec40();
    if (warp == 0) {
        // ------------- q, k, b tiles ---------------------------------------------
        if (lane == 0) {
            int issued0 = 0, issued1 = 0;  // loads issued into each slot
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1;
                if (c >= 2 &&
                    !wait_bar(&bars[H_SLOTFREE0 + s], ((c >> 1) - 1) & 1, abort_flag, peer_abort, 1))
                    break;
                const int z = (int)(t_begin + 64 * c);
                unsigned char *eq = smem + hEQ(s), *kq = smem + hEQ(s) + kH_KmOff;
                mbar_arrive_expect_tx(&bars[H_FULL0 + s], 3 * 16384);
                for (int blk = 0; blk < 2; ++blk) {
                    tma_load_3d(eq + blk * 16384, &map_b, &bars[H_FULL0 + s], 64 * blk, (int)h, z);
                    tma_load_3d(eq + blk * 16384 + 8192, &map_q, &bars[H_FULL0 + s], 64 * blk, (int)h, z);
                    tma_load_3d(kq + blk * 8192, &map_k, &bars[H_FULL0 + s], 64 * blk, (int)h, z);
                }
                (s ? issued1 : issued0) = (c >> 1) + 1;
            }
            if (issued0 > 0) drain_wait(&bars[H_FULL0], (issued0 - 1) & 1, 20);
            if (issued1 > 0) drain_wait(&bars[H_FULL1], (issued1 - 1) & 1, 20);
        }
    } else if (warp == 1) {
        // ------------- MMA issuer: [A^T | P^T] = Km [Em; Qm]^T ---------------
        if (lane == 0) {
            const uint32_t i_ap = idesc_bf16_f32(64, 128, false, false);
            const uint64_t d_km = smem_desc_sw128(sbase + hEQ(0) + kH_KmOff, 16, 1024);
            const uint64_t d_eq = smem_desc_sw128(sbase + hEQ(0), 16, 1024);
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1;
                const uint64_t dkm = desc_at(d_km, hEQ(s) - hEQ(0)), deq = desc_at(d_eq, hEQ(s) - hEQ(0));
                if (!wait_bar(&bars[H_FDONE], c & 1, abort_flag, peer_abort, 12)) break;
                if (c >= 2 && !wait_bar(&bars[H_XFREE0 + s], ((c >> 1) - 1) & 1, abort_flag, peer_abort, 13))
                    break;
                tc_fence_after();
                // M = 64 rows s (lanes 0-15 of each quarter), N = 128: Em rows, then Qm rows
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_ss(tb + 128 * s, desc_at(dkm, (kk >> 2) * 8192 + (kk & 3) * 32),
                           desc_at(deq, (kk >> 2) * 16384 + (kk & 3) * 32), i_ap, kk > 0);
                tc_commit(&bars[H_AP0 + s]);
                tc_commit(&bars[H_SLOTFREE0 + s]);
            }
            tc_commit(&bars[H_DRAIN]);
            drain_wait(&bars[H_DRAIN], 0, 22);
        }
    } else if (warp == 2) {
        // ------------- factor sender: Em, Qm, Km, half sums -> main CTA ------
        // (the main CTA's slot s is free once its chunk c-2 is fully consumed)
        if (lane == 0) {
            // (one CTA's window of the cluster's shared space is contiguous)
            const uint32_t rbase = mapa_shared(sbase, peer);
            for (int c = 0; c < nc; ++c) {
                const int s = c & 1;
                if (!wait_bar(&bars[H_FDONE], c & 1, abort_flag, peer_abort, 14)) break;
                if (c >= 2 && !wait_bar(&bars[H_MFREE0 + s], ((c >> 1) - 1) & 1, abort_flag, peer_abort, 15))
                    break;
                const uint32_t bar = rbase + kBAR + 8 * (M_F0 + s);
                mbar_remote_arrive_expect_tx(bar, kFBytes);
                bulk_copy_to_cluster(rbase + mEQ(s), sbase + hEQ(s), 32768, bar);
                bulk_copy_to_cluster(rbase + mKB(s) + kKmOff, sbase + hEQ(s) + kH_KmOff, 16384, bar);
                bulk_copy_to_cluster(rbase + mVEC(s), sbase + hVEC(s), 1024, bar);
                copy_count[s] += 1;
            }
        }
    }
    } else if (warp < 12) {
        setmaxnreg_inc152();
        // ------------- decay factors, P^T (256 threads) ----------------------
        // Element-wise layout: lane g owns key channels 4g..4g+3 (64-channel
        // block kb = g / 16), warp pw owns rows 8pw..8pw+7. Rows past the chunk
        // end are zeroed with selects. Software-pipelined: iteration c computes
        // chunk c's factors and then reads out chunk c-1's P^T, so that the
        // [A^T | P^T] MMA of a chunk runs while the next chunk's factors are
        // computed.
        const int pw = warp - 4, tp = tid - 128;
        const int g = lane, kb = g >> 4;
        const uint32_t cbyte = 8 * (g & 15);
        constexpr float kLog2e = 1.4426950408889634f;
        const float *la_s = reinterpret_cast<const float *>(smem + kH_LA);  // staged log_alpha [64][128]
        float *vecBS = reinterpret_cast<float *>(smem + kH_BSUM);          // [8][128]
        const uint32_t m_p = mapa_shared(smem_u32(&bars[M_P0]), peer);
        int la_issued = 0;  // log_alpha tiles staged so far (thread tp == 0)
        if (tp == 0) {
            ++la_issued;
            mbar_arrive_expect_tx(&bars[H_LAFULL], 32768);
            tma_load_3d(smem + kH_LA, &map_la, &bars[H_LAFULL], 0, (int)h, (int)t_begin);
        }
        for (int c = 0; c <= nc; ++c) {
            const int s = c & 1;
            const int64_t t0 = t_begin + 64 * c;
            const int L = (int)(t_end - t0 < 64 ? t_end - t0 : 64);
            if (c < nc) {
            unsigned char *e_tile = smem + hEQ(s) + kb * 16384;
            unsigned char *q_tile = e_tile + 8192;
            unsigned char *k_tile = smem + hEQ(s) + kH_KmOff + kb * 8192;

            if (!group_and(kBarPrepA, 256, wait_bar(&bars[H_LAFULL], c & 1, abort_flag, peer_abort, 3))) break;
            float4 la[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = 8 * pw + i;
                float4 x = *reinterpret_cast<const float4 *>(la_s + r * 128 + 4 * g);
                if (kPre && (prm.pre & GDR2_PROLOGUE_DECAY_SOFTPLUS))
                    x = make_float4(pre_neg_softplus(x.x), pre_neg_softplus(x.y), pre_neg_softplus(x.z),
                                    pre_neg_softplus(x.w));
                la[i] = r < L ? x : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            float4 bs = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                bs.x += la[i].x; bs.y += la[i].y; bs.z += la[i].z; bs.w += la[i].w;
            }
            *reinterpret_cast<float4 *>(vecBS + pw * 128 + 4 * g) = bs;
            // (this group barrier also publishes the block sums and frees the staging tile)
            fence_proxy_async_smem();
            if (!group_and(kBarPrepA, 256, wait_bar(&bars[H_FULL0 + s], (c >> 1) & 1, abort_flag, peer_abort, 4)))
                break;
            if (tp == 0) {
                if (c + 1 < nc) {  // stage the next chunk's log_alpha
                    ++la_issued;
                    mbar_arrive_expect_tx(&bars[H_LAFULL], 32768);
                    tma_load_3d(smem + kH_LA, &map_la, &bars[H_LAFULL], 0, (int)h, (int)(t0 + 64));
                }
            }
            // d_r = g_r - g_31 in log2 units: suffix sums for rows < 32, prefix
            // sums for rows >= 32; half sums T0 = g_31, T1 = g_63 - g_31.
            {
                float4 run = make_float4(0.f, 0.f, 0.f, 0.f), half = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int b = 0; b < 8; ++b) {
                    const float4 o4 = *reinterpret_cast<const float4 *>(vecBS + b * 128 + 4 * g);
                    const bool in_run = pw < 4 ? (b > pw && b < 4) : (b >= 4 && b < pw);
                    const bool in_half = pw < 4 ? b < 4 : b >= 4;
                    if (in_run) { run.x += o4.x; run.y += o4.y; run.z += o4.z; run.w += o4.w; }
                    if (in_half) { half.x += o4.x; half.y += o4.y; half.z += o4.z; half.w += o4.w; }
                }
                if (pw == 0 || pw == 4)
                    *reinterpret_cast<float4 *>(smem + hVEC(s) + (pw == 0 ? 0 : 512) + 16 * g) = half;
                if (pw < 4) {
#pragma unroll
                    for (int i = 7; i >= 0; --i) {
                        const float4 x = la[i];
                        la[i] = make_float4(-run.x * kLog2e, -run.y * kLog2e, -run.z * kLog2e, -run.w * kLog2e);
                        run.x += x.x; run.y += x.y; run.z += x.z; run.w += x.w;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        run.x += la[i].x; run.y += la[i].y; run.z += la[i].z; run.w += la[i].w;
                        la[i] = make_float4(run.x * kLog2e, run.y * kLog2e, run.z * kLog2e, run.w * kLog2e);
                    }
                }
            }
            // prologue: 1 / ||q_r||, 1 / ||k_r|| (a warp holds whole rows: lanes
            // 0-15 key channels 0-63, lanes 16-31 channels 64-127)
            float qs[8], ks[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) qs[i] = ks[i] = 1.f;
            if (kPre && (prm.pre & GDR2_PROLOGUE_QK_L2NORM)) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t off = sw128_offset(8 * pw + i, cbyte);
                    const uint2 qr = *reinterpret_cast<const uint2 *>(q_tile + off);
                    const uint2 kr = *reinterpret_cast<const uint2 *>(k_tile + off);
                    const float2 q0 = bf2_to_f2(qr.x), q1 = bf2_to_f2(qr.y);
                    const float2 k0 = bf2_to_f2(kr.x), k1 = bf2_to_f2(kr.y);
                    qs[i] = q0.x * q0.x + q0.y * q0.y + q1.x * q1.x + q1.y * q1.y;
                    ks[i] = k0.x * k0.x + k0.y * k0.y + k1.x * k1.x + k1.y * k1.y;
                }
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1)
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        qs[i] += __shfl_xor_sync(0xffffffffu, qs[i], m);
                        ks[i] += __shfl_xor_sync(0xffffffffu, ks[i], m);
                    }
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    qs[i] = rsqrtf(qs[i] + 1e-6f);
                    ks[i] = rsqrtf(ks[i] + 1e-6f);
                }
            }
            const bool gate_sig = kPre && (prm.pre & GDR2_PROLOGUE_GATE_SIGMOID) != 0;
            // factors, in place: b -> Em, q -> Qm, k -> Km
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int r = 8 * pw + i;
                const uint32_t off = sw128_offset(r, cbyte);
                const uint2 qr = *reinterpret_cast<const uint2 *>(q_tile + off);
                const uint2 kr = *reinterpret_cast<const uint2 *>(k_tile + off);
                const uint2 br = *reinterpret_cast<const uint2 *>(e_tile + off);
                float2 q0 = bf2_to_f2(qr.x), q1 = bf2_to_f2(qr.y);
                float2 k0 = bf2_to_f2(kr.x), k1 = bf2_to_f2(kr.y);
                float2 b0 = bf2_to_f2(br.x), b1 = bf2_to_f2(br.y);
                if constexpr (kPre) {
                    q0.x *= qs[i]; q0.y *= qs[i]; q1.x *= qs[i]; q1.y *= qs[i];
                    k0.x *= ks[i]; k0.y *= ks[i]; k1.x *= ks[i]; k1.y *= ks[i];
                }
                if (gate_sig) {
                    b0 = make_float2(pre_sigmoid(b0.x), pre_sigmoid(b0.y));
                    b1 = make_float2(pre_sigmoid(b1.x), pre_sigmoid(b1.y));
                }
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
            named_bar_sync(kBarPrepA, 256);
            if (tp == 0) {
                mbar_arrive(&bars[H_FDONE]);  // to the MMA issuer and the factor sender
            }
            }  // c < nc
            if (c == 0) continue;

            // P^T[s][r] = P[r][s] (kept for r >= s) of chunk cp = c - 1 from the M=64
            // accumulator: lane i < 16 of a warp in lane quarter q holds row
            // s = 16 q + i; the two warpgroups take the two 32-column halves
            const int cp = c - 1, sp = cp & 1;
            if (!group_and(kBarPrepA, 256, wait_bar(&bars[H_AP0 + sp], (cp >> 1) & 1, abort_flag, peer_abort, 6)))
                break;
            // the P^T buffers here and in the main CTA hold chunk cp-2 until the main
            // CTA has consumed it
            if (!group_and(kBarPrepA, 256,
                           cp < 2 || wait_bar(&bars[H_MFREE0 + sp], ((cp >> 1) - 1) & 1, abort_flag, peer_abort, 7)))
                break;
            tc_fence_after();
            {
                const int q4 = pw & 3, hf = pw >> 2;
                const uint32_t taddr = tb + 128 * sp + 64 + 32 * hf + ((uint32_t)(32 * q4) << 16);
                uint32_t v[32];
                tmem_ld32(taddr, v);
                tc_wait_ld();
                if (lane < 16) {
                    const int srow = 16 * q4 + lane;
                    unsigned char *pt = smem + hPT(sp);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t u[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int r0 = 32 * hf + 8 * q + 2 * e;
                            u[e] = pack_bf16x2(r0 >= srow ? __uint_as_float(v[8 * q + 2 * e]) : 0.f,
                                               r0 + 1 >= srow ? __uint_as_float(v[8 * q + 2 * e + 1]) : 0.f);
                        }
                        *reinterpret_cast<uint4 *>(pt + sw128_offset(srow, 64 * hf + 16 * q)) =
                            make_uint4(u[0], u[1], u[2], u[3]);
                    }
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(kBarPrepA, 256);
            if (tp == 0) {
                mbar_arrive(&bars[H_XFREE0 + sp]);
                if (!*abort_flag) {
                    const uint32_t bar = m_p + 8 * sp;
                    mbar_remote_arrive_expect_tx(bar, 8192);
                    bulk_copy_to_cluster(mapa_shared(sbase + mKB(sp), peer), sbase + hPT(sp), 8192, bar);
                    copy_count[2 + sp] += 1;
                }
            }
        }
        if (tp == 0 && la_issued > 0)  // drain a staged log_alpha load still in flight
            drain_wait(&bars[H_LAFULL], (la_issued - 1) & 1, 24);
    } else {
        setmaxnreg_inc152();
        // ------------- (I + A)^{-1} ----------------------------------------------
        const int pw = warp - 12, tp = tid - 384;
        float *sA = reinterpret_cast<float *>(smem + kH_SA);
        float *sT = reinterpret_cast<float *>(smem + kH_ST);
        const uint32_t m_t = mapa_shared(smem_u32(&bars[M_T0]), peer);
        for (int c = 0; c < nc; ++c) {
            const int s = c & 1;
            if (!group_and(kBarPrepB, 128, wait_bar(&bars[H_AP0 + s], (c >> 1) & 1, abort_flag, peer_abort, 8)))
                break;
            tc_fence_after();
            {   // A^T rows from the M=64 accumulator (lane i < 16 of warp pw: row s = 16 pw + i):
                // A^T[s][r] = A[r][s] for r > s
                const uint32_t taddr = tb + 128 * s + ((uint32_t)(32 * pw) << 16);
                // (entries with r <= s are left as computed: the solve below reads
                // only the strictly lower triangle of A)
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t v[32];
                    tmem_ld32(taddr + 32 * hf, v);
                    tc_wait_ld();
                    if (lane < 16) {
                        float *row = sA + (16 * pw + lane) * kLD + 32 * hf;
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            *reinterpret_cast<uint4 *>(row + 4 * q) =
                                make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    }
                }
            }
            tc_fence_before();
            named_bar_sync(kBarPrepB, 128);
            if (tp == 0) {
                mbar_arrive(&bars[H_XFREE0 + s]);
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
            // T into the bf16 buffer: its previous content (chunk c-2) has reached the
            // main CTA, and the main CTA's T buffer is free, once chunk c-2's W and U0
            // MMAs are done
            if (!group_and(kBarPrepB, 128,
                           c < 2 || wait_bar(&bars[H_TFREE0 + s], ((c >> 1) - 1) & 1, abort_flag,
                                                   peer_abort, 10)))
                break;
            {   // T (lower triangle incl. diagonal) -> bf16 MMA operand, stored straight into
                // the main CTA's T buffer; the 8 KB complete on its barrier
                const uint32_t bar = m_t + 8 * s;
                if (tp == 0) mbar_remote_arrive_expect_tx(bar, 8192);
                const uint32_t dst = mapa_shared(sbase + mT(s), peer);
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
                    st_async_v4(dst + sw128_offset(r, 64 * half + 16 * q), make_uint4(ue[0], ue[1], ue[2], ue[3]), bar);
                }
            }
            if (tp == 0) {
                copy_count[4 + s] += 1;
            }
        }
    }
    }

    // ---- teardown -----------------------------------------------------------
    tc_fence_before();
    cluster_sync_all();  // every copy and remote arrive of either CTA has been issued
    if (is_main && tid == 0) {
        // After an abort, copies from the helper may still be landing here: wait
        // (bounded) for the last one the helper issued into each buffer.
        const uint32_t cnt = mapa_shared(sbase + kMISC + 8, peer);
        for (int s = 0; s < 2; ++s) {
            const uint32_t n_f = ld_cluster_u32(cnt + 4 * s), n_p = ld_cluster_u32(cnt + 8 + 4 * s);
            const uint32_t n_t = ld_cluster_u32(cnt + 16 + 4 * s);
            if (n_f > 0) drain_wait(&bars[M_F0 + s], (n_f - 1) & 1, 27);
            if (n_p > 0) drain_wait(&bars[M_P0 + s], (n_p - 1) & 1, 27);
            if (n_t > 0) drain_wait(&bars[M_T0 + s], (n_t - 1) & 1, 28);
        }
    }
    cluster_sync_all();
    tc_fence_after();
    if (warp == 2) tmem_dealloc(tb, is_main ? 512 : 256);
    // a chunk's decay left the factors' range: recompute the unit exactly (this
    // CTA's half of the value columns; the chunk pass's o and state are replaced)
    // (the job is derived again from fresh reads of the CTA's coordinates, so
    // that none of the chunk pass's registers has to live until here)
    if (*range_flag && !*abort_flag) {  // (the same decision in every thread of the CTA)
        uint32_t cta;
        asm volatile("mov.u32 %0, %%ctaid.x;" : "=r"(cta));
        const uint32_t rk = cluster_ctarank();
        serial_unit<kPre>(prm, unit_job(prm, cta, rk), rk < (uint32_t)kPairs ? 0 : 64, smem, (int)threadIdx.x);
    }
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
    // two CTAs per job, kPairs pairs per cluster; 2 nseg - 1 jobs per (sequence, head)
    const int64_t units = a.num_seqs * a.H * (2 * (int64_t)a.nseg - 1);
    if (units == 0) return cudaSuccess;
    const int64_t clusters = (units + kPairs - 1) / kPairs;
    if (tokens > 0x7fffffffLL || 2 * kPairs * clusters > 0x7fffffffLL) return cudaErrorInvalidValue;
    CUtensorMap mq, mk, mb, mv, mla, mw;
    const int64_t tk = tokens > 0 ? tokens : 1;
    const void *dummy = a.q ? a.q : (const void *)a.o;
    bool ok = make_map(&mq, a.q ? a.q : dummy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tk, a.H, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&mk, a.k ? a.k : dummy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tk, a.H, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&mb, a.b ? a.b : dummy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tk, a.H, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&mv, a.v ? a.v : dummy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tk, a.H, 64, CU_TENSOR_MAP_SWIZZLE_128B) &&
              make_map(&mla, a.log_alpha ? (const void *)a.log_alpha : dummy, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, tk, a.H, 128, CU_TENSOR_MAP_SWIZZLE_NONE) &&
              make_map(&mw, a.w ? a.w : dummy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, tk, a.H, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (!ok) return cudaErrorInvalidValue;
    TcParams p;
    p.q = (const __nv_bfloat16 *)a.q;
    p.k = (const __nv_bfloat16 *)a.k;
    p.b = (const __nv_bfloat16 *)a.b;
    p.v = (const __nv_bfloat16 *)a.v;
    p.la = a.log_alpha;
    p.w = (const __nv_bfloat16 *)a.w;
    p.init_state = a.init_state;
    p.cu_seqlens = a.cu_seqlens;
    p.order = a.order;
    p.o = (__nv_bfloat16 *)a.o;
    p.final_state = a.final_state;
    p.T = a.T;
    p.H = a.H;
    p.tokens = tokens;
    p.units = units;
    p.nseg = a.nseg;
    p.seg_len = a.seg_len;
    p.pre = a.pre;
    unsigned char *ws = static_cast<unsigned char *>(a.seg_ws);
    p.psi = a.nseg > 1 ? reinterpret_cast<__nv_bfloat16 *>(ws + seg_psi_offset()) : nullptr;
    p.seg_s0 = a.nseg > 1 ? reinterpret_cast<float *>(ws + seg_state_offset(a.B, a.T, a.H)) : nullptr;
    p.seg_phi = a.nseg > 1 ? reinterpret_cast<float *>(ws + seg_phi_offset(a.B, a.T, a.H, a.nseg)) : nullptr;
    auto kernel = a.pre ? chunk_tc_kernel<true> : chunk_tc_kernel<false>;
    cudaError_t e = ensure_dynamic_smem((const void *)kernel, (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * kPairs * clusters), 1, 1);
    cfg.blockDim = dim3(kThreadsTC, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2 * kPairs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, mq, mk, mb, mv, mla, mw, p);
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
        WaitGuard g{timeout_ns, &abort_flag, &g_chunk_tc_error};
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
