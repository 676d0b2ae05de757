/*
 * gdr2.h -- C ABI of the B200 (sm_100a) Gated Delta Rule-2 operator library.
 *
 * The operator (Gated DeltaNet-2's sequence mixer). Per sequence and head the
 * recurrent state S is a d_k x d_v matrix and each token t updates it as
 *
 *     S_t = (I - k_t (b_t . k_t)^T) Diag(alpha_t) S_{t-1} + k_t (w_t . v_t)^T,
 *     o_t = S_t^T q_t,                       alpha_t = exp(log_alpha_t),
 *
 * where "." is the element-wise product, b_t in [0,1]^{d_k} is the erase gate
 * (key side) and w_t in [0,1]^{d_v} the write gate (value side). Sources:
 *   - "Gated DeltaNet-2: Decoupling Erase and Write Gates in Linear Attention
 *     for Better Memory Editing" (zhichai.net), section "Gated Delta Rule-2":
 *     the update rule and the two gates;
 *   - "엔비디아, 기억 수정 최적화 선형 어텐션 모델 공개" (ainews.random.gg),
 *     section "Gated Delta Rule-2: two gates instead of one": D_t =
 *     Diag(alpha_t) is channel-wise over key channels and the decay comes
 *     before the active edit; section "Chunkwise training and gate-aware
 *     backward": the chunkwise WY form with the cumulative channel-wise decay
 *     absorbed into asymmetric erase factors I - kbar_r ebar_r^T, chunk size
 *     C = 64;
 *   - same article, lead paragraph: decoding runs the recurrence one token at
 *     a time in constant memory.
 * The readout uses the post-update state; q is not scaled; the gates arrive
 * already in [0,1] and log_alpha already in log space (nothing is activated
 * or normalised inside the operator).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *     and 16-byte aligned. The library never allocates, frees or synchronises;
 *     every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and runs on the device that is current on the calling
 *     thread.
 *   - Token tensors are token-major: q, k, b, log_alpha are [B, T, H, d_k];
 *     v, w, o are [B, T, H, d_v]. States are [N, H, d_k, d_v] fp32 with d_v
 *     contiguous (row c of a head's state is key channel c).
 *   - q, k, v, b, w and o share `dtype`; log_alpha and states are always fp32.
 *   - Supported shapes: d_k = d_v in {64, 128}; H >= 1; sizes below 2^31
 *     elements per tensor.
 *   - Host-side validation happens before any launch; on failure nothing is
 *     launched and the status says why. A launch failure returns
 *     GDR2_ERR_CUDA (the CUDA error is then also pending in the runtime).
 *     Errors raised while kernels run surface at the caller's next
 *     synchronisation, as for any CUDA kernel.
 *   - `o` may not alias any input. Calls that share output or state buffers
 *     must be ordered by the caller (same stream or events).
 *   - Decay: any alpha in (0, 1] (log_alpha <= 0, any magnitude). The chunk
 *     kernels use the chunk form while the cumulative log-decay of every key
 *     channel stays within 64 of its value at the chunk's middle row (decay
 *     factors e^{+-64}); a chunk past that (a channel forgetting faster than
 *     about e^-2 per token on average) is computed on the device by the exact
 *     token recurrence instead -- for the bf16 d = 128 kernel the whole
 *     (sequence, head) unit, otherwise that chunk -- which is slower but
 *     exact to fp32 rounding. Nothing is reported and nothing is clamped.
 *     log_alpha > 0 (alpha > 1) is outside the operator's domain: the range
 *     test reads the chunk's half sums, which bound every factor only when the
 *     decay is monotone, so such inputs give unspecified results.
 */
#ifndef GDR2_H_
#define GDR2_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GDR2_OK = 0,
    GDR2_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment, bad dtype */
    GDR2_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d_k != d_v) */
    GDR2_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
    GDR2_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
    GDR2_ERR_DEVICE_TIMEOUT = 5 /* a bounded device-side wait gave up */
} gdr2_status;

typedef enum {
    GDR2_FP32 = 0,
    GDR2_BF16 = 1
} gdr2_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char *gdr2_status_string(gdr2_status status);

/* Library version as major*10000 + minor*100 + patch. */
int gdr2_version(void);

/*
 * gdr2_chunk_fwd -- chunkwise-parallel forward (prefill / training forward).
 *
 * Computes o_t for every token and the state after the last token of every
 * sequence, with the chunk form of the recurrence (C = 64): inside a chunk
 * the cumulative log-decay g_r (relative to the chunk start, fp32) turns the
 * token transitions into asymmetric rank-one factors I - kbar_r ebar_r^T with
 * kbar_r = k_r . exp(-g_r) and ebar_r = b_r . k_r . exp(g_r); the strictly
 * lower 64 x 64 matrix A = tril(Ebar Kbar^T) gives T = (I + A)^{-1}, the WY
 * factors W = T Ebar and U = T Z - W S0 (Z = W_gate . V), and then
 *     O   = Qbar S0 + tril(Qbar Kbar^T) U,        Qbar = Q . exp(g),
 *     S_C = Diag(exp(g_C)) S0 + (K . exp(g_C - g))^T U.
 * ("Chunkwise training and gate-aware backward", ainews.random.gg article.)
 *
 * Arguments
 *   q, k, b      [B, T, H, d_k] in `dtype`
 *   v, w         [B, T, H, d_v] in `dtype`     (w is the write gate)
 *   log_alpha    [B, T, H, d_k] fp32           (log of the per-channel decay)
 *   init_state   [N, H, d_k, d_v] fp32, or NULL for zero initial states
 *   cu_seqlens   NULL, or a DEVICE int32 array of N+1 offsets for a packed
 *                variable-length batch: then B must be 1, sequence n covers
 *                tokens cu_seqlens[n] .. cu_seqlens[n+1]-1, offsets must be
 *                non-decreasing with cu_seqlens[0] = 0 and cu_seqlens[N] = T
 *                (the device values are trusted; they are not read on the
 *                host). Chunks restart at every sequence start.
 *   B, T, H      batch, tokens per sequence (total tokens when packed), heads
 *   d_k, d_v     key / value head dimensions
 *   num_seqs     N: must equal B without cu_seqlens
 *   dtype        GDR2_FP32 or GDR2_BF16 for q, k, v, b, w, o
 *   o            [B, T, H, d_v] in `dtype` (output)
 *   final_state  [N, H, d_k, d_v] fp32 (output), or NULL to skip it;
 *                may alias init_state (each head reads its initial state
 *                before it writes its final state)
 *   workspace, workspace_bytes
 *                device scratch, 16-byte aligned. A packed batch of several
 *                sequences requires the size gdr2_chunk_fwd_workspace_size()
 *                reports: the order in which sequences are processed (longest
 *                first, computed on the device from cu_seqlens). A fixed-length
 *                bf16 batch with d = 128 and few (sequence, head) units may be
 *                given the (larger) reported size to run the segment-parallel
 *                scan: each sequence is cut into segments that run concurrently
 *                (from zero and from the identity state), then the segment
 *                states are chained in fp32 and the later segments' outputs
 *                corrected; with less (down to NULL / 0) it runs the serial
 *                scan. Contents are overwritten, so calls that share a
 *                workspace must be ordered on the GPU.
 *   stream       cudaStream_t
 * Precision: with GDR2_FP32 every product runs in fp32 on CUDA cores; with
 * GDR2_BF16 the dense intra-chunk contractions run on the tensor cores with
 * bf16 operands and fp32 accumulation while the state stays fp32.
 */
gdr2_status gdr2_chunk_fwd(const void *q, const void *k, const void *v,
                           const float *log_alpha, const void *b, const void *w,
                           const float *init_state, const int32_t *cu_seqlens,
                           int64_t B, int64_t T, int64_t H, int64_t d_k,
                           int64_t d_v, int64_t num_seqs, gdr2_dtype dtype,
                           void *o, float *final_state, void *workspace,
                           size_t workspace_bytes, void *stream);

/* Scratch bytes gdr2_chunk_fwd uses for this problem (written to *bytes), a
 * multiple of 256: for a packed batch of num_seqs > 1 sequences (B == 1), 4
 * bytes per sequence (required); for a fixed-length batch, 0 or, when the
 * segment-parallel scan applies (bf16, d = 128, at most 64 / (2P - 1) (sequence,
 * head) units for P >= 2 segments of >= 8 chunks), B*T*H*256 bytes (the
 * per-token readout maps, bf16) plus 2 * B*P*H*64 KiB (segment states, fp32)
 * (optional: a smaller workspace runs the serial scan). */
gdr2_status gdr2_chunk_fwd_workspace_size(int64_t B, int64_t T, int64_t H,
                                          int64_t d_k, int64_t d_v,
                                          int64_t num_seqs, gdr2_dtype dtype,
                                          size_t *bytes);

/*
 * gdr2_chunk_fwd_noalloc -- gdr2_chunk_fwd for callers that cannot allocate.
 *
 * (An addition of this library; the pages have no counterpart.) Some callers
 * cannot give the library scratch memory: code that is handed only its input
 * and output buffers by a host framework with no way to ask for more, or
 * deployments that reserve all device memory up front and must not call
 * cudaMalloc on the hot path (which can also stall other work on the device).
 * This entry point takes the same arguments as gdr2_chunk_fwd minus the
 * workspace and allocates nothing: the one piece of scratch the chunk forward
 * uses (the longest-first order of a packed batch, 4 bytes per sequence)
 * lives in a fixed 64 KiB array inside the library, held on every GPU that
 * loads the library until the process exits.
 *   - Limit: a packed batch (cu_seqlens, num_seqs > 1) may hold at most 16384
 *     sequences; larger ones return GDR2_ERR_UNSUPPORTED before any launch.
 *     Fixed-length batches use no scratch and have no extra limit (they run
 *     the serial scan, never the segment-parallel one).
 *   - The first call on a device looks up the array's device address (once
 *     per device, with that device current); make that first call before any
 *     stream capture. The address is kept for the rest of the process, so the
 *     calls must run in the device's primary context (the CUDA runtime's
 *     default) and not after a cudaDeviceReset; a lookup that fails returns
 *     GDR2_ERR_CUDA and is tried again on the next call.
 *   - All calls on a device share the array and it keeps the last call's
 *     contents; each call rewrites every entry it reads, so nothing has to be
 *     cleared, but calls that overlap on the GPU (unordered streams) race on
 *     it and must be serialised by the caller.
 * Results are identical to gdr2_chunk_fwd on the same inputs.
 */
gdr2_status gdr2_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                   const float *log_alpha, const void *b, const void *w,
                                   const float *init_state, const int32_t *cu_seqlens,
                                   int64_t B, int64_t T, int64_t H, int64_t d_k,
                                   int64_t d_v, int64_t num_seqs, gdr2_dtype dtype,
                                   void *o, float *final_state, void *stream);

/*
 * gdr2_chunk_bwd -- gate-aware backward (vector-Jacobian product) of the
 * recurrence over whole sequences, for training.
 *
 * Given the forward's inputs and the cotangents dO of o and dS_T of the final
 * states, returns the gradients of L = <dO, o> + <dS_T, S_T> with respect to
 * q, k, v, log_alpha, b, w and the initial states. The "Chunkwise training
 * and gate-aware backward" section of the ainews.random.gg article notes that
 * with two different diagonal gates the gate factors enter the gradient's dot
 * products; every gradient here is the chain rule of the token rule
 *     S'_t = Diag(alpha_t) S_{t-1},  u_t = w_t.v_t - S'_t^T (b_t.k_t),
 *     S_t = S'_t + k_t u_t^T,        o_t = S_t^T q_t,
 * evaluated in fp32: a forward sweep and a reverse (cotangent) sweep along
 * the tokens, each per value column, store per-token vectors and per-chunk
 * (64 tokens) checkpoints in the workspace; a per-chunk pass then forms the
 * key-side gradients row by row.
 *
 * Arguments (shapes as for gdr2_chunk_fwd; the same B, T, H, N, cu_seqlens)
 *   q, k, v, log_alpha, b, w, init_state, cu_seqlens
 *                the forward's inputs (init_state NULL = zero)
 *   d_o          [B, T, H, d_v] in `dtype`: cotangent of o
 *   d_final_state [N, H, d_k, d_v] fp32: cotangent of the final states, or
 *                NULL for zero
 *   dq, dk, db   [B, T, H, d_k] in `dtype` (outputs)
 *   dv, dw       [B, T, H, d_v] in `dtype` (outputs)
 *   d_log_alpha  [B, T, H, d_k] fp32 (output)
 *   d_init_state [N, H, d_k, d_v] fp32 (output), or NULL to skip it; may
 *                alias d_final_state
 *   workspace, workspace_bytes
 *                device scratch of at least gdr2_chunk_bwd_workspace_size()
 *                bytes, 16-byte aligned (required whenever N > 0); contents
 *                are overwritten
 * Outputs may not alias inputs (except d_init_state / d_final_state). Inputs
 * are the post-activation values (there is no prologue variant). Errors as
 * for gdr2_chunk_fwd; GDR2_ERR_WORKSPACE if the workspace is missing or small.
 */
gdr2_status gdr2_chunk_bwd(const void *q, const void *k, const void *v,
                           const float *log_alpha, const void *b, const void *w,
                           const float *init_state, const int32_t *cu_seqlens,
                           const void *d_o, const float *d_final_state,
                           int64_t B, int64_t T, int64_t H, int64_t d_k, int64_t d_v,
                           int64_t num_seqs, gdr2_dtype dtype,
                           void *dq, void *dk, void *dv, float *d_log_alpha,
                           void *db, void *dw, float *d_init_state,
                           void *workspace, size_t workspace_bytes, void *stream);

/* Scratch bytes gdr2_chunk_bwd needs (written to *bytes), a multiple of 256:
 * with S = B*T/64 + N checkpoint slots (integer division), 2 * S*H*d_k*d_v*4
 * bytes of fp32 checkpoints plus 2 * B*T*H*d_v*4 bytes of per-token fp32
 * vectors. */
gdr2_status gdr2_chunk_bwd_workspace_size(int64_t B, int64_t T, int64_t H,
                                          int64_t d_k, int64_t d_v,
                                          int64_t num_seqs, gdr2_dtype dtype,
                                          size_t *bytes);

/*
 * gdr2_recurrent_step -- one decode step for N independent sequences.
 *
 * For every sequence n and head h, with the state updated IN PLACE:
 *     S <- (I - k (b . k)^T) Diag(exp(log_alpha)) S + k (w . v)^T,
 *     o  = S^T q.
 * ("Gated Delta Rule-2" section of the zhichai.net summary; decoding to
 * constant memory per the ainews.random.gg article's lead.)
 *
 *   q, k, b      [N, H, d_k] in `dtype`;  log_alpha [N, H, d_k] fp32
 *   v, w         [N, H, d_v] in `dtype`
 *   state        [N, H, d_k, d_v] fp32, read and written in place
 *   o            [N, H, d_v] in `dtype` (output)
 * No workspace. Each (n, h) is independent, so N may be any batch size.
 */
gdr2_status gdr2_recurrent_step(const void *q, const void *k, const void *v,
                                const float *log_alpha, const void *b,
                                const void *w, float *state, int64_t N,
                                int64_t H, int64_t d_k, int64_t d_v,
                                gdr2_dtype dtype, void *o, void *stream);

/*
 * Fused prologue (bit flags for the *_preact entry points below).
 *
 * In the Gated DeltaNet-2 block ("Block design and hybrid model", ainews
 * article) the query and key paths end in L2 normalisation, the erase and write
 * gates are sigmoid projections and the decay comes from its own linear
 * branch. These flags let the kernels apply those last element-wise steps to
 * pre-activation inputs while loading them, instead of a separate pass over
 * the five tensors. Each is computed in fp32 per token and head:
 *   GDR2_PROLOGUE_QK_L2NORM      q, k <- x / sqrt(sum_c x_c^2 + 1e-6)
 *   GDR2_PROLOGUE_GATE_SIGMOID   b, w <- 1 / (1 + exp(-x))
 *   GDR2_PROLOGUE_DECAY_SOFTPLUS log_alpha <- -softplus(x) = -log(1 + exp(x))
 * (the pages do not print the decay branch's activation; -softplus is the
 * usual way to map a projection to a log-decay <= 0, and is this library's
 * reading). v passes unchanged: its SiLU precedes the operator.
 */
#define GDR2_PROLOGUE_QK_L2NORM 1u
#define GDR2_PROLOGUE_GATE_SIGMOID 2u
#define GDR2_PROLOGUE_DECAY_SOFTPLUS 4u

/* gdr2_chunk_fwd on pre-activation inputs: the `prologue` flags (a combination
 * of GDR2_PROLOGUE_*) name the activations applied to q, k, b, w, log_alpha on
 * load; everything else (arguments, layouts, workspace, errors) is exactly as
 * for gdr2_chunk_fwd, which equals this call with prologue = 0. Unknown flag
 * bits return GDR2_ERR_INVALID_ARG. */
gdr2_status gdr2_chunk_fwd_preact(const void *q, const void *k, const void *v,
                                  const float *log_alpha, const void *b, const void *w,
                                  const float *init_state, const int32_t *cu_seqlens,
                                  int64_t B, int64_t T, int64_t H, int64_t d_k,
                                  int64_t d_v, int64_t num_seqs, gdr2_dtype dtype,
                                  void *o, float *final_state, void *workspace,
                                  size_t workspace_bytes, uint32_t prologue, void *stream);

/* gdr2_recurrent_step on pre-activation inputs (same `prologue` flags). */
gdr2_status gdr2_recurrent_step_preact(const void *q, const void *k, const void *v,
                                       const float *log_alpha, const void *b,
                                       const void *w, float *state, int64_t N,
                                       int64_t H, int64_t d_k, int64_t d_v,
                                       gdr2_dtype dtype, void *o, uint32_t prologue,
                                       void *stream);

/*
 * gdr2_qed_fwd -- forward with the QED second erase direction (a reading).
 *
 * "The Query Knows What to Forget: A Second Erase Direction for Linear
 * Attention" (thelatestinai.com listing; abstract and Table 1) adds to the
 * key-directed erase of Gated Delta Rule-2 a second erase direction derived
 * from the query and orthogonal to the key, gated by b_t, with a per-head
 * strength (its Table 4 sweeps the strength at inference). The page does not
 * print the update (its equation (6)); this call computes the plain reading,
 * per (sequence, head), token by token:
 *
 *   src = q_t, or direction[h] when `direction` is given (the paper's
 *         fixed-direction control arm)
 *   p   = src - (k_t.src / k_t.k_t) k_t   with GDR2_QED_PROJECT (else src)
 *   u   = p / |p|                          (0 when |p|^2 <= 1e-12 |src|^2)
 *   f   = b_t . u                          with GDR2_QED_GATE (else u)
 *   S_t = (I - k_t (b_t . k_t)^T - strength[h] u f^T) Diag(exp(log_alpha_t)) S_{t-1}
 *         + k_t (w_t . v_t)^T
 *   o_t = S_t^T q_t
 *
 * Flags 0 .. 3 select the paper's Table 1 arms (GDR2_QED_GATE |
 * GDR2_QED_PROJECT is the full variant); strength 0 is exactly the plain rule.
 *
 * Arguments: token tensors, init_state, cu_seqlens, B, T, H, num_seqs, dtype,
 * o and final_state exactly as gdr2_chunk_fwd (d_k = d_v = 64 or 128;
 * no workspace). strength: device fp32 [H]. direction: device fp32 [H, d_k]
 * or NULL (the query). The state and all arithmetic are fp32 on the CUDA
 * cores, one CTA per (sequence, head, 32 value columns), tokens in order: a
 * reference-grade path, not a tuned one. Returns GDR2_ERR_INVALID_ARG for
 * unknown flag bits, a null strength or misaligned pointers, and the same
 * dimension errors as gdr2_chunk_fwd. Asynchronous on `stream`.
 */
#define GDR2_QED_GATE 1u
#define GDR2_QED_PROJECT 2u
gdr2_status gdr2_qed_fwd(const void *q, const void *k, const void *v, const float *log_alpha,
                         const void *b, const void *w, const float *strength,
                         const float *direction, uint32_t flags, const float *init_state,
                         const int32_t *cu_seqlens, int64_t B, int64_t T, int64_t H,
                         int64_t d_k, int64_t d_v, int64_t num_seqs, gdr2_dtype dtype,
                         void *o, float *final_state, void *stream);

/*
 * gdr2_check_device_error -- reports whether a kernel of this library gave up
 * a bounded device-side wait on the current device since the last check.
 *
 * The tensor-core kernels (the chunk forward and the segment split's output
 * correction) bound every wait inside the GPU (about one second without
 * progress); when one runs out, the affected CTA records the site in a
 * device-global error word, drains its in-flight copies and MMAs, frees its
 * tensor memory and returns, leaving its outputs incomplete. This call
 * synchronises `stream`, then reads and clears those words. Returns
 * GDR2_OK (no timeout), GDR2_ERR_DEVICE_TIMEOUT, or GDR2_ERR_CUDA if the
 * synchronisation or the read failed.
 */
gdr2_status gdr2_check_device_error(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* GDR2_H_ */
