/*
 * kda.h -- C ABI of libkda.so: the Kimi Delta Attention (KDA) channel-wise
 * gated delta-rule recurrence on NVIDIA B200 (sm_100a).
 *
 * The operation (per sequence and head; state S is dk x dv, fp32):
 *     S'  = Diag(exp(log_alpha_t)) S        one decay per KEY channel (row)
 *     r   = S'^T k_t                        value the key reads now
 *     S   = S' + k_t (beta_t (v_t - r))^T   delta write
 *     o_t = S^T q_t                         read-out after the write
 * Sources: "22580: from GPT-2 to Kimi K3, explained" (temp07.ru; English
 * original at marvinlee.cn), sections "DeltaNet, or Fast Weight Programmers"
 * (cached forward: read at the key, subtract, write the outer product, read
 * out with no denominator), "DeltaNet, or Parallelizing Linear Transformers
 * with Delta Rule" (token loop for prefill and the chunk-wise form),
 * "Gated Delta Net" (the decay alpha: 1 = pure delta rule, 0 = clear) and
 * "KDA / Kimi Linear" (a separate decay per channel); the ai-flip.ru KDA
 * explainer, section on channel-wise gating (a diagonal gate matrix) and on
 * chunking for tensor cores.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or keeps them. Tensors are contiguous
 *     and row-major in the shapes given below.
 *   - q and k are used as given (no normalisation, no 1/sqrt(d) scale).
 *   - log_alpha = log(alpha) <= 0 (fp32). -INFINITY is a full clear. The
 *     chunked prefill path clamps log_alpha to >= KDA_CHUNK_LOG_ALPHA_MIN
 *     (alpha >= 4.5e-5) so its within-chunk factorisation stays finite; the
 *     token-recurrent and decode kernels apply the gate exactly.
 *   - Work is enqueued on `stream` and runs asynchronously. Argument errors
 *     are reported synchronously (nothing is launched); launch failures map
 *     to KDA_ERR_CUDA; a device-side timeout of a bounded wait is recorded in
 *     a device status word read by kda_get_device_status().
 *   - Supported head sizes: dk, dv in {64, 128}. The chunked tensor-core
 *     path needs dk = dv = 128, bf16 inputs and chunk = 64.
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad cu_seqlens shape */
    KDA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (head size, chunk) */
    KDA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required   */
    KDA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed         */
    KDA_ERR_TIMEOUT = 5        /* a bounded device-side wait gave up           */
} kda_status;

typedef enum {
    KDA_F32 = 0,               /* q, k, v and o are fp32                       */
    KDA_BF16 = 1               /* q, k, v and o are bf16                       */
} kda_dtype;

/*
 * Gate forms (the decay alpha that multiplies the state before each token's
 * read). "22580: from GPT-2 to Kimi K3, explained": "KDA / Kimi Linear" (one
 * decay per key channel), "Gated Delta Net" (one data-dependent scalar per
 * token, multiplying the whole previous state), "DeltaNet, or Fast Weight
 * Programmers" (no decay: the plain delta rule).
 */
typedef enum {
    KDA_GATE_CHANNEL = 0,      /* log_alpha [.., H, dk] fp32                   */
    KDA_GATE_SCALAR = 1,       /* log_alpha [.., H] fp32, same on every channel */
    KDA_GATE_NONE = 2          /* alpha = 1; log_alpha unused, may be NULL      */
} kda_gate;

/*
 * Input prologue flags: raw projections instead of ready inputs, as the
 * cached forward of "DeltaNet, or Fast Weight Programmers" computes them just
 * before the recurrence. Each flag applies its transform inside the kernel:
 *   KDA_RAW_QK    q and k are raw: each token's head vector x becomes
 *                 silu(x) / max(|silu(x)|_2, 1e-12)  (F.normalize of SiLU)
 *   KDA_RAW_BETA  beta holds logits: beta = sigmoid(beta)
 *   KDA_RAW_GATE  log_alpha holds gate logits x: alpha = sigmoid(x), i.e.
 *                 log_alpha = log sigmoid(x) (a decay between 0 and 1)
 */
#define KDA_RAW_QK   0x1u
#define KDA_RAW_BETA 0x2u
#define KDA_RAW_GATE 0x4u

/* Most tokens per sequence one kda_decode_ex call takes. */
#define KDA_DECODE_MAX_TOKENS 16

/* Lower bound applied to log_alpha by the chunked prefill path. */
#define KDA_CHUNK_LOG_ALPHA_MIN (-10.0f)

/* Most sequences one kda_prefill_noalloc call accepts (its fixed scratch). */
#define KDA_NOALLOC_MAX_SEQS 65536

/* Human-readable name of a status code (static string, never NULL). */
const char *kda_status_string(kda_status status);

/* Library version as major*10000 + minor*100 + patch. */
int kda_version(void);

/*
 * Bytes of device workspace kda_prefill needs for a call with these
 * arguments (the same n_seq, H, dk, dv, dtype and chunk, and whether
 * cu_seqlens is given). It is non-zero only when the chunked tensor-core
 * kernel serves the call (bf16, dk = dv = 128, chunk = 64) and then holds:
 *   - the longest-first order of packed sequences (n_seq int32), when
 *     cu_seqlens is given;
 *   - one dk x dv fp32 hand-over slot per (sequence, head) chain, when there
 *     are at most 128 chains: a ring of CTAs may then serve each chain and
 *     passes the state between its CTAs through the slot.
 * Each part starts on a 256-byte boundary. Never fails; negative sizes count
 * as 0.
 */
size_t kda_prefill_workspace_bytes(int n_seq, int H, int dk, int dv, kda_dtype dtype,
                                   int chunk, int has_cu_seqlens);

/*
 * kda_prefill -- run the recurrence over whole sequences (prefill), with an
 * optional cached initial state, returning every output and the final state.
 *
 * Dense batch (cu_seqlens == NULL): B sequences of T tokens.
 *   q, k       [B, T, H, dk]  dtype          v, o   [B, T, H, dv]  dtype
 *   log_alpha  [B, T, H, dk]  fp32           beta   [B, T, H]      fp32
 *   init_state [B, H, dk, dv] fp32 or NULL (zeros)
 *   final_state[B, H, dk, dv] fp32 or NULL (not written)
 *   n_seq must be B (or 0, meaning B).
 * Packed variable length (cu_seqlens != NULL, a DEVICE int32 array of
 * n_seq + 1 offsets, cu[0] = 0, non-decreasing, cu[n_seq] = T): B must be 1,
 *   the token tensors are [1, T, H, *], sequence i owns tokens
 *   [cu[i], cu[i+1]) and starts from init_state[i] (or zeros), and
 *   init_state / final_state are [n_seq, H, dk, dv]. A zero-length sequence
 *   copies its initial state to its final state. The offsets are read on the
 *   device only; offsets that break the rules above give undefined output but
 *   never an out-of-bounds access (each sequence is clamped to [0, T)).
 * chunk: 0 selects the token-recurrent kernel (fp32 state in registers, any
 *   supported head size and dtype, exact gate). 64 selects the chunked
 *   tensor-core kernel (tcgen05 MMAs with TMEM accumulators) for bf16 inputs
 *   with dk = dv = 128; other dtypes and head sizes run the token-recurrent
 *   kernel whatever the chunk.
 * final_state may alias init_state (each chain reads its initial state
 *   before writing its final one). o must not alias any input.
 * The chunked kernel needs q, k, v, o, log_alpha and final_state 16-byte
 *   aligned (it moves them in 8- and 16-byte vectors); otherwise
 *   KDA_ERR_INVALID_ARG and nothing is launched.
 * workspace: at least kda_prefill_workspace_bytes(n_seq, H, dk, dv, dtype,
 *   chunk, cu_seqlens != NULL) bytes of device memory, 256-byte aligned, not
 *   shared with a call that may run at the same time; may be NULL when that
 *   is 0. Missing or too small: KDA_ERR_WORKSPACE, nothing launched.
 */
kda_status kda_prefill(const void *q, const void *k, const void *v,
                       const float *log_alpha, const float *beta,
                       const float *init_state, const int32_t *cu_seqlens,
                       int n_seq, int B, int T, int H, int dk, int dv,
                       kda_dtype dtype, int chunk,
                       void *o, float *final_state,
                       void *workspace, size_t workspace_bytes,
                       cudaStream_t stream);

/*
 * kda_decode_step -- one token per sequence against a cached state, updated
 * in place (the pages' decode call: the same forward with one token and the
 * cache from the previous call).
 *   q, k       [B, H, dk]  dtype            v, o  [B, H, dv]  dtype
 *   log_alpha  [B, H, dk]  fp32             beta  [B, H]      fp32
 *   state      [B, H, dk, dv] fp32, read and overwritten with the new state
 * The kernel is HBM-bound: each head's state is read once and written once.
 */
kda_status kda_decode_step(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta,
                           float *state, int B, int H, int dk, int dv,
                           kda_dtype dtype, void *o, cudaStream_t stream);

/*
 * kda_prefill_ex -- kda_prefill with a gate form and an input prologue.
 * Arguments as kda_prefill, plus:
 *   gate   KDA_GATE_CHANNEL: log_alpha [B, T, H, dk] (kda_prefill's form);
 *          KDA_GATE_SCALAR:  log_alpha [B, T, H], one decay per token and head
 *                            (Gated DeltaNet; 4 bytes per head-token read
 *                            instead of 4 * dk);
 *          KDA_GATE_NONE:    no decay (DeltaNet); log_alpha may be NULL.
 *   flags  any of KDA_RAW_QK, KDA_RAW_BETA, KDA_RAW_GATE (see above); 0 for
 *          ready inputs. With KDA_RAW_GATE the values in log_alpha are logits
 *          (same shape as the gate form says).
 * Both kernels take every form; the chunked kernel clamps the resulting
 * log_alpha at KDA_CHUNK_LOG_ALPHA_MIN as in kda_prefill. Unknown gate or
 * flag bits: KDA_ERR_INVALID_ARG. kda_prefill is kda_prefill_ex with
 * KDA_GATE_CHANNEL and flags 0. The workspace is the same as kda_prefill's.
 */
kda_status kda_prefill_ex(const void *q, const void *k, const void *v,
                          const float *log_alpha, const float *beta,
                          const float *init_state, const int32_t *cu_seqlens,
                          int n_seq, int B, int T, int H, int dk, int dv,
                          kda_dtype dtype, kda_gate gate, unsigned flags, int chunk,
                          void *o, float *final_state,
                          void *workspace, size_t workspace_bytes,
                          cudaStream_t stream);

/*
 * kda_decode_ex -- T tokens per sequence (1 <= T <= KDA_DECODE_MAX_TOKENS)
 * against a cached state, updated in place: the same result as T successive
 * kda_decode_step calls (or kda_prefill over the T tokens from that state),
 * with each head's state read once and written once per call (the
 * multi-token decode of speculative verification or short appends).
 *   q, k       [B, T, H, dk]  dtype           v, o  [B, T, H, dv]  dtype
 *   log_alpha  per `gate`: [B, T, H, dk], [B, T, H] or unused (NULL allowed)
 *   beta       [B, T, H] fp32                 state [B, H, dk, dv] fp32
 *   gate, flags as for kda_prefill_ex.
 * T > KDA_DECODE_MAX_TOKENS: KDA_ERR_UNSUPPORTED (use kda_prefill with
 * init_state). kda_decode_step is kda_decode_ex with T = 1,
 * KDA_GATE_CHANNEL and flags 0. The gate is applied exactly (no clamp).
 */
kda_status kda_decode_ex(const void *q, const void *k, const void *v,
                         const float *log_alpha, const float *beta,
                         float *state, int B, int T, int H, int dk, int dv,
                         kda_dtype dtype, kda_gate gate, unsigned flags,
                         void *o, cudaStream_t stream);

/*
 * kda_backward -- gradients of a loss through the recurrence (the reverse
 * mode a training step needs; "22580: from GPT-2 to Kimi K3, explained",
 * section "DeltaNet, or Parallelizing Linear Transformers with Delta Rule",
 * motivates the chunk-wise form by hardware-efficient training). Given the
 * forward inputs and dL/do (and optionally dL/dS_final), returns dL/dq,
 * dL/dk, dL/dv, dL/dlog_alpha, dL/dbeta and dL/dS_0, all fp32:
 *   q, k, v, log_alpha, beta, init_state, cu_seqlens, n_seq, B, T, H, dk, dv,
 *   dtype, gate   as for kda_prefill_ex (ready inputs; raw ones: kda_backward_ex)
 *   d_o        [B, T, H, dv] dtype           d_final [n_seq, H, dk, dv] fp32 or NULL
 *   dq, dk_out [B, T, H, dk] fp32            dv_out  [B, T, H, dv] fp32
 *   dlog_alpha the gate's shape, fp32 (NULL with KDA_GATE_NONE)
 *   dbeta      [B, T, H] fp32                d_init  [n_seq, H, dk, dv] fp32 or NULL
 * The gate is applied exactly (no clamp). Work: a forward pass that stores
 * the state every 16 tokens in the workspace, then a reverse sweep that
 * recomputes each 16-token block from its checkpoint (token-recurrent, one
 * CTA per (sequence, head, slice of value columns: 32 wide, or 8 when the
 * sequences and heads are few)). The column slices of a head
 * add their parts of dq, dk, dlog_alpha and dbeta with atomic adds, so those
 * can differ between runs in the last bits. init_state, d_final and d_init
 * must be 16-byte aligned. workspace: at least
 * kda_backward_workspace_bytes(n_seq, B * T, H, dk, dv) bytes, 256-byte
 * aligned (missing or small: KDA_ERR_WORKSPACE).
 */
size_t kda_backward_workspace_bytes(int n_seq, int64_t tokens, int H, int dk, int dv);

kda_status kda_backward(const void *q, const void *k, const void *v,
                        const float *log_alpha, const float *beta,
                        const float *init_state, const int32_t *cu_seqlens,
                        int n_seq, int B, int T, int H, int dk, int dv,
                        kda_dtype dtype, kda_gate gate,
                        const void *d_o, const float *d_final,
                        float *dq, float *dk_out, float *dv_out, float *dlog_alpha,
                        float *dbeta, float *d_init,
                        void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * kda_backward_ex -- kda_backward for inputs given as raw projections: the
 * reverse mode of kda_prefill_ex with the same prologue flags (KDA_RAW_QK,
 * KDA_RAW_BETA, KDA_RAW_GATE; the cached forward of "DeltaNet, or Fast Weight
 * Programmers" applies SiLU and L2 normalisation to q and k and a sigmoid to
 * beta before the recurrence). The gradients returned are with respect to the
 * inputs as passed: dq, dk_out through the normalisation's Jacobian
 * (I - n n^T) / max(|u|, 1e-12) (u = SiLU(x), n = u / max(|u|, 1e-12); below
 * 1e-12 the map is u / 1e-12) and SiLU's derivative; dbeta through the
 * sigmoid; dlog_alpha, for gate logits x, is dL/dx = dL/dlog_alpha times
 * sigmoid(-x). The prologue runs in fp32 inside the kernels: a first kernel
 * stores each row's 1 / max(|SiLU(x)|, 1e-12) for q and k in the workspace,
 * the token sweep applies SiLU and the sigmoids with the hardware exponential
 * and reciprocal (relative error a few 1e-7), and a last kernel on the same
 * stream maps the gradients back to the raw inputs (expf-based). flags 0 is
 * kda_backward. The workspace (kda_backward_workspace_bytes) includes the
 * row scales.
 * Arguments, layouts, workspace and errors otherwise as kda_backward; flags
 * other than the three: KDA_ERR_INVALID_ARG.
 */
kda_status kda_backward_ex(const void *q, const void *k, const void *v,
                           const float *log_alpha, const float *beta,
                           const float *init_state, const int32_t *cu_seqlens,
                           int n_seq, int B, int T, int H, int dk, int dv,
                           kda_dtype dtype, kda_gate gate, unsigned flags,
                           const void *d_o, const float *d_final,
                           float *dq, float *dk_out, float *dv_out, float *dlog_alpha,
                           float *dbeta, float *d_init,
                           void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * kda_prefill_noalloc -- the packed variable-length chunked prefill of
 * kda_prefill (cu_seqlens given, bf16, dk = dv = 128, chunk = 64) for callers
 * that cannot allocate device memory. The source pages have no counterpart:
 * this is a library convenience. kda_prefill needs a caller-provided
 * workspace for its per-call scratch (the longest-first order of the
 * sequences); this variant keeps that scratch in a fixed device array inside
 * the library instead, so a caller that may not call cudaMalloc can still run
 * it: a plugin or hook that is handed device pointers but owns no allocator, a
 * serving runtime whose device memory is already reserved by its own pool,
 * or a latency-critical path where an allocation (and the synchronisation it
 * can imply) is not acceptable.
 * Inputs and outputs are still caller-owned device memory, with the shapes of
 * kda_prefill's packed form: q, k, log_alpha [T, H, 128]; v, o [T, H, 128]
 * (bf16); beta [T, H]; cu_seqlens int32 [n_seq + 1]; init_state and
 * final_state [n_seq, H, 128, 128] fp32 or NULL.
 * Limits: n_seq <= KDA_NOALLOC_MAX_SEQS, else KDA_ERR_UNSUPPORTED and
 * nothing is launched; pointers aligned as kda_prefill's chunked path needs. The fixed scratch (256 KiB per device, held until the
 * process exits) is shared by every call on a device, so calls whose work
 * overlaps on the GPU race on it; calls on one stream are ordered and safe.
 * The first call on a device looks up the scratch's device address (once per
 * device, with that device current); make that first call before any stream
 * capture begins. The address is kept for the life of the process: after a
 * cudaDeviceReset of that device it is stale, so do not call this entry point
 * on a device that was reset. Allocates nothing and calls no allocating
 * routine.
 */
kda_status kda_prefill_noalloc(const void *q, const void *k, const void *v,
                               const float *log_alpha, const float *beta,
                               const float *init_state, const int32_t *cu_seqlens,
                               int n_seq, int T, int H, void *o, float *final_state,
                               cudaStream_t stream);

/*
 * kda_get_device_status -- synchronise `stream` and return the sticky device
 * status word of the current device: KDA_OK, or KDA_ERR_TIMEOUT when a
 * bounded wait inside a kernel gave up since the last reset (the kernel then
 * stopped its chain early, released its tensor memory and left its outputs
 * incomplete). If `reset` is non-zero the word is cleared after reading.
 * `detail` (may be NULL) receives an implementation-defined code naming the
 * wait that gave up (0 when none did).
 */
kda_status kda_get_device_status(int reset, int *detail, cudaStream_t stream);

/*
 * kda_selftest_wait_timeout -- exercise the bounded-wait failure path (a
 * test hook; the source pages have no counterpart). Launches one tiny kernel
 * on `stream` whose single thread waits, with the helpers every kernel of the
 * library uses, on an mbarrier nothing ever arrives on: once with CTA-scope
 * and once with cluster-scope acquire, each for max_ns nanoseconds of
 * %globaltimer. Both waits give up and record KDA_ERR_TIMEOUT in the device
 * status word (detail 9091: both waits, in order), exactly as a kernel
 * whose MMA or state hand-over never completed would; nothing faults or
 * traps and the context stays usable. Read the outcome with
 * kda_get_device_status(1, &detail, stream), which also clears it.
 *   max_ns  1e3 .. 1e9 (1 us to 1 s), else KDA_ERR_INVALID_ARG.
 */
kda_status kda_selftest_wait_timeout(uint64_t max_ns, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
