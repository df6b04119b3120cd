/*
 * gdla.h - C ABI of the GDLA forward core for NVIDIA B200 (sm_100a).
 *
 * Grouped Differential Latent Attention (GDLA), as described for the Motif 3
 * model (aitrends.kr/articles/94908, "314B MoE 언어 모델 Motif 3의 구조와 학습
 * 시스템", GDLA paragraphs; metalmedia.ai digest of arXiv 2608.09119, Table 1):
 *
 *   For every KV head j, GROUP = 4 signal query heads (4j..4j+3) and one noise
 *   query head (j) attend with causal softmax attention over the same K_j
 *   (dim 192) and V_j (dim 128), either over the full causal context or over
 *   a sliding window. With H_S,i and H_N,j the attention outputs,
 *       D_i     = H_S,i - lambda[t, i] * H_N,j          (j = i / 4)
 *       out_i   = sigmoid(gate_logits[t, i, :]) * D_i   (element-wise)
 *   and out is rounded once, to nearest even, to bf16.
 *
 * Readings where the pages are silent: lambda is one fp32 scalar per (token,
 * signal head) in (0, 1), precomputed by the caller as sigmoid(x W^lambda);
 * the softmax scale is 1/sqrt(192); a window of W keys includes the query
 * itself (keys t-W+1 .. t); nothing follows the subtract except the gate.
 * q and k arrive after any rotary embedding; the latent up-projection, the
 * lambda and gate projections and the output projection are ordinary GEMMs
 * outside this library.
 *
 * Conventions shared by every entry point:
 *  - All tensors are dense, row-major, caller-owned DEVICE memory unless a
 *    comment says HOST. Tensor base pointers must be 16-byte aligned.
 *  - bf16 is IEEE bfloat16 (1-8-7); lambda is fp32.
 *  - The library allocates no memory, keeps no state between calls (apart
 *    from the device-side failure word, see gdla_device_error, and per-device
 *    launch facts cached on the host: SM count, kernel attribute opt-ins) and
 *    may be called from several host threads at once.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL is the legacy
 *    default stream). GDLA_OK means every kernel was enqueued; a CUDA launch
 *    failure is reported as GDLA_ERR_CUDA.
 *  - Arguments are checked on the host before anything is launched; on an
 *    error nothing is launched and no output is written.
 *  - Results are deterministic (no atomics, fixed reduction order).
 *  - Output rows that belong to no sequence are never written.
 */
#ifndef GDLA_H
#define GDLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GDLA_API __attribute__((visibility("default")))
#else
#define GDLA_API
#endif

#define GDLA_GROUP 4          /* signal heads per noise / KV head (g) */
#define GDLA_DQK 192          /* query-key head dim */
#define GDLA_DV 128           /* value head dim */
#define GDLA_MAX_KV_HEADS 64  /* largest num_kv_heads accepted */
#define GDLA_LATENT_MAX_KV_HEADS 16  /* largest num_kv_heads of the latent-cache decode */
#define GDLA_DC 512           /* latent (compressed KV) dim */
#define GDLA_DR 64            /* shared rotary key dim */
#define GDLA_VERSION 1

typedef enum {
    GDLA_OK = 0,
    GDLA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, negative size, bad batch */
    GDLA_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels handle (e.g. > 64 KV heads) */
    GDLA_ERR_WORKSPACE = 3,    /* decode workspace missing or too small */
    GDLA_ERR_CUDA = 4          /* a CUDA call or kernel launch failed */
} gdla_status_t;

/*
 * Packed varlen prefill (GDLA core, full causal or sliding window).
 * Defined by the GDLA query-path paragraph of aitrends.kr/articles/94908
 * (D = H_S - lambda (.) Repeat_g(H_N), then the query-based gate) with the
 * head grouping of its group-ratio paragraph.
 *
 * N = sum(seqlens). Sequence b occupies packed rows [s_b, s_b + seqlens[b]).
 *   q_sig        bf16 [N, 4*num_kv_heads, 192]
 *   q_noise      bf16 [N, num_kv_heads, 192]
 *   k            bf16 [N, num_kv_heads, 192]
 *   v            bf16 [N, num_kv_heads, 128]
 *   lambda       fp32 [N, 4*num_kv_heads], values in (0, 1)
 *   gate_logits  bf16 [N, 4*num_kv_heads, 128]
 *   out          bf16 [N, 4*num_kv_heads, 128], written
 *   batch        number of sequences, >= 1
 *   seqlens      HOST int32 [batch], each >= 0 (empty sequences are skipped)
 *   num_kv_heads 1 .. GDLA_MAX_KV_HEADS
 *   window       <= 0: full causal; > 0: query t sees keys t-window+1 .. t
 *   stream       cudaStream_t to enqueue on
 * Errors: GDLA_ERR_INVALID_ARG for a null or non-16-byte-aligned pointer
 * (when N > 0), batch < 1, a negative length or N >= 2^31;
 * GDLA_ERR_UNSUPPORTED for num_kv_heads out of range; GDLA_ERR_CUDA if a
 * launch fails. N == 0 returns GDLA_OK without launching.
 */
GDLA_API gdla_status_t gdla_attn_fwd(const void *q_sig, const void *q_noise, const void *k, const void *v,
                            const float *lambda, const void *gate_logits, void *out,
                            int batch, const int32_t *seqlens, int num_kv_heads, int window,
                            void *stream);

/*
 * Prefill backward (the pages train GDLA end to end, aitrends.kr/articles/94908,
 * context-parallel and training-system paragraphs): the gradients of
 * sum(dout * out) for the packed varlen forward above, with the forward
 * recomputed (nothing is kept from it). Same shapes, layouts, seqlens and window
 * as gdla_attn_fwd, plus:
 *   dout     bf16 [N, 4*num_kv_heads, 128]   gradient of out (read)
 *   dq_sig   bf16 [N, 4*num_kv_heads, 192]   written
 *   dq_noise bf16 [N, num_kv_heads, 192]     written
 *   dk       bf16 [N, num_kv_heads, 192]     written
 *   dv       bf16 [N, num_kv_heads, 128]     written
 *   dlambda  fp32 [N, 4*num_kv_heads]        written
 *   dgate    bf16 [N, 4*num_kv_heads, 128]   written (gradient of the gate logits)
 *   workspace caller-owned device memory of gdla_attn_bwd_workspace_bytes(N,
 *            num_kv_heads) bytes, 256-byte aligned; its contents on entry do
 *            not matter
 * Every row of every gradient of a token in a sequence is written; the result
 * is deterministic (no atomics). Errors as gdla_attn_fwd, plus
 * GDLA_ERR_WORKSPACE for a missing, small or misaligned workspace. All device
 * buffers 16-byte aligned.
 */
GDLA_API size_t gdla_attn_bwd_workspace_bytes(long long total_tokens, int num_kv_heads);
GDLA_API gdla_status_t gdla_attn_bwd(const void *q_sig, const void *q_noise, const void *k, const void *v,
                                     const float *lambda, const void *gate_logits, const void *dout, void *dq_sig,
                                     void *dq_noise, void *dk, void *dv, float *dlambda, void *dgate, int batch,
                                     const int32_t *seqlens, int num_kv_heads, int window, void *workspace,
                                     size_t workspace_bytes, void *stream);

/*
 * Prologue: the attention's inputs from the hidden state (aitrends.kr/articles/94908,
 * GDLA query-path paragraph: c^Q = RMSNorm(x W^Q_a) expanded to content and rotary
 * queries; [c^KV; k^R] = x W^KV_a, c^KV RMSNorm'd once and expanded to the KV
 * heads, k^R rotated and shared by every head; group-ratio paragraph: lambda =
 * sigmoid(x W^lambda); the element-wise gate's logits x W^G). Readings: RMSNorm eps
 * 1e-6, rotary embedding of the 64 rotary dims in the rotate-half form (pairs i,
 * i + 32) with base 10000 and positions from 0 in each sequence; query heads are
 * ordered signal 0..4H-1 then noise 0..H-1, each [content 128 | rotary 64].
 * All weights are [out_features, in_features] bf16, row-major:
 *   x         bf16 [N, 4096]            hidden state of the packed tokens
 *   w_qa      bf16 [1024, 4096]         W^Q_a
 *   w_kva     bf16 [576, 4096]          W^KV_a (rows 0..511 -> c^KV, 512..575 -> k^R)
 *   gamma_q   fp32 [1024], gamma_kv fp32 [512]   RMSNorm weights
 *   w_qb      bf16 [5H*192, 1024]       W^Q_b, query head h at rows 192h..192h+191
 *   w_uk      bf16 [H, 128, 512]        per KV head: c^KV -> k_nope
 *   w_uv      bf16 [H, 128, 512]        per KV head: c^KV -> v
 *   w_lambda  bf16 [4H, 4096]           W^lambda (one per signal head)
 *   w_gate    bf16 [4H*128, 4096]       W^G
 * Outputs, in the layouts gdla_attn_fwd reads: q_sig [N, 4H, 192], q_noise [N, H, 192],
 * k [N, H, 192] (k_nope | rotated k^R), v [N, H, 128], lambda fp32 [N, 4H],
 * gate_logits [N, 4H, 128] (all bf16 but lambda). seqlens: HOST, batch <= 1024
 * sequences (positions restart at 0 in each). workspace: caller-owned, 256-byte
 * aligned, gdla_prologue_workspace_bytes(N) bytes. Errors as gdla_attn_fwd, plus
 * GDLA_ERR_WORKSPACE. Every buffer 16-byte aligned.
 */
GDLA_API size_t gdla_prologue_workspace_bytes(long long total_tokens);
GDLA_API gdla_status_t gdla_prologue(const void *x, const void *w_qa, const void *w_kva, const float *gamma_q,
                                     const float *gamma_kv, const void *w_qb, const void *w_uk, const void *w_uv,
                                     const void *w_lambda, const void *w_gate, void *q_sig, void *q_noise, void *k,
                                     void *v, float *lambda, void *gate_logits, int batch, const int32_t *seqlens,
                                     int num_kv_heads, void *workspace, size_t workspace_bytes, void *stream);

/*
 * Bytes of device workspace gdla_attn_decode needs for these sizes (0 when
 * no split-KV pass is used). Returns 0 for invalid sizes as well; the
 * workspace must be 256-byte aligned.
 */
GDLA_API size_t gdla_decode_workspace_bytes(int batch, int num_kv_heads, int max_seqlen_k, int window);

/*
 * Varlen decode: one new query token per sequence, attending over that
 * sequence's KV cache (the cache already holds the new token's key and value,
 * so the query sits at position L_b - 1). Same method as gdla_attn_fwd (the
 * KV-cache motivation is the aitrends.kr/articles/94908 paragraph contrasting
 * self-attention and MLA's compressed KV cache).
 *   q_sig        bf16 [batch, 4*num_kv_heads, 192]
 *   q_noise      bf16 [batch, num_kv_heads, 192]
 *   k_cache      bf16 [Nk, num_kv_heads, 192], sequences packed back to back
 *   v_cache      bf16 [Nk, num_kv_heads, 128]
 *   cu_seqlens_k DEVICE int32 [batch + 1]: sequence b owns cache rows
 *                cu[b] .. cu[b+1]-1; every L_b = cu[b+1]-cu[b] must be in
 *                1 .. max_seqlen_k and cu[b+1] <= num_cache_rows (a
 *                sequence that violates this gets an all-zero output)
 *   num_cache_rows HOST number of rows Nk in k_cache / v_cache, >= 1; reads
 *                never go past it
 *   max_seqlen_k HOST upper bound on every L_b, >= 1 (sizes the split plan)
 *   lambda       fp32 [batch, 4*num_kv_heads]
 *   gate_logits  bf16 [batch, 4*num_kv_heads, 128]
 *   out          bf16 [batch, 4*num_kv_heads, 128], written
 *   window       <= 0: full context; > 0: the last `window` cache rows
 *   workspace    DEVICE scratch of at least
 *                gdla_decode_workspace_bytes(batch, num_kv_heads,
 *                max_seqlen_k, window) bytes, 256-byte aligned (may be NULL
 *                when that is 0); its contents need no initialisation
 * Errors: GDLA_ERR_INVALID_ARG (null/misaligned pointers, batch < 1,
 * num_cache_rows < 1, max_seqlen_k < 1), GDLA_ERR_UNSUPPORTED (num_kv_heads out of range),
 * GDLA_ERR_WORKSPACE (workspace NULL or smaller than required),
 * GDLA_ERR_CUDA (launch failure).
 */
GDLA_API gdla_status_t gdla_attn_decode(const void *q_sig, const void *q_noise, const void *k_cache,
                               const void *v_cache, const int32_t *cu_seqlens_k, int num_cache_rows,
                               int max_seqlen_k,
                               const float *lambda, const void *gate_logits, void *out,
                               int batch, int num_kv_heads, int window,
                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode over the compressed (latent) KV cache, with the key and value
 * up-projections absorbed (aitrends.kr/articles/94908, head-configuration
 * paragraph: KV low-rank dimension 512 and one 64-wide rotary key shared by
 * every KV head, the KV heads being an up-projection of that compressed row;
 * the paragraph on MLA's compressed KV cache for decoding). The cache holds
 * one 576-wide row per token, [c (512) | k_rope (64)], 1,152 bytes instead of
 * the 10,240 of 16 expanded KV heads. Readings where the pages are silent:
 * the 192 query-key dims are 128 non-rotary then 64 rotary; per KV head j,
 * K_j = [W^UK_j c | k_rope] and V_j = W^UV_j c with W^UK_j, W^UV_j [128 x 512].
 * With q_abs = [W^UK_j^T q_nope | q_rope] (prepared by the caller), every
 * query head attends over the shared rows with scale 1/sqrt(192); its output
 * is H = W^UV_j (softmax-weighted average of c), followed by the same
 * D = H_S - lambda H_N and sigmoid gate as gdla_attn_decode.
 *   q_abs_sig    bf16 [batch, 4*num_kv_heads, 576]
 *   q_abs_noise  bf16 [batch, num_kv_heads, 576]
 *   ckv          bf16 [Nk, 576], sequences packed back to back
 *   cu_seqlens_k DEVICE int32 [batch + 1], as for gdla_attn_decode (a sequence
 *                whose length is not in 1 .. max_seqlen_k, or that ends past
 *                num_cache_rows, gets an all-zero output)
 *   num_cache_rows HOST number of rows Nk of ckv, >= 1; reads never pass it
 *   max_seqlen_k HOST upper bound on every L_b, >= 1 (sizes the split plan)
 *   w_uv         bf16 [num_kv_heads, 128, 512]
 *   lambda       fp32 [batch, 4*num_kv_heads]
 *   gate_logits  bf16 [batch, 4*num_kv_heads, 128]
 *   out          bf16 [batch, 4*num_kv_heads, 128], written
 *   num_kv_heads 1 .. 16 (all 5 * num_kv_heads query heads of a sequence share
 *                one CTA)
 *   window       <= 0: full context; > 0: the last `window` cache rows
 *   workspace    DEVICE scratch of at least gdla_decode_latent_workspace_bytes(
 *                batch, num_kv_heads, max_seqlen_k, window) bytes, 256-byte
 *                aligned; its contents need no initialisation
 * Errors: GDLA_ERR_INVALID_ARG (null/misaligned pointers, batch < 1,
 * num_cache_rows < 1, max_seqlen_k < 1), GDLA_ERR_UNSUPPORTED (num_kv_heads
 * outside 1..16), GDLA_ERR_WORKSPACE (workspace NULL, misaligned or smaller
 * than required), GDLA_ERR_CUDA (launch failure).
 */
GDLA_API size_t gdla_decode_latent_workspace_bytes(int batch, int num_kv_heads, int max_seqlen_k, int window);
GDLA_API gdla_status_t gdla_attn_decode_latent(const void *q_abs_sig, const void *q_abs_noise, const void *ckv,
                                               const int32_t *cu_seqlens_k, int num_cache_rows, int max_seqlen_k,
                                               const void *w_uv, const float *lambda, const void *gate_logits,
                                               void *out, int batch, int num_kv_heads, int window,
                                               void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode for callers that cannot allocate device memory. The paper has no
 * counterpart to this entry point; it exists for the library's users.
 *
 * Some callers only hold the buffers they are handed and may not allocate:
 * a plugin inside another inference runtime that forbids device allocation
 * on its execution path, or a service with a fixed, pre-reserved memory
 * budget where a cudaMalloc could fail or synchronise the device mid-request.
 * They cannot supply the split-KV workspace gdla_attn_decode needs. This
 * call takes the same arguments and gives the same results as
 * gdla_attn_decode, without the workspace: the split partials go to a
 * file-scope device array of GDLA_DECODE_STATIC_SCRATCH_BYTES (16 MiB) that
 * every GPU which loads the library holds until the process exits.
 *  - It calls no cudaMalloc, cudaFree or allocating library routine.
 *  - Sizes whose split plan needs more scratch than the array holds (that is,
 *    gdla_decode_workspace_bytes(batch, num_kv_heads, max_seqlen_k, window) >
 *    GDLA_DECODE_STATIC_SCRATCH_BYTES) are rejected with GDLA_ERR_WORKSPACE
 *    before anything is launched.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current); make that first call
 *    before any stream capture.
 *  - Every call shares the one array and it keeps the last call's contents.
 *    Nothing needs clearing (each slot is written before it is read), but
 *    calls whose kernels overlap on the GPU (two streams, or two host threads
 *    on different streams) race on it: serialise them.
 */
#define GDLA_DECODE_STATIC_SCRATCH_BYTES (16u << 20)
GDLA_API gdla_status_t gdla_attn_decode_noalloc(const void *q_sig, const void *q_noise, const void *k_cache,
                                                const void *v_cache, const int32_t *cu_seqlens_k,
                                                int num_cache_rows, int max_seqlen_k, const float *lambda,
                                                const void *gate_logits, void *out, int batch,
                                                int num_kv_heads, int window, void *stream);

/*
 * Device-side failure word. Every wait inside the kernels is bounded (about
 * one second of SM clock); a wait that runs out makes its CTA wind down and
 * records a nonzero code here instead of hanging the GPU. This call
 * synchronises the current device, returns the recorded code (0 = none) and,
 * if `clear` is nonzero, resets it. Returns -1 if the device cannot be read.
 *
 * A nonzero code means that at least one CTA of some call since the word was
 * last cleared stopped early: output rows that CTA owned were NOT written
 * (they keep whatever the buffer held before), so the outputs of every call
 * enqueued since the last clear must be treated as invalid. Callers that
 * cannot rule out such a stall (e.g. a GPU shared with other heavy work)
 * should check this word before trusting a result.
 */
GDLA_API int gdla_device_error(int clear);

/*
 * Self-test of that failure path: launches one CTA (on `stream`) whose thread
 * waits, with the kernels' own bounded wait, on an mbarrier that nothing ever
 * arrives on. After the wait limit (about one second) it records
 * GDLA_SELFTEST_SITE in the device failure word and the kernel returns; the
 * context stays usable. No tensor is touched. Returns GDLA_OK once the kernel
 * is enqueued, GDLA_ERR_CUDA if the launch fails.
 */
#define GDLA_SELFTEST_SITE 0x30001
GDLA_API gdla_status_t gdla_selftest_wait_timeout(void *stream);

/* Static, human-readable name of a status code. */
GDLA_API const char *gdla_status_string(gdla_status_t status);

/* GDLA_VERSION of the loaded library. */
GDLA_API int gdla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GDLA_H */
