/*
 * diffattn.h -- C ABI of the B200 (sm_100a) differential attention library.
 *
 * The operator (DIFF Transformer attention) as the pages state it:
 *
 *   A_1 = softmax(Q_1 K_1^T / sqrt(d)),  A_2 = softmax(Q_2 K_2^T / sqrt(d))
 *   DiffAttn = (A_1 - lambda * A_2) V
 *     -- "Differential Attention (V2)" lesson (AI Engineering from Scratch, Phase 10),
 *        The Concept, "The difference idea"; "Attention Variants: Sliding Window, Sparse,
 *        Differential", Build It, Step 4 (diff_attention(Q1, K1, Q2, K2, V, lam)).
 *   lambda = exp(lq1 . lk1) - exp(lq2 . lk2) + lambda_init, one scalar per head
 *     -- "Differential Attention (V2)", The Concept; Key Terms, "lambda".
 *   lambda_init = 0.8 - 0.6 * exp(-0.3 * (depth - 1))
 *     -- skill-diff-attention-integrator, "Architecture diff".
 *   V1: head dim halved per branch, V of width 2d, per-head RMSNorm after the
 *       subtraction, then the (1 - lambda_init) output scale
 *     -- "Differential Attention (V2)", "V1 vs V2"; Key Terms, "Per-head RMSNorm";
 *        Hugging Face post on the DIFF Transformer, "How?" (GroupNorm per head).
 *   V2: twice the query heads over unchanged KV heads (GQA); query heads 2p and 2p+1
 *       are the two branches of pair p and share one KV head; no per-head norm
 *     -- "Differential Attention (V2)", "V1 vs V2"; compatibility table ("GQA: yes").
 *   Causal: query i sees keys j <= i
 *     -- "Attention Variants", Build It, Step 1 (causal_mask).
 *
 * Entry points: diffattn_lambda; diffattn_fwd_prefill (V1 / V2, bf16 or f32; causal, full,
 * chunked, sliding window) and diffattn_fwd_prefill_varlen (packed sequences);
 * diffattn_fwd_decode (V2), diffattn_fwd_decode_v1, diffattn_fwd_decode_paged (block
 * table), diffattn_fwd_decode_static, diffattn_decode_workspace_size; diffattn_bwd_prefill,
 * diffattn_bwd_workspace_size, diffattn_fwd_prefill_train, diffattn_bwd_prefill_saved,
 * diffattn_lambda_bwd (training); diffattn_selftest_timeout
 * (the bounded-wait path), diffattn_selftest_exp2 (the FMA-pipe 2^x),
 * diffattn_debug_bounds_violations (the bounds-checked build); diffattn_version,
 * diffattn_status_string.
 *
 * Conventions for every entry point
 *   - Pointers are DEVICE pointers unless marked "host". The caller owns every buffer;
 *     the library allocates no device memory, frees nothing and keeps no pointer after a
 *     call. (Its own objects: the 16 MiB array of diffattn_fwd_decode_static, and one CUDA
 *     stream with two events per device for the tensor-core backward's second stream.)
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).
 *     The library never synchronizes.
 *   - Arguments are validated on the host before anything is launched. On any error
 *     status nothing is launched and no output is written.
 *   - CUDA launch failures return DIFFATTN_ERR_CUDA. Conditions a kernel detects while
 *     running (a bounded wait that gave up) are written to `dev_status` (a device int,
 *     nullable), which the caller reads after synchronizing; 0 means success, otherwise
 *     a diffattn_status value. Kernels never trap.
 *   - No C++ exception crosses this boundary.
 *   - Element strides are in elements, not bytes. The innermost dimension is always
 *     contiguous (stride 1).
 */
#ifndef DIFFATTN_H_
#define DIFFATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DIFFATTN_OK = 0,
  DIFFATTN_ERR_INVALID_ARG = -1, /* null pointer, negative size, inconsistent shape */
  DIFFATTN_ERR_UNSUPPORTED = -2, /* valid request this build does not implement */
  DIFFATTN_ERR_MISALIGNED = -3,  /* pointer or stride violates the alignment rules */
  DIFFATTN_ERR_WORKSPACE = -4,   /* workspace missing or smaller than required */
  DIFFATTN_ERR_CUDA = -5,        /* a CUDA runtime / driver call failed */
  DIFFATTN_ERR_TIMEOUT = -6      /* a kernel's bounded wait gave up (dev_status only) */
} diffattn_status;

typedef enum { DIFFATTN_F32 = 0, DIFFATTN_BF16 = 1 } diffattn_dtype;
typedef enum { DIFFATTN_V1 = 1, DIFFATTN_V2 = 2 } diffattn_variant;

/* Library ABI version (major * 100 + minor). */
int diffattn_version(void);

/* Static description of a status code. Never NULL. */
const char* diffattn_status_string(int status);

/*
 * diffattn_lambda -- the lambda re-parameterisation, on the device.
 *
 *   lambda_out[h] = exp(lq1[h,:] . lk1[h,:]) - exp(lq2[h,:] . lk2[h,:]) + lambda_init
 *   lambda_init   = 0.8 - 0.6 * exp(-0.3 * (depth - 1))
 * ("Differential Attention (V2)", The Concept; skill-diff-attention-integrator,
 * "Architecture diff"). lambda may be negative; nothing is clamped.
 *
 * lq1, lk1, lq2, lk2 : float32 [n_heads, dim], row-major, 16-byte aligned
 *                      (n_heads = V1 heads, or V2 pairs)
 * lambda_out         : float32 [n_heads]
 * lambda_init_out    : float32 [1] or NULL
 * depth              : layer depth, >= 1
 * Sizes: 1 <= n_heads <= 65535, 1 <= dim <= 4096.
 * Arithmetic: fp32 dot products in a fixed order, fp32 expf.
 */
int diffattn_lambda(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                    int n_heads, int dim, int depth, float* lambda_out, float* lambda_init_out,
                    void* stream);

/*
 * Prefill parameters.
 *
 * V1 (variant = DIFFATTN_V1): n_q_heads = n_kv_heads = H differential heads,
 *   head_dim = d per branch (d = 64 for bf16; any 1..128 multiple of 4 for f32).
 *   q    : [B, N, H, 2, d]   branch 1 at index 0, branch 2 at index 1 (contiguous, so
 *                            each (token, head) row holds q1 then q2)
 *   k    : [B, Nk, H, 2, d]
 *   v    : [B, Nk, H, 2d]
 *   out  : [B, N, H, 2d]
 *   lambda: [H]. apply_norm = 1 applies the per-head RMSNorm (over the 2d channels,
 *   eps = norm_eps, unit gain) and then multiplies by (1 - lambda_init[0]).
 * V2 (variant = DIFFATTN_V2): n_q_heads = Hq (even), n_kv_heads = Hkv with Hq/Hkv even;
 *   head_dim = d (128 for bf16; any 1..128 multiple of 4 for f32).
 *   q    : [B, N, Hq, d]     query heads 2p, 2p+1 = branches 1, 2 of pair p
 *   k, v : [B, Nk, Hkv, d]   query head h reads KV head h / (Hq / Hkv)
 *   out  : [B, N, Hq/2, d]
 *   lambda: [Hq/2]. apply_norm must be 0.
 * Strides (elements) are {batch, token, head}; the branch axis (V1) and the channel
 * axis are contiguous. bf16: q/k/v base pointers 16-byte aligned and every stride a
 * multiple of 8 elements (TMA rules); f32: 16-byte aligned, strides multiple of 4.
 * out must not alias q, k or v.
 * Nk = kv_seqlen (0 reads as N) >= N. The N queries are the LAST N of the Nk positions
 * (chunked prefill: a chunk of new tokens attends the earlier ones and itself), so query i
 * sits at position i + Nk - N.
 * causal = 1: query i attends keys 0..i + Nk - N; causal = 0: every query attends all Nk
 * keys. window = W > 0 (causal only) keeps the last W of those keys (a causal sliding
 * window: keys i + Nk - N - W + 1 .. i + Nk - N); window = 0 keeps all.
 * Nk < N, window < 0, or window > 0 with causal = 0 return DIFFATTN_ERR_INVALID_ARG.
 */
typedef struct {
  int32_t variant;    /* diffattn_variant */
  int32_t dtype;      /* diffattn_dtype of q, k, v and out */
  int32_t batch;      /* B >= 0 */
  int32_t seqlen;     /* N >= 0 queries */
  int32_t n_q_heads;  /* V1: H; V2: Hq */
  int32_t n_kv_heads; /* V1: H; V2: Hkv */
  int32_t head_dim;   /* d per branch */
  int32_t causal;     /* 1 = causal, 0 = full */
  int32_t apply_norm; /* V1: 1 = RMSNorm + (1 - lambda_init) scale; V2: 0 */
  float norm_eps;     /* RMSNorm epsilon (1e-5) */
  int64_t q_strides[3];
  int64_t k_strides[3];
  int64_t v_strides[3];
  int64_t o_strides[3];
  int32_t kv_seqlen;  /* Nk >= N keys; 0 = N */
  int32_t window;     /* causal sliding window in keys; 0 = none */
} diffattn_prefill_params;

/*
 * diffattn_fwd_prefill -- fused causal/full differential attention forward.
 * One pass over the keys; both attention maps stay on chip (never written to memory).
 * bf16: tcgen05 tensor-core kernel, fp32 accumulation, P rounded to bf16 as an MMA
 * operand only; fp32: exact-fp32 SIMT kernel.
 *
 * lambda      : float32 [n_units] (V1 heads / V2 pairs), device
 * lambda_init : float32 [1], device; read only when apply_norm = 1 (may be NULL otherwise)
 * dev_status  : nullable device int, see the conventions above
 * B == 0 or N == 0 launches nothing and returns DIFFATTN_OK.
 */
int diffattn_fwd_prefill(const diffattn_prefill_params* p, const void* q, const void* k,
                         const void* v, const float* lambda, const float* lambda_init, void* out,
                         int* dev_status, void* stream);

/*
 * diffattn_fwd_prefill_varlen -- diffattn_fwd_prefill over a variable-length batch: S
 * sequences of different lengths packed back to back in one tensor per operand (no
 * padding), as a serving system batches prompts of different lengths.
 *   p->batch      : S, the number of sequences
 *   p->seqlen     : total packed query rows (the token extent of q and out)
 *   p->kv_seqlen  : total packed key rows of k and v (0 reads as p->seqlen)
 *   strides       : the batch strides are ignored; token and head strides as for the
 *                   fixed-length call, so q is [total_q, H, 2, d] (V1) / [total_q, Hq, d]
 *                   (V2), k and v likewise over total_k rows, out over total_q rows
 *   cu_seqlens_q  : int32 [S + 1], device: sequence s owns query (and output) rows
 *                   cu_seqlens_q[s] .. cu_seqlens_q[s+1] - 1
 *   cu_seqlens_k  : int32 [S + 1], device: sequence s owns key rows
 *                   cu_seqlens_k[s] .. cu_seqlens_k[s+1] - 1
 *   max_seqlen_q  : HOST int, >= every sequence's query count (sizes the launch)
 * Each sequence is one fixed-length problem: its nq queries are the last nq of its nk
 * positions (nq <= nk; nq = nk for a plain prompt, nq < nk for a chunk after cached
 * tokens), with p->causal and p->window as for diffattn_fwd_prefill.
 * A sequence whose offsets are inconsistent (negative or decreasing counts, nq > nk,
 * rows past the packed extents, nq > max_seqlen_q) is skipped -- its output rows are not
 * written -- and DIFFATTN_ERR_INVALID_ARG is written to dev_status. Host-side errors as
 * for diffattn_fwd_prefill; NULL offsets return DIFFATTN_ERR_INVALID_ARG.
 */
int diffattn_fwd_prefill_varlen(const diffattn_prefill_params* p, const int32_t* cu_seqlens_q,
                                const int32_t* cu_seqlens_k, int max_seqlen_q, const void* q,
                                const void* k, const void* v, const float* lambda,
                                const float* lambda_init, void* out, int* dev_status,
                                void* stream);

/*
 * diffattn_bwd_prefill -- gradients of diffattn_fwd_prefill (training). The pages present
 * lambda and the projections as learnable in a pre-trained layer ("Differential Attention
 * (V2)", Key Terms, "lambda"; "V1 vs V2"); the gradient is fixed by the forward:
 *   dV = (A_1 - lambda A_2)^T dO,  dS_1 = A_1 o (dO V^T - delta_1),
 *   dS_2 = -lambda A_2 o (dO V^T - delta_2),  dQ_b = dS_b K_b / sqrt(d),
 *   dK_b = dS_b^T Q_b / sqrt(d),  dlambda = -sum dO o (A_2 V),
 * with dO the gradient reaching O = A_1 V - lambda A_2 V (V1: through the per-head RMSNorm
 * and the (1 - lambda_init) scale) and delta_b = rowsum(dO o (A_b V)). The softmax maps are
 * recomputed, never stored. V2's two branches and the pairs of a GQA group add into the
 * gradient of their shared KV head.
 *
 * p, q, k, v, lambda, lambda_init : exactly as for the forward call (f32 or bf16 inputs,
 *              kv_seqlen and window as there); head_dim <= 128, a multiple of 4
 * dout       : dL/dy in the layout and dtype of the forward's out (p->o_strides)
 * dq, dk, dv : float32, DENSE row-major in the shapes of q, k and v (V1 [B,N,H,2,d],
 *              [B,Nk,H,2,d], [B,Nk,H,2d]; V2 [B,N,Hq,d], [B,Nk,Hkv,d], [B,Nk,Hkv,d]),
 *              16-byte aligned; fully overwritten
 * dlambda    : float32 [units] (V1 heads / V2 pairs), overwritten; feed it to
 *              diffattn_lambda_bwd for the four lambda vectors
 * workspace  : >= diffattn_bwd_workspace_size(p) bytes, 256-byte aligned (per row: two
 *              log-sum-exps, two deltas, the row's dlambda share, and dO: fp32 on the exact
 *              path, bf16 for V1 on the tensor cores)
 * Arithmetic: bf16 V2 with d = 128 and bf16 V1 with d = 64 run on the tensor cores (fp32
 * accumulation; the MMA operands P_1 - lambda P_2, dS_b and, for V1, dO rounded to bf16, as
 * the forward rounds its P operand). V1's statistics pass forms O and its norm's backward
 * from probability operands split into two bf16 parts (error ~2^-18), because dlambda
 * through the norm keeps only the small part of O_2 orthogonal to O. Every other case (fp32
 * inputs, other d) runs exact fp32 on the CUDA cores. Both are deterministic (no atomics:
 * dQ rows, dK/dV rows and dlambda are each summed by one thread group in a fixed order).
 * Streams (tensor-core path): the dK/dV and dQ kernels run side by side, the dQ kernel on a
 * stream the library creates once per device, forked from `stream` and joined back to it
 * (events) before the call's last kernel. The call therefore stays ordered on `stream` and
 * can be captured into a CUDA graph. Host threads calling concurrently are serialized while
 * they enqueue; while one thread captures such a call, other threads must not call the
 * tensor-core backward on the same device until that capture ends (their dQ kernel would
 * join the capture).
 * Errors as for diffattn_fwd_prefill, plus DIFFATTN_ERR_WORKSPACE.
 */
int diffattn_bwd_workspace_size(const diffattn_prefill_params* p, size_t* bytes);
int diffattn_bwd_prefill(const diffattn_prefill_params* p, const void* q, const void* k,
                         const void* v, const float* lambda, const float* lambda_init,
                         const void* dout, float* dq, float* dk, float* dv, float* dlambda,
                         void* workspace, size_t workspace_bytes, int* dev_status, void* stream);

/*
 * diffattn_fwd_prefill_train -- diffattn_fwd_prefill for training (V2, bf16, d = 128): the
 * same output, plus what the backward needs so that diffattn_bwd_prefill_saved does not
 * recompute the forward. (The pages' training setting: "Differential Attention (V2)", Key
 * Terms, "lambda", and "V1 vs V2"; the statistics are the softmax's own, Build It, Step 1.)
 *
 * p, q, k, v, lambda, out : as for diffattn_fwd_prefill (fixed-length batches; causal, full,
 *              chunked and sliding window as there)
 * o2         : the branch-2 output O_2 / l_2 = A_2 V of every (query, pair), in out's
 *              layout (p->o_strides) and dtype, 16-byte aligned, overwritten
 * lse        : float32 [B, Hq/2, N, 2], dense, 16-byte aligned: per (batch entry, pair,
 *              query) the log-sum-exps of both branches in the log2 domain,
 *              log2 sum_j 2^(s_b,j log2(e) / sqrt(d)) with s_b the raw scores; overwritten
 * Returns DIFFATTN_ERR_UNSUPPORTED for V1, fp32 or d != 128 (those train through
 * diffattn_bwd_prefill, which recomputes); otherwise errors as for diffattn_fwd_prefill.
 */
int diffattn_fwd_prefill_train(const diffattn_prefill_params* p, const void* q, const void* k,
                               const void* v, const float* lambda, void* out, void* o2, float* lse,
                               int* dev_status, void* stream);

/*
 * diffattn_bwd_prefill_saved -- diffattn_bwd_prefill from diffattn_fwd_prefill_train's saved
 * output: the per-row deltas are taken from out and o2 (delta_2 = dO . O_2 / l_2,
 * delta_1 = dO . (out + lambda O_2 / l_2)) and the log-sum-exps from lse, instead of a
 * recompute of the forward. Same gradients, layouts, workspace size
 * (diffattn_bwd_workspace_size), arithmetic, determinism and second stream as the
 * tensor-core path of diffattn_bwd_prefill; V2, bf16, d = 128 only.
 *
 * out, o2, lse : the training forward's outputs for the same p, q, k, v and lambda; out,
 *              o2 and dout share the layout p->o_strides
 * Errors as for diffattn_bwd_prefill; DIFFATTN_ERR_UNSUPPORTED outside V2 bf16 d = 128.
 */
int diffattn_bwd_prefill_saved(const diffattn_prefill_params* p, const void* q, const void* k,
                               const void* v, const float* lambda, const void* out, const void* o2,
                               const float* lse, const void* dout, float* dq, float* dk, float* dv,
                               float* dlambda, void* workspace, size_t workspace_bytes,
                               int* dev_status, void* stream);

/*
 * diffattn_lambda_bwd -- gradients of the four lambda vectors from dL/dlambda:
 *   dlq1 = g e1 lk1, dlk1 = g e1 lq1, dlq2 = -g e2 lk2, dlk2 = -g e2 lq2,
 *   e_b = exp(lq_b . lk_b), g = dlambda[h]   (lambda_init depends on depth only).
 * Vectors float32 [n_heads, dim] as for diffattn_lambda (device); outputs overwritten.
 */
int diffattn_lambda_bwd(const float* lq1, const float* lk1, const float* lq2, const float* lk2,
                        int n_heads, int dim, const float* dlambda, float* dlq1, float* dlk1,
                        float* dlq2, float* dlk2, void* stream);

/*
 * Decode parameters (bf16 only). V2 (diffattn_fwd_decode) below; V1 uses the same struct
 * with the layouts given at diffattn_fwd_decode_v1.
 *   q       : [B, Hq, d]        one new query token per batch entry
 *   k_cache : [B, L, Hkv, d]    L = max_kv_len (cache capacity)
 *   v_cache : [B, L, Hkv, d]    same strides as k_cache
 *   kv_len  : int32 [B] or NULL (NULL = every entry holds L keys); 0 <= kv_len[b] <= L
 *   out     : [B, Hq/2, d]
 * The new query attends every cached key 0 .. kv_len[b]-1 (its own key is expected to be
 * in the cache already). Hq / Hkv must be 8 and d = 128 in this build.
 * Strides (elements): q {batch, head}, kv {batch, token, head}, out {batch, pair};
 * 16-byte aligned base pointers, strides multiples of 8 elements.
 */
typedef struct {
  int32_t variant;    /* DIFFATTN_V2 (diffattn_fwd_decode) or DIFFATTN_V1 (_v1) */
  int32_t dtype;      /* DIFFATTN_BF16 */
  int32_t batch;      /* B >= 0 */
  int32_t max_kv_len; /* L >= 0 */
  int32_t n_q_heads;  /* Hq */
  int32_t n_kv_heads; /* Hkv */
  int32_t head_dim;   /* d */
  int32_t num_splits; /* KV splits per (batch, KV head); 0 = chosen by the library */
  int64_t q_strides[2];
  int64_t kv_strides[3];
  int64_t o_strides[2];
} diffattn_decode_params;

/*
 * diffattn_decode_workspace_size -- device workspace bytes diffattn_fwd_decode (V2) or
 * diffattn_fwd_decode_v1 (V1, by p->variant) needs for these parameters (written to *bytes, a HOST pointer). The workspace holds the
 * per-split partial softmax states; its contents need no initialisation.
 */
int diffattn_decode_workspace_size(const diffattn_decode_params* p, size_t* bytes);

/*
 * diffattn_fwd_decode -- split-KV differential decode. Each (batch, KV head, split)
 * block streams its slice of the cache once with 128-bit loads and scores it for all
 * query heads of the GQA group (both branches of every pair), keeping one running
 * (max, sum, output) state per query head. A second, small kernel merges the per-split
 * states of each head and applies O = O_1/l_1 - lambda * O_2/l_2 per pair.
 *   -- "Differential Attention (V2)", "V1 vs V2": V2 keeps the KV heads of the base model
 *      and its two branches read the same cache, so decoding loads the KV cache once per
 *      step (V1 loads the value cache twice); The Concept, "The difference idea", for
 *      O = (A_1 - lambda A_2) V with one query row per step.
 *
 * lambda     : float32 [Hq/2], device
 * workspace  : device buffer of at least diffattn_decode_workspace_size() bytes,
 *              256-byte aligned; calls sharing a workspace must not overlap in time
 * dev_status : nullable device int
 */
int diffattn_fwd_decode(const diffattn_decode_params* p, const void* q, const void* k_cache,
                        const void* v_cache, const int32_t* kv_len, const float* lambda, void* out,
                        void* workspace, size_t workspace_bytes, int* dev_status, void* stream);

/*
 * diffattn_fwd_decode_v1 -- split-KV differential decode for V1 ("Differential Attention
 * (V2)", "V1 vs V2": each V1 head has two query/key branches of width d and one value
 * of width 2d; the per-head RMSNorm and the (1 - lambda_init) scale follow the
 * difference). Each (batch, head, split) block streams its slice of the cache once --
 * the value rows serve both branches -- and keeps one running (max, sum, output) per
 * branch; a second kernel merges the splits, forms O_1/l_1 - lambda O_2/l_2, and applies
 * the norm and scale. fp32 arithmetic throughout (no bf16 rounding of probabilities).
 *
 * Parameters: diffattn_decode_params with variant = DIFFATTN_V1, dtype = DIFFATTN_BF16,
 * n_q_heads = n_kv_heads = H (differential heads), head_dim = d = 64 in this build.
 *   q       : [B, H, 2, d]      branch 2 at +d inside each head's row
 *   k_cache : [B, L, H, 2, d]   branch 2's key at +d inside each cached row
 *   v_cache : [B, L, H, 2d]     same strides as k_cache
 *   kv_len  : int32 [B] or NULL (NULL = L); the query attends keys 0 .. kv_len[b]-1
 *   out     : [B, H, 2d]
 * Strides (elements): q {batch, head}, kv {batch, token, head}, out {batch, head};
 * 16-byte aligned base pointers, strides multiples of 8 elements.
 *   lambda      : float32 [H], device
 *   lambda_init : float32 [1], device; read only when apply_norm = 1 (may be NULL otherwise)
 *   apply_norm  : 1 = RMSNorm over the 2d channels (eps = norm_eps >= 0, unit gain) and
 *                 x (1 - lambda_init); 0 = the plain difference
 *   workspace   : >= diffattn_decode_workspace_size(p) bytes, 256-byte aligned
 * kv_len[b] = 0 gives a zero output row. Errors as for diffattn_fwd_decode; a V2 parameter
 * set returns DIFFATTN_ERR_INVALID_ARG.
 */
int diffattn_fwd_decode_v1(const diffattn_decode_params* p, const void* q, const void* k_cache,
                           const void* v_cache, const int32_t* kv_len, const float* lambda,
                           const float* lambda_init, int apply_norm, float norm_eps, void* out,
                           void* workspace, size_t workspace_bytes, int* dev_status,
                           void* stream);

/*
 * Paged KV cache (a block table over a shared page pool, the layout serving systems use
 * for their caches; the pages name vLLM / SGLang integration as in progress). Page i of
 * the pool holds page_size consecutive cached tokens of one batch entry, for every head.
 * Token t of batch entry b lives in row t % page_size of page block_table[b][t / page_size].
 */
typedef struct {
  int32_t page_size;         /* tokens per page: a power of two, 1 .. 65536 */
  int32_t num_pages;         /* pages in the pool (>= 1) */
  int32_t max_pages_per_seq; /* columns of block_table; page_size * this >= max_kv_len */
  int32_t reserved;          /* must be 0 */
  int64_t page_strides[3];   /* {page, token in page, head}, elements, for both pools */
} diffattn_paged_kv;

/*
 * diffattn_fwd_decode_paged -- diffattn_fwd_decode (p->variant = DIFFATTN_V2) or
 * diffattn_fwd_decode_v1 (DIFFATTN_V1) over a paged cache. Same kernels, arithmetic and
 * results as the contiguous entry points: only the address of each cached row differs.
 *   p           : as for the contiguous call; p->kv_strides is ignored
 *   pk          : HOST pointer, the pool geometry above
 *   k_pages     : V2 [num_pages, page_size, Hkv, d]; V1 [num_pages, page_size, H, 2, d]
 *   v_pages     : V2 [num_pages, page_size, Hkv, d]; V1 [num_pages, page_size, H, 2d]
 *                 (both with pk->page_strides; strides multiples of 8 elements)
 *   block_table : int32 [B, max_pages_per_seq], device, row-major; entries for pages past
 *                 kv_len[b] are never read
 *   kv_len      : int32 [B] or NULL (NULL = max_kv_len), clamped to [0, max_kv_len]
 *   lambda_init, apply_norm, norm_eps : V1 as for diffattn_fwd_decode_v1; V2: apply_norm = 0
 *   workspace   : >= diffattn_decode_workspace_size(p) bytes, 256-byte aligned
 * A block-table entry outside [0, num_pages) that a kernel meets writes
 * DIFFATTN_ERR_INVALID_ARG to dev_status; the rows of that page read as zeros (no access
 * outside the pool). Host-side errors as for the contiguous entry points.
 */
int diffattn_fwd_decode_paged(const diffattn_decode_params* p, const diffattn_paged_kv* pk,
                              const void* q, const void* k_pages, const void* v_pages,
                              const int32_t* block_table, const int32_t* kv_len,
                              const float* lambda, const float* lambda_init, int apply_norm,
                              float norm_eps, void* out, void* workspace, size_t workspace_bytes,
                              int* dev_status, void* stream);

/*
 * diffattn_fwd_decode_static -- diffattn_fwd_decode without a caller-provided workspace.
 * (A convenience of this library; the pages describe no counterpart.)
 *
 * For callers that cannot allocate device memory when they call: for example a serving
 * loop that runs from a device-memory budget fixed at start-up and must not allocate per
 * request, or a plugin whose host application owns all device memory through its own
 * pool. The per-split partial states live in a 16 MiB array inside the library instead.
 * This entry point itself allocates nothing (no cudaMalloc / cudaFree, no allocating
 * library call).
 *
 * Arguments, layouts and results are those of diffattn_fwd_decode. Differences:
 *   - num_splits = 0 picks the automatic split count when its partial states fit in the
 *     16 MiB array, otherwise the largest count that fits; an explicit num_splits whose
 *     states do not fit, or a problem that does not fit even unsplit (about
 *     B * Hq > 32000 at d = 128), returns DIFFATTN_ERR_WORKSPACE before any CUDA call.
 *   - The array is one per device and shared by every call on that device, and it keeps
 *     the previous call's contents. Nothing in it needs to start at zero (each call writes
 *     every state it reads), but two calls whose kernels overlap on the GPU (for example
 *     on two streams without ordering between them) race on it: order them.
 *   - The array's device memory is committed when the library's module for it is loaded
 *     on a device: under CUDA's default lazy module loading that is the first call of this
 *     entry point with that device current (with CUDA_MODULE_LOADING=EAGER, when the
 *     library's context starts); it is then held until the process exits. That first call
 *     also looks up the array's device address (cudaGetSymbolAddress) and caches it per
 *     device and context (a context created after a device reset gets a fresh lookup).
 *     So make one warm-up call on each device at start-up, before sizing a memory pool
 *     from the free memory that is left and before any stream capture.
 */
int diffattn_fwd_decode_static(const diffattn_decode_params* p, const void* q,
                               const void* k_cache, const void* v_cache, const int32_t* kv_len,
                               const float* lambda, void* out, int* dev_status, void* stream);

/*
 * diffattn_selftest_timeout -- exercises the kernels' bounded-wait path on purpose.
 * (A diagnostic of this library, for tests; it computes nothing.)
 *
 * Every mbarrier wait in the kernels above gives up after a time bound and then reports
 * DIFFATTN_ERR_TIMEOUT through the status word instead of hanging the GPU. This entry
 * point launches one block of 128 threads that waits, with the same wait routine, for a
 * barrier phase that nothing completes, bounded by timeout_ms instead of the kernels'
 * 2-second bound. The wait runs out, the block writes DIFFATTN_ERR_TIMEOUT to *dev_status
 * (left untouched if it already holds a non-zero code) and returns; the CUDA context stays
 * usable.
 *
 *   dev_status  device int, required.
 *   timeout_ms  1 .. 10000.
 * Returns DIFFATTN_ERR_INVALID_ARG for a null status pointer or a timeout outside that
 * range, DIFFATTN_ERR_CUDA if the launch fails, else DIFFATTN_OK (the timeout itself is
 * reported on the device, when the block finishes).
 */
int diffattn_selftest_timeout(int* dev_status, int timeout_ms, void* stream);

/*
 * diffattn_selftest_exp2 -- evaluates the V2 prefill's FMA-pipe 2^x beside CUDA's exp2f.
 * (A diagnostic of this library, for tests; the pages fix no precision for the
 * exponentials, only the max-subtracted softmax of "Differential Attention (V2)",
 * Build It, Step 1, whose terms are 2^x with x <= 0 in the log2 domain.)
 *
 * The V2 prefill evaluates a quarter of its exponentials on the FMA pipe instead of the
 * MUFU unit: x = n + f with n = rint(x) (exact in fp32), 2^f from a degree-4 polynomial
 * with minimax relative error on [-0.5, 0.5] (a Remez-exchange fit: the error
 * equioscillates at six points, |error| <= 2.7e-6), then n added to the exponent field;
 * x is clamped at -125 first, so 2^x for x <= -125 (a masked key, x = -inf) is 2^-125.
 * This entry point runs that routine, on pairs as the kernel does, over n inputs.
 *
 *   x      device float[n], inputs.
 *   y      device float[n], out: the polynomial 2^x.
 *   y_ref  device float[n], out: exp2f(x) on the same device.
 *   n      >= 0 (0 launches nothing).
 * Returns DIFFATTN_ERR_INVALID_ARG for n < 0 or a null pointer with n > 0,
 * DIFFATTN_ERR_CUDA if the launch fails, else DIFFATTN_OK (asynchronous on `stream`).
 */
int diffattn_selftest_exp2(const float* x, float* y, float* y_ref, int n, void* stream);

/*
 * diffattn_debug_bounds_violations -- the bounds-checked build's count of skipped accesses.
 * (A diagnostic of this library, for tests; the pages have no counterpart.)
 *
 * The library can be built a second time with every raw global-memory access of its kernels
 * (the ones that do not go through a TMA tensor map, which bounds its own copies) checked
 * against the extent of the tensor it touches, as computed on the host from the call's
 * shapes and strides: libdiffattn_debug.so (python -m differential_attention_05_b200.build
 * --debug). An access outside its tensor is skipped, DIFFATTN_ERR_INVALID_ARG goes to the
 * call's dev_status (when given), and a device-wide counter is incremented; nothing traps.
 * This entry point copies that counter to *count (a HOST int) and resets it; it waits for
 * the device to finish its work first (cudaMemcpy and cudaDeviceSynchronize).
 *
 * Returns DIFFATTN_OK in the bounds-checked build, DIFFATTN_ERR_UNSUPPORTED (with *count =
 * 0) in the normal build, DIFFATTN_ERR_INVALID_ARG for a null count, DIFFATTN_ERR_CUDA if
 * the copy fails.
 */
int diffattn_debug_bounds_violations(int* count);

#ifdef __cplusplus
}
#endif

#endif /* DIFFATTN_H_ */
