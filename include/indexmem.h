/*
 * indexmem.h -- C ABI of the IndexMem hot path on NVIDIA B200 (sm_100a).
 *
 * IndexMem keeps a bounded KV cache by learned eviction and compensates the
 * evicted tokens with a small latent memory. Sources, cited by page title and
 * section:
 *   [IM-sum]  "IndexMem: learned KV-cache eviction with latent memory",
 *             technical summary (gist.science), §1 Problem, §2.A Learnable
 *             indexer, §2.B Latent memory, §4 Experimental results.
 *   [IM-abs]  "IndexMem: Learned KV-Cache Eviction with Latent Memory for
 *             Long-Context LLM Inference", arXiv abstract.
 *   [MK-sum]  "MomentKV" technical summary (gist.science), Method §1 moment
 *             statistics, §2 first-order evicted output, §4 normalisation-
 *             corrected inference (the second compensation of the evicted
 *             tokens that this library computes: IMEM_READOUT_MOMENT).
 *
 * Conventions for every entry point
 *   - Tensor arguments are DEVICE pointers owned by the caller, row-major and
 *     contiguous, 16-byte aligned. The library never frees or retains them
 *     beyond the call (weights passed to imem_init are copied/repacked).
 *   - Work is enqueued asynchronously on the caller's cudaStream_t (passed as
 *     void* so this header needs no CUDA include; 0 = legacy default stream).
 *   - Arguments are validated on the host before anything is launched; an
 *     invalid call returns an error status and enqueues nothing.
 *   - Errors raised on the device (a bounded wait that ran out, an input
 *     value out of range) are recorded in the context and reported by
 *     imem_sync(). No entry point throws.
 *   - A context is bound to the device that was current at imem_init; calls
 *     must be made with that device current. Calls that share a context or a
 *     workspace must be ordered on one stream.
 *   - Calls on distinct contexts may come from several host threads at once:
 *     the library's only process-wide host state is the one-time setting of
 *     kernel attributes, per device, behind atomics (and a mutex where a
 *     shared-memory size only ever grows).
 *
 * Data types: IMEM_FP32 or IMEM_BF16 (the "model dtype") applies to X, Q, K, V,
 * the indexer weights, decode inputs, the retained cache and the decode output.
 * The memory state M, b and its weights W_phi, w_gate are always fp32.
 */
#ifndef INDEXMEM_H
#define INDEXMEM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  IMEM_OK = 0,
  IMEM_ERR_INVALID_ARG = 1,  /* null pointer, bad enum, negative size        */
  IMEM_ERR_SHAPE = 2,        /* sizes inconsistent (e.g. B > L, q_end > L)   */
  IMEM_ERR_ALIGN = 3,        /* a pointer is not 16-byte aligned             */
  IMEM_ERR_UNSUPPORTED = 4,  /* a dimension this build has no kernel for    */
  IMEM_ERR_CUDA = 5,         /* a CUDA runtime call failed                  */
  IMEM_ERR_TIMEOUT = 6,      /* a bounded device-side wait ran out          */
  IMEM_ERR_RANGE = 7         /* an input value out of the supported range:  */
                             /* an evicted index outside [0, L), or (fp32   */
                             /* inputs) a key or decay-weighted value of    */
                             /* the memory update beyond fp16's range       */
} imem_status;

typedef enum { IMEM_FP32 = 0, IMEM_BF16 = 1 } imem_dtype;

/* How the evicted tokens compensate the retained attention.
 *   IMEM_READOUT_GATED:  IndexMem's latent memory, o = o_attn + g(q) m(q)
 *                        ([IM-sum] §2.B).
 *   IMEM_READOUT_MOMENT: MomentKV's moment statistics ([MK-sum]): per KV head
 *                        the count n_e, the key and value sums s_k, s_v and
 *                        S^T = sum k v^T; the output mixes the retained
 *                        attention with a first-order estimate of the
 *                        evicted one (imem_decode_moment). */
typedef enum { IMEM_READOUT_GATED = 0, IMEM_READOUT_MOMENT = 1 } imem_readout;

/* Layer configuration.
 * Supported by this build: head_dim in {64,128}; idx_dim in {32,64};
 * idx_heads == n_q_heads (one indexer head per attention query head,
 * [IM-sum] §2.A: the multi-head queries are down-projected);
 * n_q_heads % n_kv_heads == 0 with a group of at most 8; hidden % 64 == 0;
 * mem_r in {16,32,...,128}; 0 < lambda <= 1.
 * readout = IMEM_READOUT_MOMENT requires mem_r == head_dim and lambda == 1 (the
 * statistics are plain sums); W_phi is then the identity and w_gate, eps and
 * gate_override are not used (imem_weights.W_phi and .w_gate may be NULL). */
typedef struct {
  int hidden;        /* H: hidden size of the model                        */
  int n_q_heads;     /* Hq                                                  */
  int n_kv_heads;    /* Hkv                                                 */
  int head_dim;      /* d                                                   */
  int idx_heads;     /* H_I, must equal n_q_heads                           */
  int idx_dim;       /* d_I: indexer dimension                              */
  int mem_r;         /* r: memory feature dimension                         */
  float lambda;      /* memory decay per evicted token                      */
  float eps;         /* readout denominator epsilon (1e-6 by default)       */
  int dtype;         /* imem_dtype                                          */
  float gate_override; /* NaN: learned gate g(q); otherwise g forced to it  */
  int readout;       /* imem_readout                                        */
} imem_config;

/* Layer weights, device pointers, read once by imem_init (repacked into the
 * context, so the caller may free them afterwards).
 *   W_idx_q [H_I, d, d_I]   model dtype  query down-projection per head
 *   W_idx_k [H, d_I]        model dtype  shared indexer key from hidden
 *   w_idx_g [H, H_I]        model dtype  head-gate logits from hidden
 *   W_phi   [r, d]          fp32         memory feature map phi(x) = W_phi x
 *   w_gate  [Hq, d]         fp32         readout gate g(q) = sigmoid(w_gate[h].q)
 * ([IM-sum] §2.A Architecture; §2.B Mechanism, slow weights.) */
typedef struct {
  const void* W_idx_q;
  const void* W_idx_k;
  const void* w_idx_g;
  const float* W_phi;
  const float* w_gate;
} imem_weights;

typedef struct imem_ctx imem_ctx;

/* Human-readable name of a status code (static string, never NULL). */
const char* imem_status_string(imem_status s);

/* Creates a context for one layer on the current device: validates cfg,
 * repacks the weights into the kernels' layouts (device memory owned by the
 * context) and allocates a 4-byte device error word. Synchronous.
 * Errors: INVALID_ARG (null cfg/weights/out), UNSUPPORTED (see imem_config),
 * ALIGN, CUDA. On error *out is set to NULL. */
imem_status imem_init(const imem_config* cfg, const imem_weights* w, imem_ctx** out);

/* Releases the context and its device memory (synchronises the device).
 * NULL is accepted. */
void imem_destroy(imem_ctx* ctx);

/* Bytes of caller-owned device workspace that score_and_evict, update_memory
 * and decode need for `batch` sequences of context length L and budget B.
 * The workspace must be zero-filled once before its first use (it holds
 * counters that every call leaves at zero again) and must be the same buffer
 * across the chunked score_and_evict calls of one prefill (it keeps the
 * indexer keys of earlier chunks). Errors: INVALID_ARG, SHAPE. */
imem_status imem_workspace_size(imem_ctx* ctx, int batch, int L, int B, size_t* bytes);

/* Indexer scoring with streaming per-key max, then (optionally) top-B
 * selection and compaction.  ([IM-sum] §2.A Function/Training: dense scores
 * A[s,t] pooled per key by a running max without forming the L x L matrix;
 * §1 token eviction; §4 90% eviction; §2.A pre-eviction by query ranges.)
 *
 * Inputs (model dtype): X [batch, L, H], Q [batch, L, Hq, d], K, V [batch, L, Hkv, d].
 * Only rows [q_begin, q_end) of X and Q are read by this call.
 * running_max [batch, L] fp32, in/out: for keys t in [q_begin, q_end) it is
 *   reset to -inf, then for all keys t < q_end
 *   I[t] = max(I[t], max_{s in [max(t,q_begin), q_end)} A[s,t]).
 *   Calling with consecutive ranges [0,c),[c,2c),...,[.,L) is chunked prefill.
 * finalize = 1 (requires q_end == L): selects R = the B largest I (ties to the
 *   lower position), writes idx_retained [batch, B] and idx_evicted
 *   [batch, L-B] (int32, ascending) and gathers K_ret/V_ret[:, :B] =
 *   K/V[R] into K_ret, V_ret [batch, cap, Hkv, d] (cap >= B; rows >= B are not
 *   written). finalize = 0 leaves those outputs untouched (may be NULL).
 * Errors: INVALID_ARG, SHAPE (B < 1, B > L, q ranges, cap < B), ALIGN,
 * UNSUPPORTED, CUDA. */
imem_status imem_score_and_evict(imem_ctx* ctx, int batch, int L, int B,
                                 const void* X, const void* Q, const void* K, const void* V,
                                 float* running_max, int q_begin, int q_end, int finalize,
                                 int32_t* idx_retained, int32_t* idx_evicted,
                                 void* K_ret, void* V_ret, int cap,
                                 void* workspace, void* stream);

/* The three steps of imem_score_and_evict as separate calls, for callers
 * that schedule or time them on their own (same arguments, workspace and
 * errors as there; imem_score_and_evict(..., finalize) equals
 * imem_indexer_features + imem_indexer_score (+ imem_select_compact)):
 *
 * imem_indexer_features ([IM-sum] §2.A Architecture): the indexer query
 *   q~_s = sum_h g_{s,h} RMSNorm(W_idx_q[h]^T q_{s,h}) / sqrt(d_I) and key
 *   k^_s = RMSNorm(W_idx_k^T x_s) of the tokens s in [q_begin, q_end), stored
 *   (bf16) in the workspace; running_max[:, q_begin:q_end] is reset to -inf.
 * imem_indexer_score ([IM-sum] §2.A Function/Training): for all keys t < q_end
 *   running_max[t] = max(running_max[t], max_{s in [max(t,q_begin), q_end)}
 *   q~_s . k^_t) over the features in the workspace (the features of keys
 *   t < q_begin from earlier ranges).
 * imem_select_compact ([IM-sum] §1, §4): the finalize step: selection of the B
 *   largest importances (ties to the lower position), idx_retained,
 *   idx_evicted and the gather into K_ret, V_ret; clears the workspace's
 *   decode tags. */
imem_status imem_indexer_features(imem_ctx* ctx, int batch, int L, const void* X, const void* Q,
                                  float* running_max, int q_begin, int q_end, void* workspace,
                                  void* stream);
imem_status imem_indexer_score(imem_ctx* ctx, int batch, int L, float* running_max, int q_begin,
                               int q_end, void* workspace, void* stream);
imem_status imem_select_compact(imem_ctx* ctx, int batch, int L, int B, const float* running_max,
                                const void* K, const void* V, int32_t* idx_retained,
                                int32_t* idx_evicted, void* K_ret, void* V_ret, int cap,
                                void* workspace, void* stream);

/* Latent-memory update from the evicted tokens ([IM-sum] §2.B Mechanism,
 * fast weights: decayed outer-product accumulation into M and stabiliser b).
 * For every sequence and KV head h, with phi(x) = W_phi x and the evicted
 * positions E[0..n) (ascending, from idx_evicted [batch, n_evicted]):
 *   M_h <- lambda^n M_h + sum_i lambda^(n-1-i) phi(k_{E[i],h}) v_{E[i],h}^T
 *   b_h <- lambda^n b_h + sum_i lambda^(n-1-i) phi(k_{E[i],h})
 * which equals the sequential update M <- lambda M + phi(k) v^T in order.
 * K, V [batch, L, Hkv, d] model dtype; M [batch, Hkv, r, d] fp32 in/out;
 * bstab [batch, Hkv, r] fp32 in/out. `chunk` = evicted tokens per work unit
 * (a multiple of 64, e.g. 512). n_evicted = 0 leaves M and b unchanged.
 * Precision and range: fp32 accumulation on the tensor cores. bf16 inputs:
 * the values enter as they are and each decay-weighted key as two bf16 halves
 * (hi + lo, about 16 significant bits, fp32's range). fp32 inputs: fp16
 * operands (keys converted, decay-weighted values rounded once), so keys and
 * values must stay below 65520 in magnitude (fp16 rounds larger ones to
 * infinity). Every evicted index must lie in [0, L). A value or index outside
 * that is reported by imem_sync as IMEM_ERR_RANGE (the row of an
 * out-of-range index is not read; M and bstab are then unspecified).
 * Errors: INVALID_ARG, SHAPE, ALIGN, CUDA; UNSUPPORTED for a context in
 * IMEM_READOUT_MOMENT mode (use imem_update_moments); RANGE via imem_sync. */
imem_status imem_update_memory(imem_ctx* ctx, int batch, int L, const void* K, const void* V,
                               const int32_t* idx_evicted, int n_evicted, int chunk,
                               float* M, float* bstab, void* workspace, void* stream);

/* One decode step over the retained cache with the gated memory readout
 * ([IM-sum] §2.B Output: o = o_attn + g(q) m(q); [IM-abs]).
 * q [batch, Hq, d]; k_new, v_new [batch, Hkv, d] are appended at row
 * cache_len[s] of K_ret/V_ret [batch, cap, Hkv, d] and cache_len [batch]
 * (int32, device) is incremented. Query head h uses KV head h/(Hq/Hkv):
 *   o_attn = softmax(q K^T / sqrt(d)) V over rows [0, cache_len] (new row incl.)
 *   u = W_phi q; m = M_kv^T u / (b_kv . u + eps); g = sigmoid(w_gate[h] . q)
 *   out = o_attn + g m            (out [batch, Hq, d], model dtype)
 * M, bstab are read only. A sequence whose cache is full (cache_len >= cap)
 * is left unchanged and its output row is not written; imem_sync reports it.
 * Ordering: the kernel is launched with programmatic dependent launch and
 * loads cache rows below cache_len - 1, b and M before it waits for the
 * previous kernel of the stream. It uses those copies only if the workspace's
 * decode tag of the sequence matches cache_len after the wait: the decode
 * steps (and imem_decode_online) set the tag from the length they leave;
 * a zero-filled workspace, imem_score_and_evict, imem_update_memory,
 * imem_update_moments and imem_prefill_evict_chunk clear it (0).
 * A caller that writes K_ret, V_ret,
 * cache_len, M or bstab by other means (its own kernels, copies,
 * imem_update_memory_static) between two decode steps on one workspace calls
 * imem_decode_invalidate on that workspace before the next step.
 * Errors: INVALID_ARG, SHAPE, ALIGN, CUDA; UNSUPPORTED for a context in
 * IMEM_READOUT_MOMENT mode (use imem_decode_moment). */
imem_status imem_decode(imem_ctx* ctx, int batch, const void* q, const void* k_new,
                        const void* v_new, void* K_ret, void* V_ret, int32_t* cache_len,
                        int cap, const float* M, const float* bstab, void* out,
                        void* workspace, void* stream);

/* Clears the decode tags of `batch` sequences in a workspace (stream-ordered,
 * no other effect), so that the next decode step on it loads nothing before
 * its launch-dependency wait. Call it after writing a retained cache, its
 * length or the memory state other than through this library (see
 * imem_decode, "Ordering"). Errors: INVALID_ARG, SHAPE, CUDA. */
imem_status imem_decode_invalidate(imem_ctx* ctx, int batch, void* workspace, void* stream);

/* Latent-memory update that allocates nothing (no counterpart in the paper: an
 * interface for callers that cannot allocate device memory, e.g. code running
 * inside a host framework's pre-planned memory arena or where cudaMalloc is not
 * allowed; imem_init and a workspace both need allocations such callers cannot
 * make). Same result as imem_update_memory, with no context: the caller passes
 * the dimensions, the decay lambda and W_phi [mem_r, head_dim] (fp32, device)
 * directly; K, V, idx_evicted, n_evicted, chunk, M and bstab as there. Its
 * tensor-core sums take fp16 operands for both dtypes (the register-pipelined
 * kernel, which needs no shared-memory position list), so keys and
 * decay-weighted values must stay below 65520 in magnitude.
 * Scratch: a fixed 8 MiB array in the library's device memory, held by every
 * GPU that loads the library until the process exits. batch * n_kv_heads *
 * head_dim * (head_dim + 1) * 4 bytes must fit in it (batch <= 15 at 8 KV heads
 * of dimension 128), otherwise IMEM_ERR_UNSUPPORTED and nothing is launched.
 * The first call on a device may load the library's device code there
 * (set-up, no allocation); make that first call before any stream capture.
 * Every call
 * writes the whole scratch region it uses before reading it, so nothing must
 * start at zero; calls that overlap on the GPU (any streams, any callers) race
 * on the shared array and must be serialised by the caller. The array's
 * device address is looked up on every call (no allocation), so a call stays
 * valid after cudaDeviceReset or in another context. Errors raised on the
 * device (a bounded wait that ran out, the range conditions of
 * imem_update_memory) go to one error word shared by all calls on the device;
 * imem_static_status reports and clears it. M and bstab are then unspecified.
 * Errors: INVALID_ARG, SHAPE, ALIGN, UNSUPPORTED, CUDA. */
imem_status imem_update_memory_static(int batch, int L, int n_kv_heads, int head_dim, int mem_r,
                                      float lambda, int dtype, const void* K, const void* V,
                                      const int32_t* idx_evicted, int n_evicted, int chunk,
                                      const float* W_phi, float* M, float* bstab, void* stream);

/* Waits for `stream`, then reports and clears the device error word that the
 * calls of imem_update_memory_static on the current device share (no
 * counterpart in the paper; allocates nothing): IMEM_OK, IMEM_ERR_TIMEOUT or
 * IMEM_ERR_RANGE, or IMEM_ERR_CUDA if a CUDA call fails. */
imem_status imem_static_status(void* stream);

/* Moment statistics of the evicted tokens ([MK-sum] Method §1), for a context
 * created with readout = IMEM_READOUT_MOMENT (else IMEM_ERR_UNSUPPORTED).
 * For every sequence and KV head h, over the evicted positions E[0..n):
 *   S_T_h += sum_i k_{E[i],h} v_{E[i],h}^T   (S_T [batch, Hkv, d, d] fp32: row =
 *                                            key dimension, column = value
 *                                            dimension, i.e. S^T of [MK-sum])
 *   s_k_h += sum_i k_{E[i],h},  s_v_h += sum_i v_{E[i],h}   ([batch, Hkv, d] fp32)
 *   n_e[s] += n_evicted                                     ([batch] fp32)
 * Other arguments, the workspace and the errors as imem_update_memory. The same
 * tensor-core kernel as the memory update computes S_T and s_k (identity map,
 * no decay); its loader warps add the value sums on the way. */
imem_status imem_update_moments(imem_ctx* ctx, int batch, int L, const void* K, const void* V,
                                const int32_t* idx_evicted, int n_evicted, int chunk,
                                float* S_T, float* s_k, float* s_v, float* n_e,
                                void* workspace, void* stream);

/* One decode step with the MomentKV readout ([MK-sum] Method §2, §4), for a
 * context created with readout = IMEM_READOUT_MOMENT (else
 * IMEM_ERR_UNSUPPORTED). q, k_new, v_new, K_ret, V_ret, cache_len, cap, out and
 * the workspace as imem_decode; S_T, s_k, s_v, n_e as imem_update_moments
 * (read only). Query head h uses KV head h/(Hq/Hkv):
 *   o_R = softmax(q K^T / sqrt(d)) V over rows [0, cache_len] (new row incl.),
 *   Z_R = sum of exp(q k^T / sqrt(d)) over the same rows,
 *   k_bar = s_k / n_e, v_bar = s_v / n_e, S~ = S - s_v s_k^T / n_e,
 *   f_E = v_bar + S~ q / (n_e sqrt(d)),
 *   Z_E = n_e exp(q . k_bar / sqrt(d))   (Jensen lower bound of the evicted
 *                                         partition function),
 *   w_R = Z_R / (Z_R + Z_E),  out = w_R o_R + (1 - w_R) f_E
 * and out = o_R where n_e = 0. Ordering as imem_decode, with S_T, s_k and
 * s_v in the place of M and bstab. Errors as imem_decode. */
imem_status imem_decode_moment(imem_ctx* ctx, int batch, const void* q, const void* k_new,
                               const void* v_new, void* K_ret, void* V_ret, int32_t* cache_len,
                               int cap, const float* S_T, const float* s_k, const float* s_v,
                               const float* n_e, void* out, void* workspace, void* stream);

/* Pre-eviction during chunked prefill ([IM-sum] §2.A: the indexer can evict
 * before the whole prefix has been processed, so the cache never holds more
 * than B tokens). Called once per query range, in order, the ranges contiguous
 * from 0: [q_begin, q_end) with q_end - q_begin <= chunk_max. Before a range the
 * cache holds n_R = min(B, q_begin) retained tokens; the candidates are those,
 * then the range's tokens. Their importance is pooled over the range's
 * queries by the streaming running max (retained keys keep the maximum of
 * earlier ranges; the range's keys are causal within it). If there are more
 * than B candidates, the B most important stay (ties to the lower position)
 * and the other n_ev = n_R + (q_end - q_begin) - B leave, in ascending
 * position order, into the memory: M, bstab updated as imem_update_memory does
 * with them (after all tokens evicted by earlier ranges).
 *   X, Q, K, V         as imem_score_and_evict ([batch, L, ...], model dtype).
 *   retained [batch, B] int32, out: the retained positions, ascending (the
 *                      first min(B, q_end) of each row valid after the call;
 *                      the workspace keeps the library's own copy).
 *   evicted [batch * chunk_max] int32, out: [batch, n_ev] packed, ascending.
 *   cand_importance    NULL or [batch, B + chunk_max] fp32, out: the candidates'
 *                      pooled importance before selection (row: n_R retained,
 *                      then the range's tokens; the rest of the row undefined).
 *   M, bstab           the memory, in/out (as imem_update_memory); mem_chunk as
 *                      its `chunk`.
 *   finalize = 1       (requires q_end == L): K_ret/V_ret[:, :min(B, L)] =
 *                      K/V[retained] as imem_score_and_evict does.
 *   workspace          imem_workspace_size_evict bytes, zero-filled once, the
 *                      same buffer for every range of one prefill (it keeps the
 *                      retained tokens' indexer keys and importances); it also
 *                      serves imem_decode.
 * Ordering: a range's selection, compaction (retained, evicted) and memory
 * update run on a second stream of the context, after this call's scoring
 * on `stream`, so that they overlap the next range's prologue (and the memory
 * update its scoring too). Every later call on the context makes its stream
 * wait for them: the next range's call for the compaction before its
 * scoring, every other call for all of it before it enqueues anything; the
 * call with finalize = 1 waits for its own before its compaction of K_ret,
 * V_ret (in the order of `stream`). Between two calls a caller that reads or
 * writes retained, evicted, M or bstab with its own work calls imem_join (or
 * imem_sync) on its stream first. A context runs one pre-eviction prefill at
 * a time: the call with q_begin = 0 starts a new one (the context keeps
 * which of the workspace's two candidate buffers the next range uses). The
 * second stream and its events are created at the first call: make it
 * before any stream capture, and capture whole sequences of calls up to the
 * one with finalize = 1 (a capture that ends with work still pending on the
 * second stream is unjoined).
 * Errors: INVALID_ARG, SHAPE (ranges, cap), ALIGN, CUDA; UNSUPPORTED for a
 * context in IMEM_READOUT_MOMENT mode. */
imem_status imem_workspace_size_evict(imem_ctx* ctx, int batch, int L, int B, int chunk_max,
                                      size_t* bytes);
imem_status imem_prefill_evict_chunk(imem_ctx* ctx, int batch, int L, int B, int chunk_max,
                                     const void* X, const void* Q, const void* K, const void* V,
                                     int q_begin, int q_end, int32_t* retained, int32_t* evicted,
                                     float* cand_importance, float* M, float* bstab,
                                     int mem_chunk, int finalize, void* K_ret, void* V_ret,
                                     int cap, void* workspace, void* stream);

/* Decode-time online eviction at a fixed budget ([IM-sum] §2.B: the memory
 * is updated online during inference as tokens leave the cache; §2.A: a key's
 * importance is the running maximum of its indexer scores over the queries
 * that arrive). The cache keeps B tokens in slots [0, B), in any order, with
 * per slot the indexer key khat_ret [batch, cap, 64] (bf16, d_I features then
 * zeros), the importance I_ret [batch, cap] (fp32) and the position pos_ret
 * [batch, cap] (int32); next_pos [batch] (int32) is the next token's position.
 * cap >= B + 1 (slot B is the step's scratch).
 *
 * imem_online_init: the state after a one-shot prefill (imem_score_and_evict
 * with finalize = 1, the same workspace, batch and L): khat_ret, I_ret,
 * pos_ret of the retained tokens (in idx_retained order, i.e. ascending
 * positions) and next_pos = L. running_max and idx_retained as left by that
 * call. Errors: INVALID_ARG, SHAPE (B > L, cap < B + 1), ALIGN, CUDA,
 * UNSUPPORTED (moment readout).
 *
 * imem_decode_online: one decode step. x_new [batch, H] is the new token's
 * hidden state, q, k_new, v_new as imem_decode; cache_len must be B on entry.
 *   1. out = imem_decode's output over slots [0, B) + the new token, with M,
 *      bstab before this step's eviction (the new token goes to slot B);
 *   2. the new token's indexer query q~ and key k^ are formed as in prefill
 *      (per-head projection of q, RMS norms, gates from x_new; both rounded to
 *      bf16); I_t = max(I_t, q~ . k^_t) for the cached tokens; the new token's
 *      importance is q~ . k^_new;
 *   3. the least important of the B + 1 tokens leaves (ties: the higher
 *      position leaves); M <- lambda M + phi(k) v^T, bstab <- lambda bstab +
 *      phi(k) with its key and value (every KV head); evicted [batch] (int32,
 *      out) receives its position;
 *   4. the new token takes the freed slot and the evicted token moves to
 *      slot B (nothing moves if the new token left itself): after the step
 *      slots [0, B) hold the retained tokens and slot B the one that left,
 *      with its row, indexer key, position and the importance it was chosen
 *      by, so that K_ret/V_ret/khat_ret/I_ret/pos_ret[:, :B + 1] are the
 *      B + 1 candidates of the step; cache_len returns to B; next_pos
 *      advances.
 * Streams: the new token's features (step 2 before the importances) need
 * neither the cache rows nor the memory, so they are computed on a second
 * stream owned by the context (created by imem_online_init or the first
 * step, which therefore belong before any stream capture; no device
 * memory), forked from `stream` and joined back into it by events before
 * the importances, the choice and the memory update (one kernel); under
 * stream capture this becomes two parallel branches of the graph.
 * Ordering: step 4 clears the workspace's decode tag of the sequence (slot e
 * and the memory changed after the attention step), so the next decode step
 * uses nothing it loaded before its launch-dependency wait.
 * imem_online_init does not write the cache state and leaves the tag as it is.
 * Errors: as imem_decode; UNSUPPORTED for the moment readout or more than
 * 16 KV heads; nothing is enqueued if an argument is invalid. */
imem_status imem_online_init(imem_ctx* ctx, int batch, int L, int B, const float* running_max,
                             const int32_t* idx_retained, const void* workspace, void* khat_ret,
                             float* I_ret, int32_t* pos_ret, int32_t* next_pos, int cap,
                             void* stream);
imem_status imem_decode_online(imem_ctx* ctx, int batch, int B, const void* x_new, const void* q,
                               const void* k_new, const void* v_new, void* K_ret, void* V_ret,
                               void* khat_ret, float* I_ret, int32_t* pos_ret, int32_t* next_pos,
                               int32_t* cache_len, int cap, float* M, float* bstab, void* out,
                               int32_t* evicted, void* workspace, void* stream);

/* Failure-path self-test (no counterpart in the papers): launches one CTA
 * that waits on a transaction barrier nothing completes, through the same
 * bounded wait every kernel of this library uses, with the given limit in SM
 * clock cycles (1 .. 2e9; the kernels use 2e9, about one second). The wait
 * runs out, the device records a timeout in the context's error word and the
 * next imem_sync returns IMEM_ERR_TIMEOUT (and clears it); the context stays
 * usable. Nothing faults and nothing waits without a limit.
 * Errors: INVALID_ARG (limit out of range), CUDA. */
imem_status imem_selftest_wait(imem_ctx* ctx, long long limit_cycles, void* stream);

/* Makes `stream` wait for work that the context still runs on its second
 * stream: the selection, compaction and memory update of the last range given
 * to imem_prefill_evict_chunk without finalize (no counterpart in the paper;
 * stream-ordered, no host synchronisation, nothing else enqueued). Every
 * other call of the library on the context does the same before its own
 * work; a caller needs it only before its own reads or writes of M, bstab,
 * the retained or the evicted positions between two pre-eviction calls.
 * Errors: INVALID_ARG, CUDA. */
imem_status imem_join(imem_ctx* ctx, void* stream);

/* Waits for the stream (after imem_join's wait for the context's second
 * stream), then reports the first error the device recorded for
 * this context since the last imem_sync (TIMEOUT for a bounded wait that ran
 * out, SHAPE for a decode into a full cache, RANGE for an input value out of
 * range) or a CUDA error, and clears it. */
imem_status imem_sync(imem_ctx* ctx, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* INDEXMEM_H */
