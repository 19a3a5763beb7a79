/*
 * tg.h -- C ABI of the TokenGate pruned-prefill library (libtokengate.so).
 *
 * The library implements, as CUDA kernels for NVIDIA B200 (sm_100a), the
 * inference hot path of TokenGate learned token pruning:
 *
 *   gate layer L:  score every prunable token with a small MLP  (tg_gate_score)
 *                  keep the top-K document tokens + every question token
 *                                                                (tg_topk_select)
 *                  compact the kept rows in their original order (tg_gather)
 *   layers > L:    token-gated causal GQA attention over the kept rows
 *                                                                (tg_gated_attention)
 *                  one whole decoder layer on the kept rows      (tg_pruned_prefill_layer)
 *
 * The method is described on the TokenGate pages; citations below name the
 * page and its section:
 *   [R] "TokenGate and T2Quant: a close reading" (MessageDaily blog)
 *   [K] "Stanford-Berkeley TokenGate" explainer (kg.zhiyong.dev)
 *   [M] MarkTechPost TokenGate article (farwalk translation)
 *
 * Conventions shared by every entry point
 *   - Pointers marked "device" are caller-owned device memory on the current
 *     CUDA device; the library never frees them.  Pointers marked "host" are
 *     host memory.  Scratch memory, where an op needs any, is passed in as a
 *     workspace (size from tg_workspace_bytes); the library allocates nothing.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every
 *     call only enqueues work on it and returns without synchronising, except
 *     tg_check_device_error.
 *   - Matrices are row-major and contiguous unless a leading dimension (in
 *     elements) is given.  bf16 operands and their leading dimensions must be
 *     16-byte aligned (TG_ERR_ALIGN otherwise).
 *   - Argument and shape errors are detected on the host before anything is
 *     enqueued and return a status without touching the stream.  A failed
 *     launch returns TG_ERR_CUDA.  Conditions only the device can see (a
 *     prunable mask whose count disagrees with n_prunable, a bounded wait that
 *     expired) set a sticky device error word instead of faulting; read it
 *     with tg_check_device_error.
 *   - tg_last_error() returns a human-readable detail string for the last
 *     failing call on the calling host thread.
 */
#ifndef TG_H_
#define TG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TG_OK = 0,
  TG_ERR_INVALID_ARG = 1,     /* null pointer, negative size or budget, bad enum   */
  TG_ERR_SHAPE = 2,           /* inconsistent sizes (e.g. m != min(k, np) + n - np) */
  TG_ERR_ALIGN = 3,           /* pointer or leading dimension not 16-byte aligned   */
  TG_ERR_UNSUPPORTED = 4,     /* valid but not implemented (e.g. head_dim 96)       */
  TG_ERR_WORKSPACE = 5,       /* workspace missing or smaller than required         */
  TG_ERR_CUDA = 6,            /* a CUDA runtime call or kernel launch failed        */
  TG_ERR_DEVICE_TIMEOUT = 7,  /* a bounded device-side wait expired                 */
  TG_ERR_DEVICE_CHECK = 8     /* a device-side consistency check failed             */
} tg_status;

typedef enum { TG_F32 = 0, TG_BF16 = 1 } tg_dtype;

/* Static description of a status code. */
const char* tg_status_string(int status);

/* Detail text for the last failing call on this host thread ("" if none). */
const char* tg_last_error(void);

/*
 * Synchronises `stream`, then reads and clears the device error word of the
 * current device.  Returns TG_OK, TG_ERR_DEVICE_TIMEOUT, TG_ERR_DEVICE_CHECK or
 * TG_ERR_CUDA (if the synchronisation itself failed).  `detail` (host, may be
 * NULL) receives the raw word: bits 0-7 the failing site, bits 8-31 a payload.
 */
int tg_check_device_error(void* stream, uint32_t* detail);

/*
 * For tests of the timeout path only (the TokenGate pages have no counterpart).
 * Waits on a flag in global memory that another CTA sets -- the attention
 * kernel's split-merge ready count, where the second half of a split query
 * block waits for the first half's partial result -- give up after
 * limit_ns nanoseconds (default 1 s) and wait for the count to reach
 * merge_ready_target (default: the protocol's own value).  A test sets a
 * short limit and a target no CTA reaches, so the wait runs out: the waiting
 * CTA then writes no output, records TG_ERR_DEVICE_TIMEOUT in the device error
 * word (read with tg_check_device_error) and returns; the context stays
 * usable.  0 restores a default.  Applies to the current device; synchronous.
 */
int tg_debug_set_flag_wait(uint64_t limit_ns, uint32_t merge_ready_target);

/*
 * Gate scores ([R] §4.1 "Gate module"; [M] "how does learned token pruning
 * work"): for every token j,
 *     x_j = RMSNorm(h_j) * norm_w            (eps = norm_eps)
 *     s_j = w2 . SiLU(W1 x_j + b1) + b2      if prunable[j]
 *     s_j = 0                                otherwise (question tokens)
 * and sumsq = sum over prunable j of s_j^2 (fp32, summed in a fixed order,
 * so it is deterministic), used by tg_gather for the sequence-wise RMS norm.
 *
 *   hidden   device, dtype [n][d_model]   post-attention residual of layer L
 *   norm_w   device, fp32 [d_model] or NULL (all ones)
 *   w1       device, dtype [h][d_model]   (nn.Linear layout: one row per unit)
 *   b1       device, fp32 [h] or NULL (zeros)
 *   w2       device, fp32 [h]
 *   prunable device, uint8 [n]            1 = document token, 0 = question token
 *   scores   device, fp32 [n]  out
 *   sumsq    device, fp32 [1]  out
 *   ws       device workspace (16-byte aligned) of at least
 *            tg_workspace_bytes(TG_OP_GATE_SCORE, n, 0, d_model, h, NULL)
 *            bytes; its contents on entry do not matter.
 * bf16 with d_model % 8 == 0 and h % 16 == 0, h <= 256 runs on the tcgen05
 * tensor cores (a non-NULL norm_w is folded into W1 in bf16 first); other
 * shapes and fp32 run on CUDA cores (h <= 1024) and do not use ws.
 */
int tg_gate_score(const void* hidden, int dtype, int64_t n, int32_t d_model,
                  const float* norm_w, float norm_eps,
                  const void* w1, const float* b1, const float* w2, float b2, int32_t h,
                  const uint8_t* prunable, float* scores, float* sumsq,
                  void* ws, size_t ws_bytes, void* stream);

/*
 * Masked top-K selection ([R] §4.1 "Top-K selector": S = top-K(b) U N).
 * Keeps exactly k' = min(k, n_prunable) prunable tokens -- those with the
 * largest score, where equal scores (and -0 == +0) are broken towards the
 * lower index and NaN ranks below -inf -- plus every non-prunable token.
 * The kept indices are written in ascending order, so the compacted sequence
 * keeps the original causal order.  Integer-exact and deterministic.
 *
 *   scores     device, fp32 [n]   (selection is on the raw scores; the
 *              sequence RMS norm is a positive scale and does not change it)
 *   prunable   device, uint8 [n]
 *   n_prunable number of nonzero entries of prunable (known to the caller from
 *              the prompt layout; checked on the device, a mismatch sets the
 *              device error word and the output is then unspecified but never
 *              written past m entries)
 *   k          budget, >= 0 (k >= n_prunable keeps everything)
 *   kept_idx   device, int32 [m] out, m = min(k, n_prunable) + n - n_prunable
 * Needs no workspace: the whole selection runs in one thread-block cluster.
 */
int tg_topk_select(const float* scores, const uint8_t* prunable, int64_t n, int64_t n_prunable,
                   int64_t k, int32_t* kept_idx, int64_t m, void* stream);

/*
 * tg_gate_score followed by tg_topk_select, with the selection's first radix
 * digit counted by the scoring kernel ([R] §4.1 "Gate module" and "Top-K
 * selector"): when the tensor cores score and the prompt is long enough for
 * the cluster selector (n > 4096), the scoring kernel's epilogue also counts
 * the order-preserving keys of the prunable scores by their top 11 bits, and
 * the selector reads the threshold's first digit off that histogram instead
 * of building one.  The outputs equal tg_gate_score then tg_topk_select on
 * the same stream: scores, sumsq and the kept indices (bit-exact, ascending).
 *   arguments        as tg_gate_score and tg_topk_select (m = min(k,
 *                    n_prunable) + n - n_prunable)
 *   ws               device workspace of tg_workspace_bytes(TG_OP_GATE_SELECT,
 *                    n, 0, d_model, h, NULL) bytes, 16-byte aligned
 *   flags            0, or TG_WS_KEPT_ZERO: the caller promises that ws is
 *                    zero-filled or exactly as the previous successful call
 *                    with this flag left it; the call then issues no memset
 *                    (a memset between two kernels ends their programmatic
 *                    launch overlap) and leaves the counters it uses at zero
 *                    again.  After a call that reported an error, clear ws
 *                    (or pass 0) before the next one.  With 0 the contents of
 *                    ws on entry do not matter.
 * Errors: those of tg_gate_score and tg_topk_select; TG_ERR_INVALID_ARG for an
 * unknown flag.
 */
#define TG_WS_KEPT_ZERO 1u
int tg_gate_score_select(const void* hidden, int dtype, int64_t n, int32_t d_model,
                         const float* norm_w, float norm_eps, const void* w1, const float* b1,
                         const float* w2, float b2, int32_t h, const uint8_t* prunable,
                         int64_t n_prunable, int64_t k, float* scores, float* sumsq,
                         int32_t* kept_idx, int64_t m, void* ws, size_t ws_bytes, uint32_t flags,
                         void* stream);

/*
 * Compaction of the kept rows ([R] §4.1 three-stage forward: pruned tokens
 * never enter the layers above L) plus the per-row inputs of gated attention:
 *     hidden_kept[r] = hidden[kept_idx[r]]            (bit-exact copy)
 *     pos[r]         = kept_idx[r]                    (original position)
 *     bias[r]        = s[kept_idx[r]] / rms           (importance b_j, [R] §4.1;
 *                      rms = sqrt(sumsq / n_prunable + seq_eps); 0 for question tokens)
 *     ratio[r]       = log(r + 1) / log(max(2, kept_idx[r] + 1))
 *                      (the log m_i / log max(2, p_i) factor of the temperature,
 *                       [R] §4.1 "temperature scaling")
 *   hidden      device, dtype [n][d_model];  hidden_kept device, dtype [m][d_model] out
 *   kept_idx    device, int32 [m], ascending, values in [0, n)
 *   scores      device, fp32 [n];  sumsq device, fp32 [1] (from tg_gate_score)
 *   pos/bias/ratio  device, int32/fp32/fp32 [m] out (any may be NULL to skip)
 */
int tg_gather(const void* hidden, int dtype, int64_t n, int32_t d_model,
              const int32_t* kept_idx, int64_t m,
              const float* scores, const float* sumsq, int64_t n_prunable, float seq_eps,
              void* hidden_kept, int32_t* pos, float* bias, float* ratio, void* stream);

/*
 * tg_gather fused with a row-wise RMSNorm of the gathered rows: the kept rows
 * are read once and written twice, as the bit-exact residual copy
 * hidden_kept[r] = hidden[kept_idx[r]] and as the normalised row
 *     x_norm[r] = hidden_kept[r] / sqrt(mean(hidden_kept[r]^2) + norm_eps) * norm_w
 * that the first projection of the layer above reads ([R] §4.1 three-stage
 * forward: the compacted rows go straight into the layers above the gate).
 * pos, bias and ratio are written exactly as tg_gather writes them.
 *   hidden .. ratio   as tg_gather;  norm_w device fp32 [d_model] or NULL (ones)
 *   x_norm            device dtype [m][d_model] out, 16-byte aligned
 * The normalised rows are rounded to dtype, as the layer's own RMSNorm does.
 */
int tg_gather_rmsnorm(const void* hidden, int dtype, int64_t n, int32_t d_model,
                      const int32_t* kept_idx, int64_t m,
                      const float* scores, const float* sumsq, int64_t n_prunable, float seq_eps,
                      const float* norm_w, float norm_eps, void* hidden_kept, void* x_norm,
                      int32_t* pos, float* bias, float* ratio, void* stream);

/*
 * Token-gated causal GQA attention over the m kept rows ([R] §4.1 "token-gated
 * attention", "head-wise gain", "temperature scaling"; [K]; [M]).  For query
 * head h, KV head g = h / (hq / hkv), kept row r and key c <= r:
 *     l_rc = head_temp[h] * ratio[r] * sm_scale * (q_r . k_c) + head_gain[h] * bias[c]
 *     out_r = sum_c softmax_c(l_r.) v_c
 * (the gate value g_j = softmax(b_j) multiplies exp(z_ij) in the attention
 * weights, which is the same as adding b_j to the logits; the gain acts on
 * that log-space term; the temperature rescales the content logit).
 *
 *   q    device, dtype, row r of head h at q + r*ldq + h*head_dim
 *   k, v device, dtype, row r of KV head g at k + r*ldk + g*head_dim (same for v/ldv)
 *   out  device, dtype, row r of head h at out + r*ldo + h*head_dim
 *   bias device fp32 [m] or NULL (0);  ratio device fp32 [m] or NULL (1)
 *   head_gain, head_temp  device fp32 [hq] (values after softplus)
 *   lse  device fp32 [hq][m] out (natural-log sum of exp of l) or NULL
 *   ws   device workspace of tg_workspace_bytes(TG_OP_ATTENTION, 0, m, 0, 0, shape)
 *        bytes (shape gives dtype, hq, hkv, head_dim), 16-byte aligned, or NULL.
 *        When the causal work is about one wave of the GPU, the longest query
 *        blocks are split over two CTAs whose partial results meet in ws; with
 *        ws NULL (or smaller than required) nothing is split.  The size depends
 *        on the SM count of the current device and is 0 when no split is made.
 * head_dim in {64, 128}; hq % hkv == 0.  bf16 with an even group size hq / hkv
 * runs on the tcgen05 tensor cores (fp32 softmax and accumulation): each CTA
 * there serves two query heads of one KV head, so that every K/V tile it loads
 * feeds two score tiles.  fp32 inputs, and bf16 with an odd group size (1, 3,
 * 5, ...: MHA included), run on a CUDA-core kernel in full fp32 instead -- the
 * same results within the attention tolerance, but tens of times slower at the
 * workloads' sizes (it is there for correctness, not speed).  The split
 * workspace is ignored on that path.
 */
int tg_gated_attention(const void* q, int64_t ldq, const void* k, int64_t ldk,
                       const void* v, int64_t ldv, int dtype, int64_t m,
                       int32_t hq, int32_t hkv, int32_t head_dim,
                       const float* bias, const float* head_gain, const float* head_temp,
                       const float* ratio, float sm_scale,
                       void* out, int64_t ldo, float* lse, void* ws, size_t ws_bytes, void* stream);

/*
 * Backward of tg_gated_attention ([R] §4.1 engineering notes: the biased
 * attention kernel also returns the bias gradient to the scorer).  With
 * l_rc, P = softmax_c(l) and out as in the forward and upstream dout:
 *     dP_rc = dout_r . v_c,   dl_rc = P_rc (dP_rc - dout_r . out_r)
 *     dq_r  = sum_c dl_rc head_temp[h] ratio[r] sm_scale k_c
 *     dk_c, dv_c: sums over the query heads of c's KV head and over rows
 *             of dl_rc head_temp[h] ratio[r] sm_scale q_r and of P_rc dout_r
 *     dbias_c = sum over all heads h of head_gain[h] sum_r dl_rc
 *     dgain_h = sum_{r,c} dl_rc bias[c];  dtemp_h = sum_{r,c} dl_rc ratio[r] sm_scale (q_r . k_c)
 *   q, k, v, out, dout  device, dtype, strided rows as in the forward
 *   lse   device fp32 [hq][m], the forward's (natural-log) log-sum-exp
 *   dq    device fp32 [m][hq*head_dim];  dk, dv device fp32 [m][hkv*head_dim]
 *   dbias device fp32 [m] or NULL;  dgain, dtemp device fp32 [hq] or NULL
 *   ws    device workspace of tg_workspace_bytes(TG_OP_ATTENTION_BWD, 0, m, 0, 0,
 *         shape) bytes, 16-byte aligned
 * P is recomputed from lse.  bf16 operands with 16-byte aligned bases and row
 * strides (and 16-byte aligned dq, dk, dv, bias) run on the tensor cores, with
 * P and dS rounded to bf16 for the MMAs and fp32 accumulation; fp32 operands
 * and other bf16 layouts run on CUDA cores in fp32.  Deterministic either way:
 * no atomics on values, every cross-block sum is taken in a fixed order (the
 * query heads of a KV head add their dk / dv partials in head order).
 * head_dim in {64, 128}; hq % hkv == 0.  Errors: TG_ERR_INVALID_ARG (null
 * pointer, m <= 0, bad heads or dtype), TG_ERR_UNSUPPORTED (head_dim, m >= 2^31),
 * TG_ERR_SHAPE (leading dimension), TG_ERR_WORKSPACE, TG_ERR_ALIGN (workspace).
 */
int tg_gated_attention_backward(const void* q, int64_t ldq, const void* k, int64_t ldk,
                                const void* v, int64_t ldv, const void* out, int64_t ldo,
                                const void* dout, int64_t lddo, int dtype, int64_t m,
                                int32_t hq, int32_t hkv, int32_t head_dim, const float* bias,
                                const float* head_gain, const float* head_temp, const float* ratio,
                                float sm_scale, const float* lse, float* dq, float* dk, float* dv,
                                float* dbias, float* dgain, float* dtemp,
                                void* ws, size_t ws_bytes, void* stream);

/*
 * One decode step of token-gated attention over the gated KV cache ([R] §4.1
 * Gate module: tokens produced while decoding are not prunable and score 0;
 * §4.1 engineering notes: at decode time the gate term is an additive mask on
 * the attention logits; §4.1 temperature scaling).  The new token's query
 * attends to all `length` cached rows, the last of which is its own key:
 *     l_c = head_temp[h] * ratio * sm_scale * (q_h . k_c) + head_gain[h] * bias[c]
 *     out_h = sum_c softmax_c(l) v_c
 *   q      device, dtype, [hq][head_dim] (the new token's query rows, after RoPE)
 *   k, v   device, dtype, cache row c of KV head g at k + c*ldk + g*head_dim
 *          (same for v / ldv): the kept prompt rows, then the generated ones
 *   bias   device fp32 [length] or NULL (0): the kept prompt rows' importance
 *          b_c, 0 for generated rows
 *   head_gain, head_temp  device fp32 [hq] (values after softplus)
 *   ratio  the step's temperature ratio (tg_decode_temperature_ratio)
 *   out    device, dtype, [hq][head_dim];  lse device fp32 [hq] or NULL
 *   ws     device workspace of tg_workspace_bytes(TG_OP_DECODE, 0, length, 0, 0,
 *          shape) bytes (shape gives hq, hkv, head_dim), 16-byte aligned;
 *          required (the cache is split into chunks whose partial results are
 *          merged in it).  The size depends on the SM count of the device.
 * head_dim in {64, 128}; hq % hkv == 0 with at most 8 query heads per KV head;
 * length <= 262144; cache rows 16-byte aligned.  bf16 or fp32 inputs, fp32 arithmetic on the
 * CUDA cores (the step reads the cache once and is bound by memory).  A bf16
 * cache with bias NULL or 16-byte aligned streams through shared memory by TMA
 * (one CTA per SM over all KV heads); fp32 caches, an unaligned bias, or
 * TG_DECODE_SIMT=1 in the environment take the split-KV kernel that loads the
 * cache into registers.  Both give the same results within fp32 rounding.
 */
int tg_gated_decode_attention(const void* q, const void* k, int64_t ldk, const void* v, int64_t ldv,
                              int dtype, int64_t length, int32_t hq, int32_t hkv, int32_t head_dim,
                              const float* bias, const float* head_gain, const float* head_temp,
                              float ratio, float sm_scale, void* out, float* lse,
                              void* ws, size_t ws_bytes, void* stream);

/*
 * Temperature ratio of the query generated at decode step t (0-based) after a
 * prompt of n_prompt tokens of which m_kept were kept ([R] §4.1 temperature
 * scaling, read as for a kept prompt row): the query is kept row m_kept + t at
 * original position n_prompt + t, so
 *     ratio = log(m_kept + t + 1) / log(max(2, n_prompt + t + 1)).
 * Host function; returns 0 for negative arguments.
 */
float tg_decode_temperature_ratio(int64_t m_kept, int64_t n_prompt, int64_t t);

/* Weights of one Qwen3-style decoder layer (device pointers). */
typedef struct {
  const float* w_in_norm;    /* fp32 [d_model]                                  */
  const void* w_qkv;         /* dtype [(hq + 2*hkv)*head_dim][d_model]: q rows, then k, then v */
  const float* w_q_norm;     /* fp32 [head_dim] (used when qk_norm != 0)        */
  const float* w_k_norm;     /* fp32 [head_dim] (used when qk_norm != 0)        */
  const void* w_o;           /* dtype [d_model][hq*head_dim]                    */
  const float* w_post_norm;  /* fp32 [d_model]                                  */
  const void* w_gate_up;     /* dtype [2*d_ff][d_model]: gate rows, then up rows */
  const void* w_down;        /* dtype [d_model][d_ff]                           */
  const float* head_gain;    /* fp32 [hq]  softplus(gamma), per head            */
  const float* head_temp;    /* fp32 [hq]  softplus(sigma), per head            */
} tg_layer_weights;

typedef struct {
  int32_t dtype;             /* TG_F32 or TG_BF16 */
  int32_t d_model, hq, hkv, head_dim, d_ff;
  int32_t qk_norm;           /* per-head RMSNorm of q and k before RoPE (Qwen3) */
  float rope_theta;          /* rotate-half RoPE base */
  float norm_eps;            /* RMSNorm epsilon */
} tg_layer_shape;

/*
 * One decoder layer above the gate, run on the m kept rows only ([R] §4.1
 * three-stage forward; [M]: the layers above L process only the kept tokens
 * and never create KV for pruned ones):
 *   x = RMSNorm(h) ; q,k,v = x Wqkv^T ; (q,k per-head RMSNorm) ;
 *   RoPE(q,k) at the ORIGINAL positions pos ; a = gated attention (see above,
 *   sm_scale = 1/sqrt(head_dim)) ; h += a Wo^T ; y = RMSNorm(h) ;
 *   h += (SiLU(y Wg^T) * (y Wu^T)) Wd^T
 * Intermediates are rounded to the layer dtype between steps.
 *   hidden_kept device dtype [m][d_model], updated in place
 *   pos  device int32 [m];  bias/ratio device fp32 [m] or NULL (0 / 1)
 *   ws   device workspace of tg_workspace_bytes(TG_OP_LAYER, 0, m, 0, 0, shape) bytes
 * With bias = NULL, ratio = NULL and pos = 0..m-1 this is the plain unpruned
 * layer (used for the layers below the gate).
 */
int tg_pruned_prefill_layer(const tg_layer_weights* weights, const tg_layer_shape* shape,
                            void* hidden_kept, const int32_t* pos, const float* bias,
                            const float* ratio, int64_t m, void* ws, size_t ws_bytes, void* stream);

/* Parts of a decoder layer (tg_gather_prefill_layer's `part`). */
enum { TG_LAYER_ATTENTION = 1, TG_LAYER_MLP = 2, TG_LAYER_FULL = 3 };

/*
 * The two halves of tg_pruned_prefill_layer, for the gate layer L itself
 * ([R] §4.1 Gate module and three-stage forward; [K] "tying the mechanism
 * together"; [M] "how does learned token pruning work": the gate scores layer
 * L's normalised post-attention residual, so layer L's attention runs on every
 * token and its MLP, a row-wise step, only on the kept ones):
 *   tg_layer_attention_block:  h += Attn(RMSNorm(h)) Wo^T   (steps up to the
 *                              O projection; the post-attention residual)
 *   tg_layer_mlp_block:        h += (SiLU(y Wg^T) * (y Wu^T)) Wd^T, y = RMSNorm(h)
 *                              with w_post_norm
 * Arguments as tg_pruned_prefill_layer (the MLP half reads only w_post_norm,
 * w_gate_up and w_down; the attention half every other weight), with the
 * same workspace size.  Calling the two in a row is the whole layer.
 */
int tg_layer_attention_block(const tg_layer_weights* weights, const tg_layer_shape* shape, void* hidden,
                             const int32_t* pos, const float* bias, const float* ratio, int64_t m,
                             void* ws, size_t ws_bytes, void* stream);
int tg_layer_mlp_block(const tg_layer_weights* weights, const tg_layer_shape* shape, void* hidden,
                       int64_t m, void* ws, size_t ws_bytes, void* stream);

/*
 * tg_gather followed by a layer part on the kept rows, with the gather folded
 * into that part's first RMSNorm ([R] §4.1 three-stage forward: the kept rows
 * are compacted and go straight into the layers above): one pass reads
 * hidden[kept_idx[r]], writes it to hidden_kept[r] (bit-exact) together with
 * pos, bias and ratio exactly as tg_gather does, and writes the normalised row
 * the part's first projection reads; the rest of the part then runs on the
 * kept rows as tg_pruned_prefill_layer (part TG_LAYER_FULL: the whole gated
 * layer above the gate) or tg_layer_mlp_block (part TG_LAYER_MLP: the gate
 * layer's own MLP half) would.  The result equals tg_gather then that call.
 *   hidden, n, kept_idx, m, scores, sumsq, n_prunable, seq_eps, hidden_kept,
 *   pos, bias, ratio   as tg_gather (dtype and d_model from shape); the full
 *                      layer needs pos; bias / ratio may be NULL (0 / 1 in
 *                      attention, and not written)
 *   ws                 as tg_pruned_prefill_layer for m rows
 */
int tg_gather_prefill_layer(const tg_layer_weights* weights, const tg_layer_shape* shape, int part,
                            const void* hidden, int64_t n, const int32_t* kept_idx, int64_t m,
                            const float* scores, const float* sumsq, int64_t n_prunable, float seq_eps,
                            void* hidden_kept, int32_t* pos, float* bias, float* ratio,
                            void* ws, size_t ws_bytes, void* stream);

/*
 * The same layer over a batch of requests whose kept rows are concatenated
 * (varlen batching; [R] §4.1 three-stage forward, per request): rows
 * seg_rows[r] .. seg_rows[r+1]-1 of hidden_kept, pos, bias and ratio belong to
 * request r.  Every step but attention is row-wise and runs once over all
 * seg_rows[nseg] rows; attention runs request by request, so a row only sees
 * keys of its own request (its causal prefix among them).
 *   seg_rows  host int64 [nseg + 1], seg_rows[0] = 0, non-decreasing (a
 *             request may have no rows)
 *   ws        device workspace of tg_layer_varlen_workspace_bytes(shape,
 *             seg_rows, nseg) bytes, 16-byte aligned
 * Equals tg_pruned_prefill_layer called on each request's rows on its own.
 */
int tg_pruned_prefill_layer_varlen(const tg_layer_weights* weights, const tg_layer_shape* shape,
                                   void* hidden_kept, const int32_t* pos, const float* bias,
                                   const float* ratio, const int64_t* seg_rows, int32_t nseg,
                                   void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes of tg_pruned_prefill_layer_varlen (0 for an invalid request). */
size_t tg_layer_varlen_workspace_bytes(const tg_layer_shape* shape, const int64_t* seg_rows, int32_t nseg);

/*
 * Row-wise linear layer of the decoder layer above, exported so that each of
 * its GEMMs can be called (and timed) on its own:
 *   epilogue TG_EPI_STORE     y = x W^T
 *   epilogue TG_EPI_RESIDUAL  y = y + x W^T          (y holds the residual on entry)
 *   epilogue TG_EPI_SWIGLU    y = SiLU(x Wg^T) * (x Wu^T), where W is [2*n_out][k_in]
 *                             with the gate rows first and the up rows after them
 *   x device dtype, row r at x + r*ldx, k_in columns
 *   w device dtype [n_out or 2*n_out][k_in] (nn.Linear layout)
 *   y device dtype, row r at y + r*ldy, n_out columns
 * bf16 runs on the tcgen05 tensor cores (k_in % 8 == 0; n_out % 32 == 0, or
 * n_out % 128 == 0 for SwiGLU); fp32 and other bf16 shapes run on CUDA cores,
 * where SwiGLU is not offered (TG_ERR_UNSUPPORTED).
 */
enum { TG_EPI_STORE = 0, TG_EPI_RESIDUAL = 1, TG_EPI_SWIGLU = 2 };
int tg_linear(const void* x, int64_t ldx, const void* w, void* y, int64_t ldy, int dtype,
              int64_t m, int32_t n_out, int32_t k_in, int epilogue, void* stream);

enum { TG_OP_GATE_SCORE = 0, TG_OP_LAYER = 1, TG_OP_ATTENTION = 2, TG_OP_DECODE = 3, TG_OP_ATTENTION_BWD = 4,
       TG_OP_GATE_SELECT = 5 };

/* Workspace bytes needed by an op: TG_OP_GATE_SCORE and TG_OP_GATE_SELECT use n, d_model and h;
 * TG_OP_LAYER and TG_OP_ATTENTION use m and shape (TG_OP_ATTENTION reads its
 * dtype, hq, hkv and head_dim); TG_OP_DECODE uses m = the cache length and
 * shape's hq, hkv and head_dim; TG_OP_ATTENTION_BWD uses m and shape's hq, hkv and head_dim.  Returns 0 for an invalid request, and 0 for
 * TG_OP_ATTENTION when the attention needs no workspace. */
size_t tg_workspace_bytes(int op, int64_t n, int64_t m, int32_t d_model, int32_t h, const tg_layer_shape* shape);

/*
 * tg_gate_score without a workspace argument, for callers that cannot
 * allocate device memory when they score a prompt (a serving runtime that owns
 * all of HBM through its own pool and passes the library only the request's
 * tensors, a plugin interface with no workspace hook, or a latency-critical
 * path that must avoid cudaMalloc's device-wide synchronisation).  The TokenGate
 * pages have no counterpart of this call; it computes exactly what
 * tg_gate_score computes, with the same arguments minus ws / ws_bytes.
 *
 * Scratch lives in a fixed array compiled into the library,
 * tg_gate_score_noalloc_scratch_bytes() bytes (2 MiB + 64 KiB) on every device
 * that loads the library, held until the process exits.  Only the tensor-core
 * path of tg_gate_score (see there) uses scratch: calls that take it and whose
 * scratch would not fit (about n/32 + 2*d_model*h bytes, e.g. n up to 2^20
 * tokens with d_model*h up to 2^20) are rejected with TG_ERR_UNSUPPORTED
 * before anything is enqueued; calls on the CUDA-core path (fp32, or shapes the
 * tensor cores do not take) need none and have no size limit from it.  The
 * call allocates and frees nothing.
 *
 * The first call on each device looks up the array's device address (with
 * that device current) and caches it; make that first call before any stream
 * capture.  All calls on a device share the one array and leave the last
 * call's contents in it (the part that must start at zero is cleared by each
 * call on its stream), so calls whose executions overlap on the GPU -- on
 * different streams, or from several host threads -- race on it and must be
 * serialised by the caller.
 */
int tg_gate_score_noalloc(const void* hidden, int dtype, int64_t n, int32_t d_model,
                          const float* norm_w, float norm_eps,
                          const void* w1, const float* b1, const float* w2, float b2, int32_t h,
                          const uint8_t* prunable, float* scores, float* sumsq, void* stream);

/* Size in bytes of the per-device scratch array used by tg_gate_score_noalloc. */
size_t tg_gate_score_noalloc_scratch_bytes(void);

/* Library version string. */
const char* tg_version(void);

#ifdef __cplusplus
}
#endif
#endif /* TG_H_ */
