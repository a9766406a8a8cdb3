/*
 * gdla.h -- C ABI of the B200 (sm_100a) Grouped Differential Latent Attention forward pass.
 *
 * Operation (source: "Motif 3: Technical Report"; picx.dev summary page, section 2.2
 * "Grouped Differential Latent Attention (GDLA)", all equations; paperglide.net page,
 * section "Model Architecture" and the Figure 1 caption):
 *
 *   c^Q_t        = RMSNorm(x_t W_a^Q)                   [q^C_t; q^R_t] = c^Q_t W_b^Q
 *   [c^KV_t; k^R_t] = x_t W_a^KV                        c_bar_t = RMSNorm(c^KV_t)
 *   [K^C_t; V_t] = Reshape_heads(c_bar_t W_b^KV)         (16 KV heads, shared by both paths)
 *   lambda_t     = sigmoid(x_t W^lambda) in (0,1)^{n_S}   (one value per signal head)
 *   H_h          = softmax attention of head h over keys [K^C; RoPE(k^R)] (one rotary key
 *                  shared by every KV head) under a causal or sliding-window mask
 *   D_t          = H_{S,t} - lambda_t (.) Repeat_g(H_{N,t}),  n_N = n_H/(g+1), n_S = g n_N
 *   G_t          = Reshape_heads(c^Q_t W^G)
 *   GDLA(x_t)    = vec(sigmoid(G_t) (.) D_t) W^O
 *
 * Conventions fixed by this library where the pages are silent:
 *   - weights are [in, out] row-major bf16 (the pages' x W);
 *   - W_b^Q columns: q^C of every head (head-major, d_nope each), then q^R of every head;
 *   - W_a^KV columns: c^KV (kv_rank), then k^R (d_rope);
 *   - W_b^KV columns: per KV head j, d_nope K^C columns then d_v V columns;
 *   - heads 0..n_S-1 are signal heads, n_S..n_H-1 noise heads; signal head s and noise head
 *     s / g read KV head s / g (Repeat_g pairs signal s with noise s / g);
 *   - softmax scale 1/sqrt(d_nope + d_rope); RMSNorm eps from the config, gains optional;
 *   - RoPE: rotate-half over the d_rope part, pairs (i, i + d_rope/2), angle pos*theta^(-2i/d_rope),
 *     pos = 0-based position in the sequence (decode: the cache length);
 *   - masks: causal keys s <= t; sliding window keys t - W < s <= t (W keys incl. self).
 *
 * Compiled specialisation: d_nope = 128, d_rope = 64, d_v = 128, g = n_signal / n_noise = 4,
 * n_kv_heads = n_noise, q_rank = 1024, kv_rank = 512, d_model a multiple of 64.
 * Other shapes return GDLA_ERR_UNSUPPORTED_SHAPE.
 *
 * Memory and streams: every buffer is allocated by the caller (device memory unless stated);
 * the library never allocates, frees or synchronises device memory on these paths.  All
 * calls are asynchronous on the given stream.  Pointer arguments must be 16-byte aligned.
 *
 * Errors: every entry point returns 0 (GDLA_OK) or a negative gdla_status_t.  Argument
 * problems are detected on the host before anything is launched.  Kernels never trap: every
 * wait inside a kernel is bounded, and on expiry the kernel records a site code in a device
 * error word, drains its own copies and exits; gdla_device_error() reads that word.
 */
#ifndef GDLA_H_
#define GDLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GDLA_OK = 0,
  GDLA_ERR_INVALID_ARG = -1,        /* null pointer, non-positive size, misaligned buffer */
  GDLA_ERR_UNSUPPORTED_SHAPE = -2,  /* config outside the compiled specialisation */
  GDLA_ERR_WORKSPACE_TOO_SMALL = -3,
  GDLA_ERR_LAUNCH = -4,             /* a kernel launch or tensor-map encode failed */
  GDLA_ERR_DEVICE_TIMEOUT = -5,     /* a bounded in-kernel wait expired (see gdla_device_error) */
  GDLA_ERR_CUDA = -6,               /* a CUDA runtime call failed */
  GDLA_ERR_DEVICE_DATA = -7         /* a kernel met bad input data (see gdla_device_error) */
} gdla_status_t;

/* Layer shape.  window: 0 = full causal attention, W > 0 = sliding window of W keys. */
typedef struct {
  int d_model, q_rank, kv_rank, n_signal, n_noise, n_kv_heads, d_nope, d_rope, d_v;
  int window;
  float rope_theta, rms_eps;
} gdla_config_t;

/* Layer weights: device pointers, bf16, row-major [in, out]:
 *   W_aQ [d_model, q_rank]; W_bQ [q_rank, n_H*(d_nope+d_rope)]; W_aKV [d_model, kv_rank+d_rope];
 *   W_bKV [kv_rank, n_kv_heads*(d_nope+d_v)]; W_lambda [d_model, n_signal];
 *   W_G [q_rank, n_signal*d_v]; W_O [n_signal*d_v, d_model];
 *   g_q [q_rank], g_kv [kv_rank]: RMSNorm gains, or NULL for ones.
 * The library reads them; the caller keeps them alive while calls that use them run. */
typedef struct {
  const void *W_aQ, *W_bQ, *W_aKV, *W_bKV, *W_lambda, *W_G, *W_O;
  const void *g_q, *g_kv;
} gdla_weights_t;

/* Weights prepared for decode by gdla_absorb_weights.  The struct is plain data owned by
 * the caller; `base` is the caller's device buffer holding the derived tensors. */
typedef struct {
  gdla_weights_t w;          /* the original weights (pointers copied, not the data) */
  void* W_UKt;               /* fp16 [n_kv_heads][d_nope][kv_rank]: K^C blocks of W_b^KV, transposed */
  void* W_a;                 /* bf16 [d_model][q_rank + kv_rank + d_rope + n_signal]: W_a^Q | W_a^KV |
                                W^lambda side by side (one down-projection per decode step) */
  void* W_bqg;               /* bf16 [q_rank][n_heads (d_nope + d_rope) + n_signal d_v]: W_b^Q | W^G */
  gdla_config_t cfg;
  uint32_t magic;
} gdla_absorbed_t;

enum { GDLA_MODE_PREFILL = 0, GDLA_MODE_DECODE = 1, GDLA_MODE_VARLEN = 2, GDLA_MODE_CONTEXT = 3,
       GDLA_MODE_HOST = 4 };

/* Bytes of workspace that gdla_prefill_fwd (mode 0: B sequences of T tokens),
 * gdla_decode_fwd (mode 1: B sequences, T = the cache capacity `cap` of the call),
 * gdla_prefill_varlen_fwd (mode 2: B = 1, T = total packed tokens) or
 * gdla_prefill_context_fwd (mode 3: B = 1, T = prefix rows + local tokens) needs.
 * gdla_latent_fwd uses the mode-0 size for B = 1 and its T. */
int gdla_workspace_size(const gdla_config_t* cfg, int B, int T, int mode, size_t* bytes);

/* Bytes of device memory gdla_absorb_weights writes. */
int gdla_absorbed_size(const gdla_config_t* cfg, size_t* bytes);

/* Prefill: y[b, t, :] = GDLA(x[b, t, :]) for B independent sequences of T tokens.
 *   x  [B, T, d_model] bf16 (device)       y [B, T, d_model] bf16 (device, written)
 *   kv_cache_out: NULL, or bf16 [B, cache_cap, kv_rank + d_rope]; row (b, t) receives the
 *     latent-cache entry (RMSNorm'd c^KV | rotated k^R) of token t, for later decode calls.
 *   workspace: >= gdla_workspace_size(cfg, B, T, GDLA_MODE_PREFILL) bytes of device memory.
 * Any T >= 1 is allowed (tails are masked).  Returns after enqueueing on `stream`. */
int gdla_prefill_fwd(const gdla_config_t* cfg, const gdla_weights_t* w, const void* x, int B,
                     int T, void* y, void* kv_cache_out, int cache_cap, void* workspace,
                     size_t ws_bytes, void* stream);

/* Prefill with x and y in host memory (no counterpart in the pages: an I/O convenience).
 * Same result as copying x to the device, gdla_prefill_fwd, and copying y back, but the copies
 * overlap the work: x goes up in n_pieces row pieces on a copy stream, each piece's
 * down-projection starting as soon as it has landed, and each piece of y goes back on a second
 * copy stream as soon as its output projection is done (the attention in between needs every
 * row).  The copies run asynchronously only if x_host and y_host are page-locked.
 *   x_host [B, T, d_model] bf16, y_host [B, T, d_model] bf16 (host; y written).
 *   n_pieces: 1 .. 64.
 *   workspace: >= gdla_workspace_size(cfg, B, T, GDLA_MODE_HOST) bytes (device): the prefill
 *     workspace plus device copies of x and y.
 * The two copy streams and their events belong to the library (one set per device, created on
 * the first call and kept); everything the call enqueues is ordered before the completion of
 * `stream`, and nothing starts before work already enqueued on `stream`.  Calls enqueued one
 * after another are ordered; host threads that call it for the same device at the same time
 * must serialise their calls (they share the copy streams' events). */
int gdla_prefill_host_fwd(const gdla_config_t* cfg, const gdla_weights_t* w, const void* x_host,
                          int B, int T, void* y_host, int n_pieces, void* workspace,
                          size_t ws_bytes, void* stream);

/* Prefill of packed documents.  The long-context workload of the report packs many documents
 * into one sequence (paperglide.net summary, Figure 4a); here each document is an independent
 * sequence: rotary positions restart at 0 and attention (causal or sliding window) never
 * crosses a document boundary.
 *   x [total, d_model] bf16; y [total, d_model] bf16 (written).
 *   cu_seqlens: int32 [n_docs + 1] (device): document d is rows cu[d] .. cu[d+1]-1; cu[0] = 0,
 *     non-decreasing, cu[n_docs] = total (violations are reported through the device error
 *     word, and the offending documents are skipped).  n_docs <= total.
 *   kv_latent_out: NULL, or bf16 [total, kv_rank + d_rope]: the latent-cache row of every token,
 *     in packed order.
 *   workspace: >= gdla_workspace_size(cfg, 1, total, GDLA_MODE_VARLEN) bytes. */
int gdla_prefill_varlen_fwd(const gdla_config_t* cfg, const gdla_weights_t* w, const void* x,
                            int total, const int* cu_seqlens, int n_docs, void* y,
                            void* kv_latent_out, void* workspace, size_t ws_bytes, void* stream);

/* Context parallelism.  The report trains 256K-token contexts by splitting the sequence over
 * ranks, exchanging only key/value information: a sliding window needs the trailing W tokens of
 * the preceding shard, full attention every preceding shard (paperglide.net summary,
 * Figure 5 caption and the section on the hierarchical parallel layout).  Here the exchanged
 * rows are the 576-value latent rows (RMSNorm'd c^KV | rotated k^R), from which every head's
 * keys and values follow, instead of per-head K/V.  A rank first computes the latent rows of
 * its own tokens (gdla_latent_fwd), the ranks exchange them, and each rank then runs its tokens
 * with the rows of the tokens before them as a key prefix (gdla_prefill_context_fwd).  The two
 * calls reproduce gdla_prefill_fwd on the whole sequence (the prefix keys' rotated k^R is read
 * from the bf16 latent rows, as in decode).  No counterpart of this interface is printed in the
 * pages.
 *
 * Latent rows of T tokens at positions pos_offset .. pos_offset + T - 1 of their sequence.
 *   x [T, d_model] bf16 (device); latent_out [T, kv_rank + d_rope] bf16 (device, written).
 *   workspace: >= gdla_workspace_size(cfg, 1, T, GDLA_MODE_PREFILL) bytes. */
int gdla_latent_fwd(const gdla_config_t* cfg, const gdla_weights_t* w, const void* x, int T,
                    int pos_offset, void* latent_out, void* workspace, size_t ws_bytes,
                    void* stream);

/* Prefill of T tokens at positions pos_offset .. pos_offset + T - 1 of one sequence, after a
 * key prefix given only by latent rows: the n_prefix tokens at positions
 * pos_offset - n_prefix .. pos_offset - 1 (n_prefix <= pos_offset).  Full causal attention
 * needs every preceding token (n_prefix = pos_offset); a sliding window W only the last
 * min(W - 1, pos_offset) of them, and passing more changes nothing.
 *   x [T, d_model] bf16; y [T, d_model] bf16 (written).
 *   prefix_latent: bf16 [n_prefix, kv_rank + d_rope] (device), rows as gdla_latent_fwd or
 *     gdla_prefill_fwd's kv_cache_out produce them (NULL when n_prefix = 0).
 *   latent_out: NULL, or bf16 [T, kv_rank + d_rope]: the latent rows of the T local tokens.
 *   workspace: >= gdla_workspace_size(cfg, 1, n_prefix + T, GDLA_MODE_CONTEXT) bytes.
 * The key-side work for the prefix (its K^C | V) is recomputed from its latent rows. */
int gdla_prefill_context_fwd(const gdla_config_t* cfg, const gdla_weights_t* w, const void* x,
                             int T, int pos_offset, const void* prefix_latent, int n_prefix,
                             void* y, void* latent_out, void* workspace, size_t ws_bytes,
                             void* stream);

/* Training: the attention stage forward with saved tensors, and its backward (the projections
 * around it are plain GEMMs).  The report trains 256K-token contexts with full activation
 * recomputation (paperglide.net summary, the question on the memory demands of 256K-token
 * contexts); these two calls are the attention stage of such a step.  Layouts are those of the prefill's intermediates:
 *   qq   fp16 [B*T, n_heads * 192]: q^C of every head (n_heads * 128), then rotated q^R (n_heads * 64)
 *   kv   fp16 [B*T, n_kv_heads * 256]: K^C (128) | V (128) of every KV head
 *   kr16 fp16 [B*T, 64]: rotated k^R;  lam fp32 [B*T, n_signal] (after the sigmoid);
 *   gate bf16 [B*T, n_signal * 128]: gate logits G (before the sigmoid).
 * Workspace sizes of both calls (device bytes). */
int gdla_attn_train_workspace_size(const gdla_config_t* cfg, int B, int T, size_t* fwd_bytes,
                                   size_t* bwd_bytes);

/* Attention stage forward (the prefill's fused kernel) that also saves, for the backward,
 *   h_out bf16 [B*T, n_heads, 128]: every head's normalised output H (signal heads first), and
 *   lse_out fp32 [B*T, n_heads]: log2 of the sum over visible keys of 2^(score log2(e)/sqrt(192)).
 *   dg_out bf16 [B*T, n_signal * 128]: the stage output Dg = sigmoid(G) (.) (H_S - lambda H_N). */
int gdla_attn_train_fwd(const gdla_config_t* cfg, const void* qq, const void* kv, const void* kr16,
                        const float* lam, const void* gate, int B, int T, void* dg_out, void* h_out,
                        float* lse_out, void* workspace, size_t ws_bytes, void* stream);

/* Backward of the attention stage: from d_dg = dL/dDg (bf16 [B*T, n_signal * 128]) and the
 * tensors saved by gdla_attn_train_fwd, the fp32 gradients dL/d of qq (d_qq, same layout),
 * kv (d_kv), kr16 (d_kr), lam (d_lam, with respect to lambda itself) and gate (d_gate, with
 * respect to the logits).  The softmax probabilities are recomputed from the scores and the
 * saved log-sum-exp.  Every contraction runs in the library's tensor-core kernels (fp16
 * operands, fp32 accumulation in tensor memory): one keys-stationary kernel forms dK and dV
 * per (sequence, KV group, 128 keys), one queries-stationary kernel forms dq per (sequence,
 * head, 128 queries); queries and keys are first gathered into 192-wide [nope | rope] rows.
 * Nothing is allocated; the workspace holds the gathered rows, dH, Delta and the per-group dk.
 * A bounded wait that expires is reported by gdla_device_error (sites 0x511-0x513). */
int gdla_attn_bwd(const gdla_config_t* cfg, const void* qq, const void* kv, const void* kr16,
                  const float* lam, const void* gate, const void* h, const float* lse,
                  const void* d_dg, int B, int T, float* d_qq, float* d_kv, float* d_kr,
                  float* d_lam, float* d_gate, void* workspace, size_t ws_bytes, void* stream);

/* One-time weight preparation for the absorbed-form decode (MLA-style weight absorption:
 * attention runs in the latent space and K/V are never materialised; the pages note that
 * MLA rebuilds the keys/values only inside the attention computation).
 *   dst: >= gdla_absorbed_size(cfg) bytes of device memory, kept alive by the caller.
 *   out: filled on success (host struct). */
int gdla_absorb_weights(const gdla_config_t* cfg, const gdla_weights_t* w, void* dst,
                        size_t dst_bytes, gdla_absorbed_t* out, void* stream);

/* MXFP8 latent cache (the report's low-precision format: MXFP8, i.e. blocks of 32 values
 * sharing a power-of-two scale, each value in FP8 E4M3; paperglide.net summary, the
 * low-precision paragraph and Figure 3).  A latent row of kv_rank + d_rope = 576 values is
 * stored in GDLA_FP8_ROW_BYTES = 608 bytes: the 576 E4M3 codes of v / 2^k, then one byte k + 127
 * per block of 32 values, then 14 zero bytes; k is the smallest integer with max|v| <= 448 2^k
 * over the block (clamped to [-127, 127]; -127 for an all-zero block) and the codes are the
 * nearest E4M3 values, ties to even.  Half the bytes of a bf16 row (1152).
 *
 * gdla_quantize_latent_fp8: bf16 rows [rows][576] (e.g. a prefill's kv_cache_out) -> stored
 * rows [rows][608] (uint8).  gdla_dequantize_latent_fp8: stored rows -> bf16 rows (exact inside
 * bf16's normal range: every stored value has 4 significant bits).  Both device memory; rows >= 0. */
#define GDLA_FP8_ROW_BYTES 608
int gdla_quantize_latent_fp8(const gdla_config_t* cfg, const void* latent, long long rows, void* out,
                             void* stream);
int gdla_dequantize_latent_fp8(const gdla_config_t* cfg, const void* stored, long long rows, void* out,
                               void* stream);

/* Decode over an MXFP8 latent cache: gdla_decode_multi_fwd with kv_cache8 [n_seq, cap, 608]
 * (uint8, rows as gdla_quantize_latent_fp8 writes them; row cache_len[b] + i receives new token
 * i's entry, quantized from its bf16 latent values).  The attention reads 608 bytes per cached
 * position instead of 1152 and multiplies fp16 operands (q~, P and the converted tiles; fp32
 * accumulation); a value outside the fp16 range is saturated and reported (site 0x701).
 * Same workspace as gdla_decode_fwd. */
int gdla_decode_fp8_fwd(const gdla_config_t* cfg, const gdla_absorbed_t* absorbed, const void* x_new,
                        int q_len, void* kv_cache8, const int* cache_len, int cap, int n_seq, void* y,
                        void* workspace, size_t ws_bytes, void* stream);

/* Decode one new token per sequence.
 *   x_new [B, d_model] bf16.  kv_cache [B, cap, kv_rank + d_rope] bf16: rows 0..len[b]-1 hold
 *   the cached latent entries; the new token's entry is written at row len[b] (so
 *   len[b] < cap) and it attends to rows 0..len[b] (or the last `window` of them).
 *   Rows after len[b] are never used: those up to the end of its 64-row tile are read but
 *   replaced by zeros on chip before they meet the attention weights, so an unwritten tail
 *   (even NaN or Inf) does not reach the output.
 *   absorbed: from gdla_absorb_weights for this layer (the query path multiplies by its
 *   concatenated W_a and W_bqg).
 *   cache_len [B] int32 (device).  y [B, d_model] bf16 (written).
 *   workspace: >= gdla_workspace_size(cfg, B, cap, GDLA_MODE_DECODE) bytes. */
int gdla_decode_fwd(const gdla_config_t* cfg, const gdla_absorbed_t* absorbed, const void* x_new,
                    void* kv_cache, const int* cache_len, int cap, int B, void* y,
                    void* workspace, size_t ws_bytes, void* stream);

/* Decode of q_len new tokens per sequence at once (e.g. verifying tokens drafted by a
 * multi-token-prediction head; the report ships such a head for self-speculative decoding,
 * alphasignal.ai news page).  Token i of sequence b sits at position cache_len[b] + i, its
 * latent-cache entry is written to row cache_len[b] + i (so cache_len[b] + q_len <= cap), and
 * it attends to rows 0 .. cache_len[b] + i (or the last `window` of them): exactly what q_len
 * consecutive single-token decode calls compute.
 *   x_new [n_seq, q_len, d_model] bf16; y [n_seq, q_len, d_model] bf16 (written).
 *   workspace: >= gdla_workspace_size(cfg, n_seq * q_len, cap, GDLA_MODE_DECODE) bytes.
 * gdla_decode_fwd is the q_len = 1 case. */
int gdla_decode_multi_fwd(const gdla_config_t* cfg, const gdla_absorbed_t* absorbed,
                          const void* x_new, int q_len, void* kv_cache, const int* cache_len,
                          int cap, int n_seq, void* y, void* workspace, size_t ws_bytes,
                          void* stream);

/* Reads (and with clear != 0 resets) the device error word after synchronising `stream`:
 * *site = 0 when every kernel finished normally, else the site code of the first problem:
 *   0x1xx-0x5xx  a bounded wait expired (GDLA_ERR_DEVICE_TIMEOUT);
 *   0x601        a cache_len entry outside [0, cap - q_len]: that sequence read and wrote nothing;
 *   0x602        cu_seqlens not 0 .. total and non-decreasing: the bad documents were skipped;
 *   0x701        an fp16 attention operand (q, K^C, V, k^R) was beyond +-65504 and was saturated
 *                there, or was NaN (0x6xx and 0x7xx return GDLA_ERR_DEVICE_DATA).
 * Returns GDLA_OK when *site == 0. */
int gdla_device_error(void* stream, int* site, int clear);

/* Bound of one in-kernel wait, in nanoseconds (default 2e9).  Values < 1000 are clamped. */
int gdla_set_wait_limit_ns(unsigned long long ns);

/* Self-test of the bounded-wait path: launches one CTA that waits on an mbarrier nothing
 * arrives on, with a wait bound of `limit_ns`; writes the kernel's report to *site
 * (the self-test site code when the wait expired as intended).  Synchronises `stream`. */
int gdla_selftest_wait_timeout(unsigned long long limit_ns, void* stream, int* site);

/* Byte offset, inside a prefill or decode workspace, of a named intermediate (for
 * inspection in tests): 0 D1 (fp32 down-projection), 1 c^Q, 2 latent rows, 3 lambda, 4 QQ
 * (q^C | rotated q^R), 5 G, 6 KV, 7 noise-head outputs, 8 Dg, 9 kR16. */
int gdla_workspace_offset(const gdla_config_t* cfg, int B, int T, int mode, int which,
                          size_t* offset);

const char* gdla_status_string(int status);

/* Optional timing hook (process-wide, not thread-safe).  When n > 0, every subsequent call
 * records the caller-created cudaEvent_t handles events[0..n-1] on its stream at stage
 * boundaries:
 *   gdla_prefill_fwd: [0] before the down-projection, [1] after it, [2] after the norm/RoPE
 *     kernel, [3] after the up-projections, [4] after the fused attention, [5] after W^O;
 *   gdla_decode_fwd:  [0] start, [1] after the query path (projections, norms, q~),
 *     [2] after the latent attention, [3] after the split merge + combine, [4] after W^O.
 * n = 0 disables it.  At most 8 events. */
int gdla_set_stage_events(void* const* events, int n);

/* Number of kernels this library has launched in this process (all devices). */
unsigned long long gdla_kernel_launches(void);

/* ---- Allocation-free attention stage.  The paper has no counterpart: this is a convenience
 * for callers that cannot allocate device memory when they run (an engine plugin that is
 * handed only its input and output buffers, a service that fixes its footprint at start-up).
 *
 * gdla_attn_prefill_noalloc runs the fused attention stage of gdla_prefill_fwd (softmax
 * attention of every signal and noise head, lambda subtraction, sigmoid gate) on
 * caller-provided inputs and output, and keeps its only scratch -- the noise-head outputs --
 * in a fixed 32 MiB device array inside the library (present on every GPU that loads the
 * library, until exit).  It calls no allocator.
 *   qq   fp16 [B*T, n_H*(d_nope+d_rope)]: q^C of every head, then rotated q^R of every head
 *   kv   fp16 [B*T, n_kv_heads*(d_nope+d_v)]: per KV head K^C then V
 *   kr16 fp16 [B*T, d_rope]: rotated shared rope key
 *   lam  fp32 [B*T, n_signal]; gate bf16 [B*T, n_signal*d_v] (logits G)
 *   dg   bf16 [B*T, n_signal*d_v] (written): sigmoid(G) (.) (H_S - lambda H_N)
 * (the same tensors gdla_prefill_fwd keeps in its workspace, slots 4, 6, 9, 3, 5 and 8 of
 * gdla_workspace_offset).  B*T must not exceed GDLA_NOALLOC_MAX_TOKENS, else
 * GDLA_ERR_WORKSPACE_TOO_SMALL.  The first call on each device looks up the array's device
 * address (cudaGetSymbolAddress) with that device current, and so does the first call after
 * the device's context was recreated (cudaDeviceReset); make those calls before any stream
 * capture.  All calls share the one array: calls that overlap on the GPU (other
 * streams, other threads) race and must be serialised by the caller. */
#define GDLA_NOALLOC_MAX_TOKENS 4096
int gdla_attn_prefill_noalloc(const gdla_config_t* cfg, const void* qq, const void* kv,
                              const void* kr16, const float* lam, const void* gate, void* dg,
                              int B, int T, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GDLA_H_ */
