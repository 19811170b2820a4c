/*
 * orthrus.h - C ABI of the B200 (sm_100a) Orthrus dual-view decode step.
 *
 * Orthrus ("Memory-Efficient Parallel Token Generation via Dual-View
 * Diffusion"; opentrain.ai abstract, atlas.scime.ai summary "Approach")
 * augments a frozen autoregressive (AR) decoder with a trainable attention
 * path per layer. One decode step:
 *   1. draft view: one forward over the block [y, MASK x (K-1)] with the draft
 *      attention module; every block position attends to the frozen model's
 *      KV cache and to all block positions (bidirectional); the argmax of block
 *      row i is the draft d_{i+1}                      -> orthrus_draft_block
 *   2. verify view: one causal forward of the frozen model over [y, d_1..d_K];
 *      the argmax of block row j is g_j; the block's base K/V is written into
 *      cache slots n..n+K                               -> orthrus_verify_block
 *   3. greedy consensus: a = number of leading d_i == g_{i-1}; commit
 *      d_1..d_a and g_a; slots n..n+a become live; n += a+1; y = g_a
 *                                                       -> orthrus_accept_commit
 * (Hacker News summary "Idea": the diffusion head projects K tokens in
 * parallel and the AR head verifies in a second pass, accepting the longest
 * matching prefix; news article "KV Cache Overhead": one shared cache, only
 * the AR view updates it.) orthrus_decode_step runs all three.
 *
 * Conventions used by every call:
 *   - All device memory is owned and allocated by the caller. The library
 *     allocates nothing: the per-model "plan" is a caller-provided HOST buffer
 *     of orthrus_plan_bytes() bytes, and all scratch lives in a caller-provided
 *     DEVICE workspace of orthrus_workspace_bytes() bytes.
 *   - Every call is asynchronous on the given CUDA stream and performs no host
 *     synchronisation; results are valid once the stream reaches them.
 *   - Host-detectable misuse (NULL pointers, sizes out of range) returns an
 *     error before anything is launched. Conditions found on the device
 *     (cache overrun, NaN logits, a bounded wait that ran out) are recorded in
 *     a sticky device int32 status word (first error wins), readable through
 *     orthrus_status_ptr(); kernels then stop writing the cache.
 *   - Matrices are row-major. bf16 = IEEE bfloat16 bits (uint16); fp16 = IEEE
 *     binary16 bits (uint16).
 *   - Model layout: W_qkv rows = q heads | k heads | v heads (each head_dim rows);
 *     W_gate_up rows = gate (d_ff) | up (d_ff); W_o [d_model][n_heads*head_dim];
 *     W_down [d_model][d_ff]; embed and lm_head [vocab][d_model] (untied).
 *   - KV cache: K and V [n_layers][batch][n_kv_heads][capacity][head_dim],
 *     post-QK-norm and post-RoPE, rounded to bf16 values (the cache precision)
 *     and held in the fp16 encoding, which represents every bf16 value of
 *     magnitude in [2^-17, 65504] exactly (smaller ones to within 2^-25): one
 *     tensor-core MMA takes operands of one type, and the attention's q and
 *     softmax weights are fp16. cache.len[b] (device int32) = live slots.
 *   - Shapes supported by the kernels: head_dim in {64, 128}; d_model, d_ff and
 *     n_heads*head_dim multiples of 128; vocab a multiple of 128;
 *     n_heads / n_kv_heads in {1, 2, 4, 8}; 1 <= K <= 64.
 */
#ifndef ORTHRUS_H
#define ORTHRUS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* orthrus_stream; /* same type as cudaStream_t */

typedef enum {
  ORTHRUS_OK = 0,
  ORTHRUS_ERR_ARG = 1,         /* NULL pointer, size or shape out of range                */
  ORTHRUS_ERR_CAPACITY = 2,    /* len + block > cache capacity (host or device detected)  */
  ORTHRUS_ERR_CUDA = 3,        /* a CUDA runtime call failed                               */
  ORTHRUS_ERR_TIMEOUT = 4,     /* a device-side bounded wait ran out (device status only) */
  ORTHRUS_ERR_NAN = 5,         /* a NaN logit reached an argmax (device status only)      */
  ORTHRUS_ERR_UNSUPPORTED = 6, /* shape outside what the kernels implement                */
  ORTHRUS_ERR_WORKSPACE = 7    /* plan or workspace buffer too small                       */
} orthrus_status;

/* Decoder shape (Qwen3-style: pre-RMSNorm, optional per-head q/k RMSNorm,
 * rotate-half RoPE at absolute positions, SwiGLU MLP). mask_id is the token
 * placed at draft-block positions 2..K. */
typedef struct {
  int32_t n_layers, d_model, n_heads, n_kv_heads, head_dim, d_ff, vocab, mask_id, qk_norm;
  float rope_theta, rms_eps;
} orthrus_config;

/* Device pointers to the weights. Per-layer members are HOST arrays of
 * n_layers DEVICE pointers. Norm gains are fp32; matrices are bf16. Every
 * pointer is 16-byte aligned (tensor-map bases; norm gains are read as
 * 16-byte vectors); orthrus_plan_init returns ORTHRUS_ERR_ARG otherwise.
 * wd_* are the draft attention module's own projections and q/k norm gains;
 * the draft view reuses attn_norm, mlp_norm, the MLP, final_norm and lm_head. */
typedef struct {
  const void* embed;      /* bf16 [vocab][d_model]     */
  const float* final_norm; /* fp32 [d_model]            */
  const void* lm_head;    /* bf16 [vocab][d_model]     */
  const float* const* attn_norm; /* [L] fp32 [d_model]  */
  const float* const* mlp_norm;  /* [L] fp32 [d_model]  */
  const void* const* w_qkv;      /* [L] bf16 [(H+2Hkv)d][d_model] */
  const void* const* w_o;        /* [L] bf16 [d_model][H d]       */
  const float* const* q_norm;    /* [L] fp32 [d] (unused if !qk_norm) */
  const float* const* k_norm;    /* [L] fp32 [d]                  */
  const void* const* w_gate_up;  /* [L] bf16 [2 d_ff][d_model]    */
  const void* const* w_down;     /* [L] bf16 [d_model][d_ff]      */
  const void* const* wd_qkv;     /* [L] bf16, shape of w_qkv      */
  const void* const* wd_o;       /* [L] bf16, shape of w_o        */
  const float* const* wd_q_norm; /* [L] fp32 [d]                  */
  const float* const* wd_k_norm; /* [L] fp32 [d]                  */
} orthrus_weights;

/* The one shared KV cache (base view only). */
typedef struct {
  void* k;        /* fp16 encoding of bf16 values [L][batch][Hkv][capacity][d] */
  void* v;        /* fp16 encoding of bf16 values [L][batch][Hkv][capacity][d] */
  int32_t* len;   /* device int32 [batch]: live slots per sequence */
  int32_t batch;
  int32_t capacity;
} orthrus_cache;

/* ---- set-up ------------------------------------------------------------ */

/* Host bytes the plan needs (TMA descriptors for every weight, the cache and
 * the workspace, plus launch geometry). */
size_t orthrus_plan_bytes(const orthrus_config* cfg);

/* Device bytes of the workspace for a plan with this batch, cache capacity,
 * block size limit max_block (1 <= K <= max_block <= 64) and row limit
 * max_rows (rows of one forward: at least batch*(max_block+1); prefill runs
 * in causal chunks of at most max_rows tokens). 0 for an invalid request.
 * Includes the draft view's block scratch, 2 * L * batch * max_block * Hkv *
 * d * 2 bytes: 4.5 MiB at the Qwen3-8B shape with K = 32 and batch 1, the
 * pages' "about 4.5 MiB, flat" KV overhead (Hacker News summary "Results"). */
size_t orthrus_workspace_bytes(const orthrus_config* cfg, int32_t batch, int32_t capacity, int32_t max_block,
                               int32_t max_rows);

/* Byte offset of the draft block scratch (K part, then V part) inside the
 * workspace, and its total size (K and V). */
size_t orthrus_block_scratch_offset(const orthrus_config* cfg, int32_t batch, int32_t capacity, int32_t max_block,
                                    int32_t max_rows);
size_t orthrus_block_scratch_bytes(const orthrus_config* cfg, int32_t batch, int32_t max_block);

/* Fill the caller's host buffer `plan` for these weights, cache and workspace
 * and zero the workspace on `stream`. Pointers are captured: weights, cache
 * and workspace must stay allocated, at the same addresses, while the plan is
 * used. Errors: ORTHRUS_ERR_ARG, ORTHRUS_ERR_UNSUPPORTED, ORTHRUS_ERR_WORKSPACE,
 * ORTHRUS_ERR_CUDA. */
orthrus_status orthrus_plan_init(void* plan, size_t plan_bytes, const orthrus_config* cfg,
                                 const orthrus_weights* w, const orthrus_cache* cache, int32_t max_block,
                                 int32_t max_rows, void* workspace, size_t workspace_bytes, orthrus_stream stream);

/* Device pointer to the sticky int32 status word (inside the workspace), and
 * a call that resets it to ORTHRUS_OK on `stream`. */
int32_t* orthrus_status_ptr(const void* plan);
orthrus_status orthrus_clear_status(const void* plan, orthrus_stream stream);

/* Number of kernels one call of orthrus_decode_step launches for block size K
 * (planted drafts add one device-to-device copy, not a kernel). */
int32_t orthrus_decode_step_launches(const void* plan, int32_t K);

/* Kernel kinds reported by orthrus_trace. */
enum {
  ORTHRUS_KIND_EMBED = 0,      /* block embedding + RoPE table + capacity check   */
  ORTHRUS_KIND_RMSNORM = 1,    /* RMSNorm to bf16                                  */
  ORTHRUS_KIND_GEMM_QKV = 2,   /* q/k/v projection + QK-norm + RoPE + K/V store   */
  ORTHRUS_KIND_ATTENTION = 3,  /* block attention                                  */
  ORTHRUS_KIND_GEMM_O = 4,     /* output projection + residual                     */
  ORTHRUS_KIND_GEMM_GATE_UP = 5, /* gate/up projection + SwiGLU                    */
  ORTHRUS_KIND_GEMM_DOWN = 6,  /* down projection + residual                       */
  ORTHRUS_KIND_LM_HEAD = 7,    /* LM head + running argmax                         */
  ORTHRUS_KIND_ARGMAX = 8,     /* argmax finalisation                              */
  ORTHRUS_KIND_ACCEPT = 9,     /* greedy consensus + KV commit                     */
  ORTHRUS_KIND_OTHER = 10,     /* poisoning, length updates, planted-draft copy    */
  ORTHRUS_KIND_END = 11,       /* marker after the last launch of a call          */
  ORTHRUS_KIND_FORWARD = 12,   /* persistent kernel: one whole draft or verify forward
                                  (and, in orthrus_decode_step, the consensus)     */
  ORTHRUS_KIND_SAMPLE = 13     /* temperature sampling: categorical draws, row statistics */
};

/* Profiling hook. While set, every launch made by the calls below is preceded
 * by cudaEventRecord(events[i], stream) with kinds[i] = its ORTHRUS_KIND_*, and
 * each call ends with an ORTHRUS_KIND_END marker; *count holds the number of
 * events used (recording stops at `capacity`). events are cudaEvent_t handles
 * created by the caller with timing enabled; launch i lasted
 * elapsed(events[i], events[i+1]). Pass events == NULL to switch it off.
 * Host memory of `kinds` and `count` must stay valid while the hook is set. */
orthrus_status orthrus_trace(void* plan, void* const* events, int32_t* kinds, int32_t capacity, int32_t* count);

/* Profiling hook of the persistent forward kernel (the draft and verify views of
 * blocks whose token rows fit it: at most 96 at head dim 128). While set, every
 * launch of it writes, for each CTA c and phase p (p = 0 embedding, 1 + 6 l +
 * {0..5} = layer l's q/k/v projection, attention, chunk merge, output projection,
 * gate/up, down, 1 + 6 L = LM head), sixteen globaltimer stamps (ns, uint64) at
 * device_buf[(c * (2 + 6 L) + p) * 16 + e]: e = 0/1 first/last weight load
 * issued, 2/3 activation dependency met/last activation load issued, 4/5 first
 * MMA/last MMA commit, 6/7 epilogue dependency met/phase finished; for the last
 * epilogue segment of a projection phase 8..13 = accumulator ready, partial stored,
 * arrival counted, partials loaded, epilogue done, completion signalled; in an
 * attention phase 14/15 = first score tile ready, O read (9/10 row maxima done and
 * P written for the first tile, 8 later score tiles ready). Entries of events that
 * did not occur keep their previous contents. device_buf: device memory of at least
 * orthrus_timeline_bytes(plan) bytes, owned by the caller; NULL switches the hook
 * off. */
size_t orthrus_timeline_bytes(const void* plan);
orthrus_status orthrus_timeline(void* plan, void* device_buf, size_t bytes);

/* ---- the decode step ---------------------------------------------------- */

/* AR prefill (atlas summary "Approach": the frozen backbone does prefill and
 * builds the KV cache). tokens: device int32 [batch][max_prompt];
 * prompt_len: HOST int32 [batch], 1 <= prompt_len[b] <= max_prompt. Writes the
 * prompt's K/V to slots [0, prompt_len[b]), sets cache.len[b] = prompt_len[b]
 * and pending[b] (device int32 [batch]) = argmax at the last prompt row: the
 * first generated token. Runs causal chunks of at most max_rows tokens.
 * Errors: ORTHRUS_ERR_ARG; ORTHRUS_ERR_CAPACITY if a prompt exceeds capacity. */
orthrus_status orthrus_prefill(const void* plan, const int32_t* tokens, const int32_t* prompt_len, int32_t max_prompt,
                               int32_t* pending, orthrus_stream stream);

/* Draft view (atlas summary "Approach": predict a block of K tokens in one
 * forward over the same KV cache). pending: device int32 [batch]. Writes
 * draft (device int32 [batch][K]) with d_1..d_K. logits (nullable): device
 * fp32 [batch][K][vocab] of the draft rows, for checking. The cache is read,
 * never written; the block's draft-view K/V stays in the block scratch. */
orthrus_status orthrus_draft_block(const void* plan, const int32_t* pending, int32_t K, int32_t* draft, float* logits,
                                   orthrus_stream stream);

/* Verify view (HN summary "Idea": the AR head verifies in a second pass).
 * Causal forward of the frozen model over [pending, draft[0..K-1]] at
 * positions len..len+K. Writes ar_argmax (device int32 [batch][K+1]) with
 * g_0..g_K and the block's base K/V into cache slots [len, len+K]; len is not
 * changed. K = 0 is plain greedy AR decoding of one token. logits (nullable):
 * fp32 [batch][K+1][vocab]. Device error ORTHRUS_ERR_CAPACITY if
 * len + K + 1 > capacity (the block is then not written). */
orthrus_status orthrus_verify_block(const void* plan, const int32_t* pending, const int32_t* draft, int32_t K,
                                    int32_t* ar_argmax, float* logits, orthrus_stream stream);

/* Greedy consensus and KV commit (HN summary "Idea": accept the longest
 * matching prefix; opentrain.ai abstract: exact consensus). Per sequence:
 * a = number of leading i with draft[i-1] == ar_argmax[i-1]; committed[b] =
 * d_1..d_a, g_a, then -1 up to K+1 entries; accept_len[b] = a;
 * cache.len[b] += a + 1; pending[b] = g_a. With poison_dead != 0 the dead
 * verify slots [len+a+1, len+K] of every layer are overwritten with NaN
 * (a check that nothing reads past len). All device int32 arrays. */
orthrus_status orthrus_accept_commit(const void* plan, int32_t* pending, const int32_t* draft,
                                     const int32_t* ar_argmax, int32_t K, int32_t* accept_len, int32_t* committed,
                                     int32_t poison_dead, orthrus_stream stream);

/* One full Orthrus step: draft view, (planted drafts copied over the draft
 * view's output when `planted` is not NULL: device int32 [batch][K]), verify
 * view, accept/commit. pending is updated in place; accept_len [batch] and
 * committed [batch][K+1] as in orthrus_accept_commit. */
orthrus_status orthrus_decode_step(const void* plan, int32_t* pending, int32_t K, const int32_t* planted,
                                   int32_t* accept_len, int32_t* committed, orthrus_stream stream);

/* Second (and further) denoising step of the draft view: the 2-step iterative
 * variant that the single-step block projection is compared with (atlas
 * summary "Surprising findings"). The pages leave the mechanism open; this
 * call takes the plainest reading: the draft view runs again over
 * [pending, prev_draft[0..K-2]] at positions len..len+K-1 (the previous step's
 * predictions in place of the masks; prev_draft[K-1] has no input slot and is
 * not read) and writes the new argmaxes to draft (device int32 [batch][K]).
 * draft may be the same buffer as prev_draft (ids are read before any is
 * written). logits (nullable): fp32 [batch][K][vocab]. The cache is read only.
 * Errors: ORTHRUS_ERR_ARG (NULL pointers, K outside [1, max_block]); a draft
 * id outside [0, vocab) sets the device status ORTHRUS_ERR_ARG. */
orthrus_status orthrus_draft_refine(const void* plan, const int32_t* pending, const int32_t* prev_draft, int32_t K,
                                    int32_t* draft, float* logits, orthrus_stream stream);

/* orthrus_decode_step with draft_steps (1..8) denoising steps of the draft
 * view: one orthrus_draft_block, then draft_steps - 1 orthrus_draft_refine in
 * place, then (planted, verify, consensus) as orthrus_decode_step, which is
 * this call with draft_steps = 1. */
orthrus_status orthrus_decode_step_ex(const void* plan, int32_t* pending, int32_t K, int32_t draft_steps,
                                      const int32_t* planted, int32_t* accept_len, int32_t* committed,
                                      orthrus_stream stream);

/* ---- decoding at temperature T > 0 (rejection sampling) ----------------
 * The pages name rejection sampling as the method at T > 0 and describe it
 * only briefly (atlas summary "Limitations"). These calls implement standard
 * speculative sampling (Leviathan et al. 2023; Chen et al. 2023) on the
 * Orthrus block, with every random number an input uniform on [0, 1):
 *   q_i = softmax(draft logits row i / T), i = 0..K-1; d_{i+1} ~ q_i;
 *   p_j = softmax(verify logits row j / T), j = 0..K;
 *   d_i accepted iff u_accept[i-1] * q_{i-1}(d_i) < p_{i-1}(d_i), in order up
 *   to the first rejection (a = number accepted); the last committed token is
 *   drawn with u_final from max(0, p_a - q_a) (normalised) if d_{a+1} was
 *   rejected, else from p_K (the bonus token).
 * The committed tokens are then distributed as sampling from the frozen model
 * at temperature T. A categorical draw with the uniform v is the inverse CDF:
 * the first index (in index order) with positive weight whose running sum
 * exceeds v times the total, sums in fp32. */

/* One draw per row: out[r] ~ softmax(logits[r] / temperature) with
 * uniforms[r]. logits: device fp32 [rows][vocab] (4-byte alignment is
 * enough); uniforms: device fp32 [rows]; out: device int32 [rows].
 * 1 <= vocab <= 262144; temperature > 0 and finite. status (device int32,
 * nullable): set to ORTHRUS_ERR_NAN (and out[r] = -1) when a row holds a NaN
 * or +inf logit or only -inf. Errors: ORTHRUS_ERR_ARG. No plan needed. */
orthrus_status orthrus_sample_tokens(const float* logits, int32_t rows, int32_t vocab, float temperature,
                                     const float* uniforms, int32_t* out, int32_t* status, orthrus_stream stream);

/* Rejection-sampling consensus and KV commit (the T > 0 counterpart of
 * orthrus_accept_commit, with the same outputs and bookkeeping: committed[b] =
 * d_1..d_a, last token, then -1; accept_len[b] = a; cache.len[b] += a + 1;
 * pending[b] = last token). draft: device int32 [batch][K]; draft_logits:
 * fp32 [batch][K][vocab] (the orthrus_draft_block logits the drafts were drawn
 * from); verify_logits: fp32 [batch][K+1][vocab] (orthrus_verify_block's);
 * u_accept: fp32 [batch][K]; u_final: fp32 [batch]. K = 0 draws one token
 * from p_0: plain sampled AR decoding (draft, draft_logits, u_accept may then
 * be NULL). The row statistics go to the workspace. With the device status
 * set (NaN logit, earlier error) nothing is committed and accept_len = -1.
 * Errors: ORTHRUS_ERR_ARG. */
orthrus_status orthrus_accept_sample(const void* plan, int32_t* pending, const int32_t* draft,
                                     const float* draft_logits, const float* verify_logits, int32_t K,
                                     float temperature, const float* u_accept, const float* u_final,
                                     int32_t* accept_len, int32_t* committed, orthrus_stream stream);

/* One Orthrus step at temperature T: draft view (logits to draft_logits),
 * drafts drawn with u_draft (fp32 [batch][K]), verify view (logits to
 * verify_logits), orthrus_accept_sample. draft_logits [batch][K][vocab] and
 * verify_logits [batch][K+1][vocab] are caller-owned fp32 device buffers.
 * Outputs as orthrus_accept_sample. */
orthrus_status orthrus_decode_step_sampled(const void* plan, int32_t* pending, int32_t K, float temperature,
                                           const float* u_draft, const float* u_accept, const float* u_final,
                                           float* draft_logits, float* verify_logits, int32_t* accept_len,
                                           int32_t* committed, orthrus_stream stream);

/* ---- dynamic block size --------------------------------------------------
 * The pages leave K to future work: choose it by how certain the generation
 * is, larger for predictable text (code completion), smaller for open-ended
 * text (news article, "Future Directions: Larger K and Higher Acceptance",
 * item 1). Here certainty is the per-position acceptance rate alpha: a draft
 * position is accepted with probability alpha until the first rejection, so a
 * block of K drafts commits
 *     E[a + 1 | K] = 1 + alpha + alpha^2 + ... + alpha^K
 * tokens on average. Among candidate block sizes with measured step times, the
 * policy picks the one that commits the most tokens per unit time, summed over
 * the batch (one K serves every sequence of a launch). These calls run on the
 * host only: no GPU, no stream; the caller feeds them the host copy of each
 * step's accept lengths. */

/* Running acceptance counts of one sequence, exponentially forgotten. */
typedef struct {
  float accepted; /* decayed sum of accepted drafts (the accept lengths a)        */
  float rejected; /* decayed number of steps that ended in a rejection (a < K)    */
} orthrus_accept_stats;

/* stats[b] = decay * stats[b] + (a_b, 1 if a_b < K else 0) for b < batch, with a_b =
 * accept_len[b] of a step run at block size K; a negative a_b (a failed step) leaves
 * stats[b] unchanged. decay in (0, 1] (1 = plain counts). Errors: ORTHRUS_ERR_ARG
 * (NULL pointers, batch < 1, K outside [0, 64], decay outside (0, 1], a_b > K). */
orthrus_status orthrus_accept_stats_update(orthrus_accept_stats* stats, const int32_t* accept_len, int32_t batch,
                                           int32_t K, float decay);

/* alpha of one sequence: (accepted + 1) / (accepted + rejected + 2), the rate of the
 * censored geometric counts under Laplace's rule of succession (1/2 with no data).
 * Returns -1 for a NULL pointer or negative counts. */
float orthrus_accept_rate(const orthrus_accept_stats* stats);

/* The K among ks[0 .. n_options) that maximises sum_b E[a_b + 1 | K] / step_ms[i] with
 * alpha_b = orthrus_accept_rate(&stats[b]); ties go to the smaller K. Every ks[i] in
 * [1, 64] and step_ms[i] > 0 (the caller's measured time of one decode step at K = ks[i]).
 * Returns that K, or -1 on bad arguments. */
int32_t orthrus_choose_block_size(const orthrus_accept_stats* stats, int32_t batch, const int32_t* ks,
                                  const float* step_ms, int32_t n_options);

/* ---- single kernels, exposed for parity tests and microbenchmarks ------ */

/* Block attention (the K1 kernel alone) for one layer's cache:
 *   q        fp16 [batch][Hkv][Q*G][d]: row i*G + g is query head kvh*G+g at block position i
 *            (post-norm, post-RoPE);
 *   k_cache, v_cache  fp16 [batch][Hkv][capacity][d];
 *   k_blk, v_blk      fp16 [batch][Hkv][blk_stride][d] (draft mode only: the
 *            block's own K/V, blk_stride >= Q);
 *   len      device int32 [batch]: cache rows [0, len[b]) precede the block;
 *   mode 0 = draft: every row sees cache[0,len) and block rows [0,Q);
 *   mode 1 = verify: the block's K/V already sit in cache slots [len, len+Q);
 *            row i sees cache[0, len+i].
 *   out      bf16 [2][batch*Q][H*d] (token-major, head h at columns h*d..): the
 *            result x as two planes, hi = bf16(x) then lo = bf16(x - hi).
 * Scratch comes from `workspace` (orthrus_attention_workspace_bytes). */
size_t orthrus_attention_workspace_bytes(int32_t batch, int32_t n_kv_heads, int32_t group, int32_t Q, int32_t head_dim,
                                         int32_t capacity);
orthrus_status orthrus_attention(const void* q, const void* k_cache, const void* v_cache, const void* k_blk,
                                 const void* v_blk, const int32_t* len, int32_t batch, int32_t n_kv_heads,
                                 int32_t group, int32_t Q, int32_t head_dim, int32_t capacity, int32_t blk_stride,
                                 int32_t mode, void* out, void* workspace, size_t workspace_bytes,
                                 int32_t* status, orthrus_stream stream);

/* Y[M][N] = X[M][Kd] * W[N][Kd]^T on the tensor cores (the K2 kernel with a
 * plain fp32 store epilogue). X, W bf16; Y fp32. N a multiple of 128, Kd a
 * multiple of 64. Scratch from `workspace` (orthrus_linear_workspace_bytes). */
size_t orthrus_linear_workspace_bytes(int32_t M, int32_t N, int32_t Kd);
orthrus_status orthrus_linear(const void* X, const void* W, float* Y, int32_t M, int32_t N, int32_t Kd,
                              void* workspace, size_t workspace_bytes, int32_t* status, orthrus_stream stream);

/* Allocation-free variant of orthrus_linear. This entry point has no
 * counterpart in the paper; it exists for callers that cannot allocate device
 * memory, such as a plugin or custom-operator interface that is handed only its
 * input and output buffers by a host framework owning all device memory, or a
 * runtime that works inside a fixed, pre-reserved memory budget.
 * Same operation and arguments as orthrus_linear, without the workspace: the
 * scratch (split-tile partial sums and tile counters) lives in a static device
 * array of 4 MiB + 64 KiB inside the library, which every GPU that loads the
 * library holds until the process exits. The call allocates nothing.
 * Limits: (M+127)/128 * N/128 <= 16384 weight tiles, else ORTHRUS_ERR_WORKSPACE;
 * the GEMM runs on at most 32 CTAs so the partial sums fit the array.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current); make that first call before any stream
 * capture. All calls share the one array and it keeps the previous call's
 * contents (the call clears the tile counters itself): calls that overlap on the
 * GPU (different streams, or concurrent host threads) race and must not be
 * issued. status: device int32 or NULL. */
orthrus_status orthrus_linear_noalloc(const void* X, const void* W, float* Y, int32_t M, int32_t N, int32_t Kd,
                                      int32_t* status, orthrus_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* ORTHRUS_H */
