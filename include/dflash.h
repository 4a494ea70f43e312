/*
 * dflash.h -- C ABI of libdflash.so: the single-pass block-diffusion draft
 * step of speculative decoding and its greedy verification, on one B200
 * (sm_100a).
 *
 * What is computed (web summaries of three papers):
 *   - "DFlash: Block Diffusion for Flash Speculative Decoding", methodology
 *     steps 1-4: the target's hidden states condition a draft model that
 *     emits a whole block of tokens in one forward pass; the target checks
 *     the block in parallel, the accepted tokens are emitted at once and the
 *     first rejected slot is replaced by the target's own token.
 *   - "DFLARE" summary, section 2.1: draft layer i fuses the T target layers
 *     with its own weights alpha^(i) = softmax(W_fuse[i, :]), then RMSNorm;
 *     section 2.2: separate projections W^t_K, W^t_V for the target context
 *     and W^d_K, W^d_V for the draft block's own hidden states.
 *   - "D2SD" summary, methodology steps 2-4: K prefixes of the first draft,
 *     cut at its lowest-confidence slots, are re-drafted in one batched pass
 *     and the longest accepted candidate wins.
 *
 * Conventions (every entry point):
 *   - Tensors are caller-owned DEVICE pointers unless marked "host".  The
 *     library never allocates or frees device memory; scratch space comes
 *     from a caller workspace sized by dflash_workspace_size().
 *   - Row-major layouts.  Weights are [out][in] (the nn.Linear layout).
 *     Token ids are int32.  Activations and weights are fp32 when
 *     cfg->dtype == DFLASH_FP32 and bf16 when cfg->dtype == DFLASH_BF16;
 *     RMSNorm gains and W_fuse are always fp32; the residual stream h is
 *     always fp32.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls enqueue work asynchronously and return; they launch
 *     nothing when they return an error.
 *   - Every argument is validated on the host before any launch; a bad
 *     argument returns DFLASH_EINVAL (or DFLASH_EUNSUPPORTED for a shape the
 *     kernels do not cover) and dflash_last_error() says which.
 *   - Errors found on the device (a non-finite logit, a bounded wait that
 *     ran out) are recorded in the first bytes of the workspace;
 *     dflash_check() synchronises the stream and returns them.
 *   - Calls are stateless and thread-safe as long as concurrent calls use
 *     different workspaces.
 *   - Weight, activation, state and cache pointers must be 16-byte aligned;
 *     token, index and per-token arrays (int32, fp32, int64) must be
 *     naturally aligned (4 or 8 bytes); hidden, ffn and head_dim must be
 *     multiples of 8 (bf16) or 4 (fp32).  A misaligned pointer is refused
 *     with DFLASH_EINVAL before any launch.
 */
#ifndef DFLASH_H_
#define DFLASH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DFLASH_OK = 0,
  DFLASH_EINVAL = 1,       /* bad argument (null pointer, bad size, ...) */
  DFLASH_EUNSUPPORTED = 2, /* valid but not covered (e.g. head_dim 96) */
  DFLASH_ECUDA = 3,        /* a CUDA runtime call failed */
  DFLASH_ETIMEOUT = 4,     /* a bounded device-side wait ran out */
  DFLASH_ENUMERIC = 5,     /* a non-finite logit reached the LM-head argmax */
  DFLASH_EBOUNDS = 6       /* debug-bounds build only (libdflash_debug.so, compiled
                            * with -DDFLASH_DEBUG_BOUNDS): an index read from
                            * device memory (a request id, a context length, a
                            * new-row count, a token id) fell outside its
                            * buffer; the access was skipped, no trap */
} dflash_status;

typedef enum { DFLASH_FP32 = 0, DFLASH_BF16 = 1 } dflash_dtype;

/* Model shapes.  B <= 32; head_dim in {64, 128}; n_q_heads a multiple of
 * n_kv_heads (GQA); n_draft_layers D <= 16; n_target_layers T <= 16. */
typedef struct {
  int32_t hidden;          /* H */
  int32_t n_q_heads;       /* Hq */
  int32_t n_kv_heads;      /* Hkv */
  int32_t head_dim;        /* d */
  int32_t ffn;             /* F (SwiGLU width) */
  int32_t n_draft_layers;  /* D */
  int32_t n_target_layers; /* T */
  int32_t block;           /* B: anchor slot + B-1 mask slots */
  int32_t vocab;           /* V */
  int32_t mask_token_id;   /* embedding row used for masked slots */
  float rope_theta;        /* rotate-half RoPE base (Q and K) */
  float rms_eps;           /* RMSNorm epsilon */
  int32_t dtype;           /* dflash_dtype */
} dflash_config;

/* One draft layer's weights (device pointers). */
typedef struct {
  const void* w_q;     /* [Hq*d][H]   query projection */
  const void* w_kt;    /* [Hkv*d][H]  W^t_K: key projection of the fused target context */
  const void* w_vt;    /* [Hkv*d][H]  W^t_V */
  const void* w_kd;    /* [Hkv*d][H]  W^d_K: key projection of the draft block */
  const void* w_vd;    /* [Hkv*d][H]  W^d_V */
  const void* w_o;     /* [H][Hq*d]   attention output projection */
  const void* w_gate;  /* [F][H] */
  const void* w_up;    /* [F][H] */
  const void* w_down;  /* [H][F] */
  const float* g_fuse; /* [H] gain of the RMSNorm after the layer's fusion */
  const float* g_attn; /* [H] pre-attention RMSNorm gain */
  const float* g_mlp;  /* [H] pre-MLP RMSNorm gain */
} dflash_layer_weights;

typedef struct {
  const float* w_fuse;                /* [D][T] fusion logits (softmax over T per layer) */
  const dflash_layer_weights* layers; /* HOST array [D] */
  const void* embed;                  /* [V][H] slot embeddings */
  const float* g_final;               /* [H] final RMSNorm gain */
  const void* lm_head;                /* [V][H] */
  /* DFlash-style context fusion (DFLARE summary, section 1 item 1 and
   * section 2.2, describing the DFlash baseline).  NULL (the default): every
   * draft layer fuses the T target layers with its own softmax weights
   * (w_fuse, g_fuse).  Non-NULL: ONE fully connected layer maps the
   * concatenated target states of a row to a single context shared by all
   * draft layers, c = RMSNorm_{g_fc}(concat(h_1..h_T) W_fc^T); w_fuse and the
   * layers' g_fuse are then unused.  (DFlash also shares the K/V projection
   * between context and block: pass w_kt = w_kd and w_vt = w_vd.) */
  const void* w_fc;                   /* [H][T*H] (nullable) */
  const float* g_fc;                  /* [H] fp32 (required with w_fc) */
} dflash_weights;

/* ------------------------------------------------------------------------
 * Workspace
 * ----------------------------------------------------------------------*/

/* Bytes of workspace needed by dflash_draft_step (and by any single-op call
 * below) for up to n_req requests, n_blocks blocks, n_ctx_new new context
 * rows in total and a longest context of max_ctx_len rows.  Returns 0 for an
 * invalid config.  Workspace must be 256-byte aligned. */
size_t dflash_workspace_size(const dflash_config* cfg, int32_t n_req,
                             int32_t n_blocks, int64_t n_ctx_new,
                             int64_t max_ctx_len);

/* Zero the workspace's status header (call once after allocating it). */
dflash_status dflash_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, then read and clear the device status recorded in
 * the workspace header by earlier calls that used `ws`.  Returns DFLASH_OK,
 * DFLASH_ETIMEOUT, DFLASH_ENUMERIC, DFLASH_EBOUNDS (debug-bounds build) or
 * DFLASH_ECUDA. */
dflash_status dflash_check(void* ws, void* stream);

/* Message describing the last error returned to the calling thread. */
const char* dflash_last_error(void);

/* Number of kernels this library has launched since it was loaded (a host
 * counter; launches replayed from a CUDA graph are not counted). */
uint64_t dflash_launch_count(void);

const char* dflash_version(void);

/* ------------------------------------------------------------------------
 * Steps of the draft pass (each usable on its own)
 * ----------------------------------------------------------------------*/

/* Adaptive layer fusion, DFLARE summary section 2.1.
 * states [N][T][H] (dtype) -> fused [D][N][H] (dtype):
 *   alpha_i = softmax(w_fuse[i, :]),  u = sum_j alpha_ij * states[n, j, :],
 *   fused[i, n, :] = u / sqrt(mean(u^2) + eps) * g_fuse[i][:].
 * w_fuse: device [D][T] fp32.  g_fuse: HOST array of D device pointers, each
 * [H] fp32.  N may be 0 (no launch). */
dflash_status dflash_fuse_ctx(const dflash_config* cfg, const void* states,
                              int64_t n_rows, const float* w_fuse,
                              const float* const* g_fuse, void* fused,
                              void* stream);

/* The draft step's split form of the same fusion (DFLARE summary, section
 * 2.1; the split itself is this library's, the pages normalise before the
 * projection of section 2.2), bf16 only.  RMSNorm is
 * one scalar per row, and the context K/V projection and RoPE are linear, so
 * dflash_draft_step applies the row scale in the projection's epilogue: the
 * fusion stores the rows unnormalised and needs no cross-warp reduction per
 * row.  Outputs:
 *   fused[i, n, :] = u * g_fuse[i][:]                    [D][N][H] bf16
 *   rss[i][n][w]   = partial sums of u^2, w < P          [D][N][P] fp32
 * with P = dflash_fuse_rss_parts(hidden) and sum_w rss[i][n][w] = sum(u^2),
 * the parts added in a fixed order, so that
 *   dflash_fuse_ctx's fused[i, n, :] = fused[i, n, :] / sqrt(sum_w rss[i][n][w] / H + eps).
 * ws: a workspace of at least 256 bytes (its header takes the device status;
 * read it with dflash_check).  N may be 0 (no launch). */
int32_t dflash_fuse_rss_parts(int32_t hidden);
dflash_status dflash_fuse_ctx_rss(const dflash_config* cfg, const void* states,
                                  int64_t n_rows, const float* w_fuse,
                                  const float* const* g_fuse, void* fused, float* rss,
                                  void* ws, size_t ws_bytes, void* stream);

/* DFlash-style FC context fusion (DFLARE summary, section 1 item 1 and
 * section 2.2): states [N][T][H] (dtype), viewed as [N][T*H] ->
 *   fused[n, :] = RMSNorm_{g_fc}(states[n] W_fc^T)   [N][H] (dtype)
 * w_fc [H][T*H] (dtype), g_fc [H] fp32.  The fp32 product is staged in the
 * workspace (N*H*4 bytes after the header); N may be 0 (no launch). */
dflash_status dflash_fc_fuse_ctx(const dflash_config* cfg, const void* states,
                                 int64_t n_rows, const void* w_fc,
                                 const float* g_fc, void* fused, void* ws,
                                 size_t ws_bytes, void* stream);

/* K/V projection, DFLARE summary section 2.2 (called with W^t for context
 * rows and with W^d for block rows):
 *   k_out[dst(m)] = RoPE(x[m] W_K^T, pos[m]),  v_out[dst(m)] = x[m] W_V^T
 * x [M][H]; pos device [M] int32 (RoPE position); dst_row device [M] int64
 * (destination row in k_out/v_out, NULL = m); k_out/v_out [rows][Hkv][d]
 * (may be a packed context KV cache).  RoPE is rotate-half with
 * inv_freq_i = theta^(-2i/d). */
dflash_status dflash_kv_project(const dflash_config* cfg, const void* x,
                                int64_t M, const int32_t* pos,
                                const int64_t* dst_row, const void* w_k,
                                const void* w_v, void* k_out, void* v_out,
                                void* ws, size_t ws_bytes, void* stream);

/* Block attention (KV injection, DFLARE summary section 2.2): for block b
 * of request r = block_req[b] and query head h,
 *   out = softmax(q K^T / sqrt(d)) V  over keys [ctx KV of r ; block KV of b],
 * with q head h reading kv head h / (Hq/Hkv), no mask.
 * q, out [nb*B][Hq][d]; k_blk, v_blk [nb*B][Hkv][d]; k_ctx, v_ctx packed
 * [sum L][Hkv][d]; ctx_off device [R+1] int64 row offsets of each request's
 * context (L_r = ctx_off[r+1] - ctx_off[r], may be 0); block_req device [nb]
 * int32; max_ctx_len = max_r L_r (host, sizes the split-KV grid).  The
 * packed caches may hold at most 2^28 rows (bf16 path: the TMA tensor maps
 * over them span that many rows). */
dflash_status dflash_block_attn(const dflash_config* cfg, int32_t n_blocks,
                                const void* q, const void* k_blk,
                                const void* v_blk, const void* k_ctx,
                                const void* v_ctx, const int64_t* ctx_off,
                                const int32_t* block_req, int64_t max_ctx_len,
                                void* out, void* ws, size_t ws_bytes,
                                void* stream);

/* Pre-norm SwiGLU MLP with residual, in place on fp32 h [M][H]:
 *   x = RMSNorm_{g_mlp}(h);  h += (silu(x W_gate^T) * (x W_up^T)) W_down^T. */
dflash_status dflash_mlp(const dflash_config* cfg, int64_t M, float* h,
                         const float* g_mlp, const void* w_gate,
                         const void* w_up, const void* w_down, void* ws,
                         size_t ws_bytes, void* stream);

/* LM head with the argmax fused in (logits never reach memory):
 *   tok[m] = the lowest v with x[m] . w_lm[v] maximal;  max_logit[m] = that
 *   maximum (nullable);  conf[m] (nullable) = softmax probability of tok[m]
 *   = 1 / sum_v exp(z_v - max z), the per-position confidence the D2SD
 *   summary (methodology step 1) asks the first drafter for.  x [M][H]
 *   (already normed); w_lm [V][H]. */
dflash_status dflash_lmhead_argmax(const dflash_config* cfg, int64_t M,
                                   const void* x, const void* w_lm,
                                   int32_t* tok, float* max_logit, float* conf,
                                   void* ws, size_t ws_bytes, void* stream);

/* Greedy verification, DFlash summary methodology step 3 and D2SD summary
 * methodology step 4.  draft, target: [R][K][B] int32; slot 0 of a block is
 * the anchor and target[j] is the target's argmax after slots 0..j.
 *   n_k   = max m <= B-1 with draft[k][j] == target[k][j-1] for 1 <= j <= m
 *   best  = lowest k with maximal n_k
 *   n_acc[r] = n_best, best_k[r] = best,
 *   out_tok[r] = draft[best][1..n], target[best][n], then -1 up to B.
 * B <= 32, K <= 32.  R == 0 launches nothing.  No workspace. */
dflash_status dflash_accept(int32_t R, int32_t K, int32_t B,
                            const int32_t* draft, const int32_t* target,
                            int32_t* n_acc, int32_t* best_k, int32_t* out_tok,
                            void* stream);

/* D2SD prefix selection, D2SD summary methodology steps 2-3.  For each
 * request the K slots of 1..B-1 with the lowest confidence (ties: lower
 * slot) are the cuts p_1 < ... < p_K; candidate k = r*K + k keeps slots
 * 0..p_k-1 of base_tokens[r] and masks the rest:
 *   known_len[r*K+k] = p_k,  cand_tokens[r*K+k][s] = s < p_k ? base : mask.
 * block_req (nullable) receives r for every candidate.  1 <= K <= B-1. */
dflash_status dflash_d2sd_candidates(int32_t R, int32_t B, int32_t K,
                                     int32_t mask_token_id,
                                     const int32_t* base_tokens,
                                     const float* conf, int32_t* known_len,
                                     int32_t* cand_tokens, int32_t* block_req,
                                     void* stream);

/* LM-head argmax that allocates nothing and takes no workspace.  The pages
 * have no counterpart to this entry point; it exists for callers that cannot
 * call cudaMalloc or hand over a workspace -- e.g. a plugin inside a serving
 * process whose device memory belongs to that process's caching allocator,
 * or a real-time loop that must not allocate after start-up.
 * Computes exactly what dflash_lmhead_argmax computes.  Its scratch (one
 * 8-byte key per token) is a fixed array in the library's device globals,
 * present on every GPU that loads the library until the process exits, so:
 *   - M may be at most 4096 tokens; larger M returns DFLASH_EINVAL;
 *   - the first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture;
 *   - all calls share the array: calls that overlap on the GPU (different
 *     streams, or different host threads on one device) race;
 *   - the cached address stays valid until the device's primary context is
 *     reset (cudaDeviceReset); do not call this entry point after a reset;
 *   - device-side errors are NOT reported: there is no workspace header, so
 *     neither a non-finite logit (DFLASH_ENUMERIC) nor a bounded wait that
 *     ran out (DFLASH_ETIMEOUT) reaches the caller, and the tokens of such a
 *     call are undefined; callers that need those checks use
 *     dflash_lmhead_argmax with a workspace and dflash_check;
 *   - with at most 64 tokens it runs the one-CTA-per-tile weight-streaming
 *     kernel (the stream-K kernel of dflash_lmhead_argmax needs workspace
 *     partials), so at batch 1 it is somewhat slower than that entry point;
 *     65 tokens and more take the same token-major kernel as it does. */
dflash_status dflash_lmhead_argmax_noalloc(const dflash_config* cfg, int64_t M,
                                           const void* x, const void* w_lm,
                                           int32_t* tok, float* max_logit,
                                           void* stream);

/* ------------------------------------------------------------------------
 * Temperature-1 drafting and stochastic verification
 *
 * DFlash summary, methodology step 3 (the standard speculative acceptance
 * test, a comparison of log probabilities; the first rejected slot is filled
 * by the target's own generation) and DFLARE summary, section 4 (stochastic
 * decoding at temperature 1).  Readings: each drafted slot is sampled from
 * the draft's softmax q_j by the Gumbel-max rule; slot j is accepted while
 * log U_j < log p_j(d_j) - log q_j(d_j); the token at the first rejected
 * slot is drawn from norm(max(0, p_j - q_j)) (the draw that keeps the
 * emitted tokens distributed as the target's), and when every slot passes
 * one more token is drawn from the target's distribution for the next slot.
 * Every uniform is a Philox4x32-10 draw (Salmon et al., SC 2011) with key
 * (seed low 32 bits, seed high 32 bits) and counter words (c0, c1, c2, c3):
 *   draft noise, token row m, id v:      (v >> 2, m, offset, 0x44524654) word v & 3
 *   acceptance, request r, slot j:       (j, r, offset, 0x41435054)      word 0
 *   residual / next-slot noise, r, j, v: (v >> 2, 64 r + j, offset, 0x52455344) word v & 3
 * and a word x becomes U = (floor(x / 2^9) + 1/2) / 2^23 in (0, 1); the
 * Gumbel variate is -log(-log U).
 * ----------------------------------------------------------------------*/

/* LM head writing its logits: logits[m][v] = x[m] . w_lm[v] (fp32 [M][V]). */
dflash_status dflash_lmhead_logits(const dflash_config* cfg, int64_t M,
                                   const void* x, const void* w_lm,
                                   float* logits, void* ws, size_t ws_bytes,
                                   void* stream);

/* Gumbel-max draw of every row of logits [M][V] (fp32):
 *   tok[m] = argmax_v (logits[m][v] + G(seed, offset, m, v)) (lowest id on
 *   an exact tie); logq[m] = logits[m][tok[m]] - lse[m] (nullable);
 *   lse[m] = log sum_v exp(logits[m][v]) (nullable).  No workspace. */
dflash_status dflash_sample(const dflash_config* cfg, int64_t M,
                            const float* logits, uint64_t seed, uint32_t offset,
                            int32_t* tok, float* logq, float* lse, void* stream);

/* Stochastic acceptance, one candidate block per request.  draft [R][B]
 * int32 (slot 0 = anchor); draft_logits [R][B][V] fp32 with row logsumexp
 * draft_lse [R][B]; target_logp [R][B][V] fp32 log probabilities, row j =
 * the target's distribution for slot j+1 (after reading slots 0..j).
 *   n_acc[r] = accepted drafted slots; out_tok[r] = draft[r][1..n], the
 *   drawn token, then -1 up to B.
 * Needs 8 * R bytes of workspace after the header.  B <= 32. */
dflash_status dflash_accept_stochastic(int32_t R, int32_t B, int32_t V,
                                       const int32_t* draft,
                                       const float* draft_logits,
                                       const float* draft_lse,
                                       const float* target_logp, uint64_t seed,
                                       uint32_t offset, int32_t* n_acc,
                                       int32_t* out_tok, void* ws,
                                       size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The whole draft step (+ optional verification)
 * ----------------------------------------------------------------------*/

typedef struct {
  int32_t n_req;               /* R */
  int32_t n_blocks;            /* nb (blocks of one request may be several: D2SD) */
  int64_t n_ctx_new;           /* host: rows in new_states = sum_r (L_r - cached_r) */
  int64_t max_ctx_len;         /* host: max_r L_r */
  const int32_t* block_req;    /* [nb] request of each block */
  const int32_t* block_tokens; /* [nb][B] slot tokens; slots < known_len are used */
  const int32_t* known_len;    /* [nb] known leading slots (NULL = 1: anchor only) */
  const void* new_states;      /* [n_ctx_new][T][H] target states of the rows to add */
  const int64_t* ctx_off;      /* [R+1] row offsets of each request in the KV caches */
  const int64_t* new_off;      /* [R+1] row offsets in new_states (NULL = ctx_off) */
  const int32_t* ctx_cached;   /* [R] rows already in the caches (NULL = all 0) */
  void* const* k_cache;        /* host [D]: per layer, [sum L][Hkv][d] */
  void* const* v_cache;        /* host [D] */
  int32_t* draft_tokens;       /* out [nb][B]: slots < known_len copy the input */
  float* max_logit;            /* out [nb][B] (nullable) */
  float* confidence;           /* out [nb][B] (nullable): softmax probability of each
                                  drafted token (D2SD per-position confidence) */
  const int32_t* target_tokens;/* [nb][B] target argmax per slot (NULL = no verify) */
  int32_t n_cand;              /* K candidates per request in verification (nb = R*K) */
  int32_t* n_acc;              /* out [R] */
  int32_t* best_k;             /* out [R] */
  int32_t* out_tok;            /* out [R][B] */
  /* Temperature-1 mode (see dflash_sample / dflash_accept_stochastic).
   * sample = 0: greedy argmax drafting, greedy verification (the fields
   * below are unused).  sample = 1: the LM head writes draft_logits, every
   * drafted slot is a Gumbel-max draw (row ids b*B + s), and with
   * target_logp set the step verifies stochastically (n_cand must be 1);
   * target_tokens, max_logit and confidence are then unused. */
  int32_t sample;
  uint32_t rng_offset;         /* counter word c2 of every draw (e.g. the step number) */
  uint64_t seed;               /* Philox key */
  float* draft_logits;         /* out [nb][B][V] fp32 (required with sample = 1) */
  float* draft_logq;           /* out [nb][B] (nullable): log q of each drafted token */
  const float* target_logp;    /* [nb][B][V] fp32 (nullable: no verification) */
  /* Device-resident lengths, for a decode loop that never reads back to the
   * host between steps (see dflash_advance).  ctx_len (nullable): request r's
   * context is the ctx_len[r] rows starting at cache row ctx_off[r], and
   * ctx_off[r+1] - ctx_off[r] is its capacity; max_ctx_len must bound every
   * ctx_len (it sizes the attention split).  new_count (nullable, needs
   * ctx_len): new_states then holds B slots per request ([n_req][B][T][H],
   * n_ctx_new = n_req * B), of which the first new_count[r] are the context
   * rows ctx_len[r] - new_count[r] .. ctx_len[r] - 1; the other slots are
   * skipped (new_off and ctx_cached are then unused). */
  const int32_t* ctx_len;
  const int32_t* new_count;
} dflash_step_args;

/* One draft step (DFlash summary, methodology step 2; DFLARE sections
 * 2.1-2.2): fuse + project the new context rows into the caches for every
 * layer, then for every block run D layers of [RMSNorm -> Q, K^d, V^d ->
 * attention over (context ; block) -> O proj + residual -> RMSNorm ->
 * SwiGLU + residual], the final RMSNorm and the LM-head argmax.  Block slot
 * s sits at position L_r + s.  With target_tokens set it also runs
 * dflash_accept over the blocks grouped as [R][n_cand][B].
 * Rows [ctx_cached[r], L_r) of request r are (re)computed from new_states;
 * earlier rows are read from the caches as they are. */
dflash_status dflash_draft_step(const dflash_config* cfg,
                                const dflash_weights* w,
                                const dflash_step_args* a, void* ws,
                                size_t ws_bytes, void* stream);

/* Roll the speculative window forward on the device (DFlash summary,
 * methodology step 4; D2SD summary, methodology step 5), after verification
 * and before the next dflash_draft_step, with no host round trip.  For
 * request r with n = n_acc[r] accepted tokens of candidate k = best_k[r]
 * (best_k nullable = 0):
 *   new_states[r][j] = verify_states[r][k][j]   for j = 0 .. n
 *     (the target's hidden states of the verified block's anchor and
 *     accepted slots, [T][H] each; layouts [R][K][B][T][H] and [R][B][T][H])
 *   new_count[r] = n + 1;  ctx_len[r] += n + 1  (in place)
 *   block_tokens[r] = (out_tok[r][n], mask, ..., mask);  known_len[r] = 1
 * so that the next draft step, given ctx_len and new_count, fuses and
 * projects exactly the n + 1 new rows and drafts from the new anchor.
 * ctx_off [R+1] gives each request's cache capacity; a context that would
 * outgrow it is clipped there and DFLASH_EINVAL is recorded in the
 * workspace header (dflash_check reports it). */
dflash_status dflash_advance(const dflash_config* cfg, int32_t R, int32_t K,
                             const int32_t* n_acc, const int32_t* best_k,
                             const int32_t* out_tok, const void* verify_states,
                             int32_t* ctx_len, const int64_t* ctx_off,
                             void* new_states, int32_t* new_count,
                             int32_t* block_tokens, int32_t* known_len, void* ws,
                             size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Failure-detection self test
 * ----------------------------------------------------------------------*/

/* Launch one kernel that waits on a shared-memory barrier nothing will
 * arrive at, giving up after limit_ns nanoseconds (<= 2 s).  The kernel
 * records DFLASH_ETIMEOUT in the workspace header and returns, leaving the
 * context usable; dflash_check() then reports it.  This exercises the same
 * bounded-wait path every pipelined kernel of the library uses. */
dflash_status dflash_selftest_wait_timeout(void* ws, size_t ws_bytes,
                                           int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DFLASH_H_ */
