// Host-side declarations shared by the libdflash translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "../../include/dflash.h"

namespace dfl {

constexpr int kNumSMs = 148;
constexpr int kMaxLayers = 16;
constexpr int kMaxTargetLayers = 16;
constexpr int kMaxBlock = 32;

// Host launch counter (dflash_launch_count).
void count_launch(int n = 1);

// ---------------------------------------------------------------- GEMM
// Weight-stationary GEMM with a fused epilogue.  For every output segment s
// (a weight matrix W_s [rows_s][K], or a gate/up pair for SwiGLU) and every
// token m of X [M][K]:  y[m][r] = sum_k X[m][k] W_s[r][k], then the
// segment's epilogue op writes the result.
constexpr int kMaxSegs = 3;
enum EpiOp { EPI_NONE = 0, EPI_STORE = 1, EPI_RESID = 2, EPI_SWIGLU = 3, EPI_STORE_F32 = 4 };

struct GemmOut {
  const void* w0;      // weights [rows][K]; the gate matrix for EPI_SWIGLU
  const void* w1;      // EPI_SWIGLU: the up matrix [rows][K]
  int rows;            // output features of the segment
  int op;              // EPI_STORE: out = y (dtype), optional RoPE and row scatter
                       // EPI_RESID: fp32 out += y
                       // EPI_SWIGLU: out = silu(y_gate) * y_up (dtype)
                       // EPI_STORE_F32: fp32 out = y (no RoPE, no scatter)
  int rope;            // EPI_STORE: rotate-half RoPE over heads of head_dim
  void* out;
  int64_t out_stride;  // elements between output rows
  int use_dst;         // EPI_STORE: token m goes to output row dst[m]
};

struct GemmJob {
  GemmOut seg[kMaxSegs];
  int nseg = 0;
  const void* x = nullptr;   // [M][K] dtype
  int64_t M = 0;
  int K = 0;
  int dtype = 0;
  const int32_t* pos = nullptr;   // RoPE positions [M]
  const int64_t* dst = nullptr;   // [M]
  int head_dim = 0;
  double theta = 1e6;
  const float2* rope_tab = nullptr;   // (cos, sin) [rope_len][head_dim / 2]
  int rope_len = 0;
  // EPI_STORE rows scaled by rsqrt(sum_w rss[m][w] * rss_inv + rss_eps) (the
  // RMSNorm of an unnormalised input row; rss [M][rss_parts]; nullptr: no
  // scale; bf16 tensor-core paths only)
  const float* rss = nullptr;
  int rss_parts = 0;
  float rss_inv = 0.f;
  float rss_eps = 0.f;
};

struct GemmPlan {
  int tok_major;     // 1: tokens on the MMA's M (large M), features per tile = bn
  int stream_k;      // 1: persistent stream-K weight-major kernel (small M)
  int sk_grid;       // its CTAs
  int sk_slots;      // partial slots reserved per tile
  int bn;            // token tile (weight-major) or feature tile (token-major)
  int row_tiles;     // tiles along the output features (all segments)
  int tok_tiles;
  int two;           // token-major on CTA pairs (cta_group::2, 256-feature tiles)
  int splits;        // K splits
  int kb_per_split;  // k-blocks per split
  size_t partial_floats;
  size_t counters;
};

GemmPlan plan_gemm(const GemmJob& job);
// Launch (one kernel for bf16; GEMM + finish for fp32).  `partial` and
// `counters` are workspace regions of plan.partial_floats floats and
// plan.counters words; counters must be zero (they are left zero).
cudaError_t launch_gemm(const GemmJob& job, const GemmPlan& plan, float* partial,
                        uint32_t* counters, uint32_t* status, cudaStream_t st);

// LM head: keys[m] = max over v of argmax_key(x[m] . W[v], v).  keys must be
// zero on entry (launch_argmax_finish leaves them zero).  With `partial`
// (plan_lmhead().partial_floats floats) and `counters` (zero, left zero) the
// small-M path runs the stream-K kernel; without them, one CTA per tile.
// With `lse` ([lmhead_tiles()][M]) every vocabulary tile also leaves its
// (max, sum exp) share of each token's log-sum-exp for the confidence.
GemmPlan plan_lmhead(int dtype, int V, int64_t M, int K);
int lmhead_tiles(int dtype, int V, int64_t M);
cudaError_t launch_lmhead_argmax(int dtype, const void* W, int V,
                                 const void* X, int64_t M, int K,
                                 unsigned long long* keys, uint32_t* status,
                                 cudaStream_t st, float* partial = nullptr,
                                 uint32_t* counters = nullptr, float2* lse = nullptr);

// ---------------------------------------------------------------- others
cudaError_t launch_fuse(int dtype, const void* states, int64_t N, int T, int H,
                        int D, const float* w_fuse, const float* const* g_fuse,
                        void* fused, float eps, uint32_t* status, cudaStream_t st);
// bf16 fusion for the step's context branch without the norm: fused[i][n] =
// u_i * g_i and rss[i][n][w] = consumer warp w's share of sum(u_i^2), for
// w < fuse_unnorm_parts(H); the context K/V GEMM applies rsqrt(sum / H + eps)
// per row (GemmJob::rss).
int fuse_unnorm_parts(int H);
cudaError_t launch_fuse_unnorm(const void* states, int64_t N, int nT, int H, int D,
                               const float* w_fuse, const float* const* g_fuse, void* fused,
                               float* rss, uint32_t* status, cudaStream_t st);
// Largest hidden size the fusion kernel covers for T target layers.
int fuse_hidden_limit(int dtype, int nT);
cudaError_t launch_embed(int dtype, const void* embed, int H, int nb, int B,
                         const int32_t* block_tokens, const int32_t* known_len,
                         int mask_id, int vocab, float* h, uint32_t* status, cudaStream_t st);
cudaError_t launch_rmsnorm(int dtype, const float* h, int64_t M, int H,
                           const float* g, float eps, void* x, cudaStream_t st);
cudaError_t launch_prep_rows(int R, int nb, int B, const int32_t* block_req,
                             const int64_t* ctx_off, const int64_t* new_off,
                             const int32_t* ctx_cached, const int32_t* ctx_len,
                             const int32_t* new_count, int64_t n_new,
                             int32_t* blk_pos, int32_t* new_pos,
                             int64_t* new_dst, uint32_t* zero, int64_t n_zero,
                             uint32_t* status, cudaStream_t st);
cudaError_t launch_advance(int R, int K, int B, int64_t row_bytes, const int32_t* n_acc,
                           const int32_t* best_k, const int32_t* out_tok, const void* verify_states,
                           int32_t* ctx_len, const int64_t* ctx_off, void* new_states,
                           int32_t* new_count, int32_t* block_tokens, int32_t* known_len,
                           int mask_id, uint32_t* status, cudaStream_t st);
// tokens (+ max logit) from the argmax keys; resets the keys to zero.
cudaError_t launch_argmax_finish(unsigned long long* keys, int64_t M,
                                 int B, const int32_t* block_tokens,
                                 const int32_t* known_len, int32_t* tok,
                                 float* max_logit, cudaStream_t st,
                                 const float2* lse = nullptr, int lse_tiles = 0,
                                 float* conf = nullptr);
cudaError_t launch_zero(void* p, size_t bytes, cudaStream_t st);
// RoPE table: tab[p][i] = (cos, sin)(p * theta^(-2i/d)), p < len, i < d/2.
cudaError_t launch_rope_table(float2* tab, int len, int head_dim, double theta,
                              cudaStream_t st);

// Kernel launch with programmatic dependent launch enabled: the kernel may
// start while the previous kernel on the stream finishes; every kernel of
// this library calls pdl_wait() before touching memory the previous kernel
// may write.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

struct AttnPlan {
  int splits;
  int chunk;        // context keys per split (multiple of 64)
  int row_chunks;   // CTAs along the query rows of one (block, kv head)
  int rows_per_cta;
  int cluster;      // bf16: splits merged in one CTA cluster (power of two); 0: combine kernel
};
AttnPlan plan_attn(int dtype, int nb, int B, int Hq, int Hkv, int d,
                   int64_t max_ctx_len);
size_t attn_ws_bytes(const AttnPlan& p, int nb, int B, int Hq, int d);
// ctx_len (nullable): request r has ctx_len[r] context rows from ctx_off[r]
// (else ctx_off[r + 1] - ctx_off[r]).
cudaError_t launch_attn(int dtype, const AttnPlan& plan, int nb, int B, int Hq,
                        int Hkv, int d, const void* q, const void* kb,
                        const void* vb, const void* kc, const void* vc,
                        const int64_t* ctx_off, const int32_t* block_req,
                        void* out, float* ws, uint32_t* status, cudaStream_t st,
                        const int32_t* ctx_len = nullptr);

cudaError_t launch_accept(int R, int K, int B, const int32_t* draft,
                          const int32_t* target, int32_t* n_acc,
                          int32_t* best_k, int32_t* out_tok, cudaStream_t st);
cudaError_t launch_d2sd(int R, int B, int K, int mask_id, const int32_t* base,
                        const float* conf, int32_t* known_len, int32_t* cand,
                        int32_t* block_req, cudaStream_t st);
// Temperature-1 sampling (sampling.cu): Gumbel-max draw per stored logit
// row (row ids 0..M-1 select the noise); known-prefix slots keep their input.
cudaError_t launch_sample_rows(const float* logits, int64_t M, int V, uint64_t seed,
                               uint32_t offset, int B, const int32_t* block_tokens,
                               const int32_t* known_len, int32_t* tok, float* logq,
                               float* lse, uint32_t* status, cudaStream_t st);
// Stochastic acceptance of one candidate per request; keys [R] scratch.
cudaError_t launch_accept_stochastic(int R, int B, int V, const int32_t* draft,
                                     const float* draft_logits, const float* draft_lse,
                                     const float* target_logp, uint64_t seed, uint32_t offset,
                                     int32_t* n_acc, int32_t* out_tok,
                                     unsigned long long* keys, uint32_t* status,
                                     cudaStream_t st);
cudaError_t launch_wait_selftest(uint32_t* status, int64_t limit_ns,
                                 cudaStream_t st);

// Tensor maps (driver entry point fetched through the runtime).
bool encode_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner,
                         uint64_t outer, uint32_t box_inner, uint32_t box_outer);
// 3-D bf16 map, dims (d0 fastest, d1, d2), dense strides, 128-byte swizzle.
bool encode_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                         uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2);

}  // namespace dfl
