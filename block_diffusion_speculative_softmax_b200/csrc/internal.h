// Host-side declarations shared by the libdflash translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dflash.h"

namespace dfl {

constexpr int kNumSMs = 148;
constexpr int kMaxLayers = 16;
constexpr int kMaxTargetLayers = 16;
constexpr int kMaxBlock = 32;

// Host launch counter (dflash_launch_count).
void count_launch(int n = 1);

// ---------------------------------------------------------------- GEMM
// Partial products of a "weight-stationary" GEMM: for every segment s
// (a weight matrix W_s [rows_s][K]) and every token m of X [M][K]:
//   partial[split][m][col0_s + r] = sum_{k in split} X[m][k] * W_s[r][k].
struct GemmSeg {
  const void* w;
  int rows;
};
constexpr int kMaxSegs = 3;

struct GemmPlan {
  int bn;          // token tile (tcgen05 N) or SIMT token tile
  int splits;      // K splits
  int kb_per_split;
  int n_cols;      // sum of segment rows
};

// Split plan for M tokens, K reduction length, given segments.  Same plan
// for workspace sizing and for the launch.
GemmPlan plan_gemm(int dtype, const int* seg_rows, int nseg, int64_t M, int K);

cudaError_t launch_gemm_partial(int dtype, const GemmSeg* segs, int nseg,
                                const void* X, int64_t M, int K,
                                const GemmPlan& plan, float* partial,
                                uint32_t* status, cudaStream_t st);

// LM head: keys[m] = max over v of argmax_key(x[m] . W[v], v).
cudaError_t launch_lmhead_argmax(int dtype, const void* W, int V,
                                 const void* X, int64_t M, int K,
                                 unsigned long long* keys, uint32_t* status,
                                 cudaStream_t st);

// ---------------------------------------------------------------- epilogues
enum EpiOp { EPI_NONE = 0, EPI_STORE = 1, EPI_RESID = 2, EPI_SWIGLU = 3 };
struct EpiSeg {
  int op;             // EpiOp.  EPI_SWIGLU: this segment holds the gate, the
                      // next one the up projection; writes silu(g) * u.
  int rows;           // outputs of the segment
  int col0;           // column of the segment in the partial buffer
  int rope;           // rotate-half RoPE over heads of head_dim
  void* out;          // STORE/SWIGLU: dtype [*][out_stride]; RESID: fp32
  int64_t out_stride; // elements between output rows
  int use_dst;        // STORE: row m goes to dst_row[m]
};
struct EpiParams {
  EpiSeg seg[kMaxSegs];
  int nseg;
  int64_t M;
  int n_cols;
  int splits;
  const float* partial;
  const int32_t* pos;      // RoPE positions [M]
  const int64_t* dst_row;  // [M] or null
  int head_dim;
  int out_bf16;
  double inv_freq[64];
};
cudaError_t launch_gemm_finish(const EpiParams& p, cudaStream_t st);

// ---------------------------------------------------------------- others
cudaError_t launch_fuse(int dtype, const void* states, int64_t N, int T, int H,
                        int D, const float* w_fuse, const float* const* g_fuse,
                        void* fused, float eps, cudaStream_t st);
// Largest hidden size the fusion kernel covers for T target layers.
int fuse_hidden_limit(int dtype, int nT);
cudaError_t launch_embed(int dtype, const void* embed, int H, int nb, int B,
                         const int32_t* block_tokens, const int32_t* known_len,
                         int mask_id, float* h, cudaStream_t st);
cudaError_t launch_rmsnorm(int dtype, const float* h, int64_t M, int H,
                           const float* g, float eps, void* x, cudaStream_t st);
cudaError_t launch_prep_rows(int R, int nb, int B, const int32_t* block_req,
                             const int64_t* ctx_off, const int64_t* new_off,
                             const int32_t* ctx_cached, int64_t n_new,
                             int32_t* blk_pos, int32_t* new_pos,
                             int64_t* new_dst, cudaStream_t st);
cudaError_t launch_argmax_finish(const unsigned long long* keys, int64_t M,
                                 int B, const int32_t* block_tokens,
                                 const int32_t* known_len, int32_t* tok,
                                 float* max_logit, cudaStream_t st);

struct AttnPlan {
  int splits;
  int chunk;        // context keys per split (multiple of 64)
  int row_chunks;   // CTAs along the query rows of one (block, kv head)
  int rows_per_cta;
};
AttnPlan plan_attn(int dtype, int nb, int B, int Hq, int Hkv, int d,
                   int64_t max_ctx_len);
size_t attn_ws_bytes(const AttnPlan& p, int nb, int B, int Hq, int d);
cudaError_t launch_attn(int dtype, const AttnPlan& plan, int nb, int B, int Hq,
                        int Hkv, int d, const void* q, const void* kb,
                        const void* vb, const void* kc, const void* vc,
                        const int64_t* ctx_off, const int32_t* block_req,
                        void* out, float* ws, uint32_t* status,
                        cudaStream_t st);

cudaError_t launch_accept(int R, int K, int B, const int32_t* draft,
                          const int32_t* target, int32_t* n_acc,
                          int32_t* best_k, int32_t* out_tok, cudaStream_t st);
cudaError_t launch_d2sd(int R, int B, int K, int mask_id, const int32_t* base,
                        const float* conf, int32_t* known_len, int32_t* cand,
                        int32_t* block_req, cudaStream_t st);
cudaError_t launch_wait_selftest(uint32_t* status, int64_t limit_ns,
                                 cudaStream_t st);

// Tensor maps (driver entry point fetched through the runtime).
bool encode_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner,
                         uint64_t outer, uint32_t box_inner, uint32_t box_outer);

}  // namespace dfl
