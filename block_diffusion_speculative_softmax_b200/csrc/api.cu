// C ABI of libdflash.so: argument validation, workspace layout and the
// kernel sequence of one draft step.  No entry point allocates memory.
#include <atomic>
#include <cstdlib>
#include <mutex>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <string>

#include "common.cuh"
#include "internal.h"

namespace dfl {

static std::atomic<uint64_t> g_launches{0};
void count_launch(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }

namespace {

thread_local std::string t_err;

dflash_status fail(dflash_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  t_err = buf;
  return s;
}

dflash_status cuda_fail(cudaError_t e, const char* what) {
  return fail(DFLASH_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define DFL_CUDA(call, what)                          \
  do {                                                \
    cudaError_t e_ = (call);                          \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

#define DFL_CHECK(cond, status, ...)                 \
  do {                                               \
    if (!(cond)) return fail(status, __VA_ARGS__);   \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
size_t esize(const dflash_config* c) { return c->dtype == DFLASH_BF16 ? 2 : 4; }

dflash_status check_config(const dflash_config* c) {
  DFL_CHECK(c != nullptr, DFLASH_EINVAL, "config is NULL");
  DFL_CHECK(c->dtype == DFLASH_FP32 || c->dtype == DFLASH_BF16, DFLASH_EINVAL,
            "dtype must be DFLASH_FP32 (0) or DFLASH_BF16 (1), got %d", c->dtype);
  const int mult = c->dtype == DFLASH_BF16 ? 8 : 4;
  DFL_CHECK(c->hidden > 0 && c->hidden % mult == 0, DFLASH_EINVAL,
            "hidden must be a positive multiple of %d, got %d", mult, c->hidden);
  DFL_CHECK(c->ffn > 0 && c->ffn % mult == 0, DFLASH_EINVAL,
            "ffn must be a positive multiple of %d, got %d", mult, c->ffn);
  DFL_CHECK(c->n_q_heads > 0 && c->n_kv_heads > 0 && c->n_q_heads % c->n_kv_heads == 0,
            DFLASH_EINVAL, "n_q_heads (%d) must be a positive multiple of n_kv_heads (%d)",
            c->n_q_heads, c->n_kv_heads);
  DFL_CHECK(c->head_dim == 64 || c->head_dim == 128, DFLASH_EUNSUPPORTED,
            "head_dim must be 64 or 128, got %d", c->head_dim);
  DFL_CHECK(c->n_draft_layers >= 1 && c->n_draft_layers <= kMaxLayers, DFLASH_EINVAL,
            "n_draft_layers must be in [1, %d], got %d", kMaxLayers, c->n_draft_layers);
  DFL_CHECK(c->n_target_layers >= 1 && c->n_target_layers <= kMaxTargetLayers, DFLASH_EINVAL,
            "n_target_layers must be in [1, %d], got %d", kMaxTargetLayers, c->n_target_layers);
  DFL_CHECK(c->block >= 1 && c->block <= kMaxBlock, DFLASH_EINVAL,
            "block must be in [1, %d], got %d", kMaxBlock, c->block);
  DFL_CHECK(c->vocab >= 2, DFLASH_EINVAL, "vocab must be >= 2, got %d", c->vocab);
  DFL_CHECK(c->mask_token_id >= 0 && c->mask_token_id < c->vocab, DFLASH_EINVAL,
            "mask_token_id %d outside [0, vocab)", c->mask_token_id);
  DFL_CHECK(std::isfinite(c->rope_theta) && c->rope_theta > 0.f, DFLASH_EINVAL,
            "rope_theta must be positive");
  DFL_CHECK(std::isfinite(c->rms_eps) && c->rms_eps >= 0.f, DFLASH_EINVAL,
            "rms_eps must be >= 0");
  DFL_CHECK(c->hidden <= fuse_hidden_limit(c->dtype, c->n_target_layers), DFLASH_EUNSUPPORTED,
            "hidden %d too large for the fusion kernel with T=%d (max %d)", c->hidden,
            c->n_target_layers, fuse_hidden_limit(c->dtype, c->n_target_layers));
  return DFLASH_OK;
}

#define DFL_PTR(p, name)                                                         \
  do {                                                                           \
    if ((p) == nullptr) return fail(DFLASH_EINVAL, "%s is NULL", name);          \
    if (!aligned16(p)) return fail(DFLASH_EINVAL, "%s is not 16-byte aligned", name); \
  } while (0)

// Index and per-token arrays (int32 / fp32 / int64, nullable): naturally
// aligned, so a misaligned pointer is refused on the host and never reaches
// a kernel.
#define DFL_ALIGNED(p, n, name)                                                  \
  do {                                                                           \
    if ((p) != nullptr && (reinterpret_cast<uintptr_t>(p) % (n)) != 0)           \
      return fail(DFLASH_EINVAL, "%s is not %d-byte aligned", name, n);          \
  } while (0)

// ------------------------------------------------------------------ jobs
GemmJob job_base(const dflash_config* c, const void* x, int64_t M, int K) {
  GemmJob j;
  j.x = x;
  j.M = M;
  j.K = K;
  j.dtype = c->dtype;
  j.head_dim = c->head_dim;
  j.theta = c->rope_theta;
  return j;
}

// K/V projection of context rows (W^t) or block rows (W^d): K with RoPE.
GemmJob job_kv(const dflash_config* c, const void* x, int64_t M, const int32_t* pos,
               const int64_t* dst, const void* wk, const void* wv, void* k_out, void* v_out) {
  const int kvd = c->n_kv_heads * c->head_dim;
  GemmJob j = job_base(c, x, M, c->hidden);
  j.nseg = 2;
  j.seg[0] = {wk, nullptr, kvd, EPI_STORE, 1, k_out, kvd, dst != nullptr};
  j.seg[1] = {wv, nullptr, kvd, EPI_STORE, 0, v_out, kvd, dst != nullptr};
  j.pos = pos;
  j.dst = dst;
  return j;
}

GemmJob job_qkv(const dflash_config* c, const dflash_layer_weights& l, const void* x, int64_t M,
                const int32_t* pos, void* q, void* kb, void* vb) {
  const int qd = c->n_q_heads * c->head_dim, kvd = c->n_kv_heads * c->head_dim;
  GemmJob j = job_base(c, x, M, c->hidden);
  j.nseg = 3;
  j.seg[0] = {l.w_q, nullptr, qd, EPI_STORE, 1, q, qd, 0};
  j.seg[1] = {l.w_kd, nullptr, kvd, EPI_STORE, 1, kb, kvd, 0};
  j.seg[2] = {l.w_vd, nullptr, kvd, EPI_STORE, 0, vb, kvd, 0};
  j.pos = pos;
  return j;
}

GemmJob job_resid(const dflash_config* c, const void* w, const void* x, int64_t M, int K,
                  float* h) {
  GemmJob j = job_base(c, x, M, K);
  j.nseg = 1;
  j.seg[0] = {w, nullptr, c->hidden, EPI_RESID, 0, h, c->hidden, 0};
  return j;
}

// DFlash FC fusion: fp32 u = states[N][T*H] W_fc^T (RMSNorm follows).
GemmJob job_fc(const dflash_config* c, const void* states, int64_t N, const void* w_fc,
               float* u) {
  GemmJob j = job_base(c, states, N, c->n_target_layers * c->hidden);
  j.nseg = 1;
  j.seg[0] = {w_fc, nullptr, c->hidden, EPI_STORE_F32, 0, u, c->hidden, 0};
  return j;
}

// LM head writing fp32 logits [M][V] (temperature-1 mode).
GemmJob job_logits(const dflash_config* c, const void* x, int64_t M, const void* w_lm,
                   float* logits) {
  GemmJob j = job_base(c, x, M, c->hidden);
  j.nseg = 1;
  j.seg[0] = {w_lm, nullptr, c->vocab, EPI_STORE_F32, 0, logits, c->vocab, 0};
  return j;
}

GemmJob job_swiglu(const dflash_config* c, const void* wg, const void* wu, const void* x,
                   int64_t M, void* act) {
  GemmJob j = job_base(c, x, M, c->hidden);
  j.nseg = 1;
  j.seg[0] = {wg, wu, c->ffn, EPI_SWIGLU, 0, act, c->ffn, 0};
  return j;
}

// ------------------------------------------------------------------ layout
struct Layout {
  size_t h = 0, x = 0, q = 0, kb = 0, vb = 0, attn = 0, act = 0, fused = 0, partial = 0,
         attn_ws = 0, zero = 0, keys = 0, counters = 0, blk_pos = 0, new_pos = 0, new_dst = 0,
         rope = 0, partial_side = 0, counters_side = 0, lse = 0, row_lse = 0, rss = 0, total = 0;
  int rope_len = 0;
  size_t zero_bytes = 0;   // [keys | counters], zeroed at the start of a step
};

struct Needs {
  size_t partial_floats = 0;
  size_t counters = 0;
  void take(const GemmPlan& p) {
    partial_floats = std::max(partial_floats, p.partial_floats);
    counters = std::max(counters, p.counters);
  }
};

// Scratch of the GEMMs of one step.  A workspace sized for (M, n_new) must
// also serve every smaller call (a D2SD first pass drafts fewer blocks than
// its second, a steady step fuses fewer rows), and smaller token counts can
// need MORE split-K scratch, so every smaller block count and a dense sample
// of smaller row counts are planned too.
Needs step_needs(const dflash_config* c, int64_t M, int64_t n_new) {
  Needs n;
  dflash_layer_weights l{};
  auto ctx_rows = [&](int64_t r) {
    n.take(plan_gemm(job_kv(c, nullptr, r, nullptr, nullptr, 0, 0, 0, 0)));
    n.take(plan_gemm(job_fc(c, nullptr, r, nullptr, nullptr)));
  };
  if (n_new > 0) {
    ctx_rows(n_new);
    for (int64_t r = 1; r < n_new && r <= 4096; r += (r < 128 ? 1 : 64)) ctx_rows(r);
  }
  for (int64_t m = std::min<int64_t>(M, c->block); m > 0 && m <= M;
       m = (m == M) ? M + 1 : std::min<int64_t>(M, m + c->block)) {
    n.take(plan_gemm(job_kv(c, nullptr, m, nullptr, nullptr, 0, 0, 0, 0)));
    n.take(plan_gemm(job_qkv(c, l, nullptr, m, nullptr, 0, 0, 0)));
    n.take(plan_gemm(job_resid(c, nullptr, nullptr, m, c->n_q_heads * c->head_dim, 0)));
    n.take(plan_gemm(job_swiglu(c, nullptr, nullptr, nullptr, m, 0)));
    n.take(plan_gemm(job_resid(c, nullptr, nullptr, m, c->ffn, 0)));
    n.take(plan_lmhead(c->dtype, c->vocab, m, c->hidden));
    n.take(plan_gemm(job_logits(c, nullptr, m, nullptr, nullptr)));
  }
  return n;
}

Layout make_layout(const dflash_config* c, int32_t n_req, int32_t nb, int64_t n_new,
                   int64_t max_ctx) {
  (void)n_req;
  Layout L;
  const size_t e = esize(c);
  const int64_t M = static_cast<int64_t>(nb) * c->block;
  const size_t H = c->hidden, F = c->ffn, qd = static_cast<size_t>(c->n_q_heads) * c->head_dim,
               kvd = static_cast<size_t>(c->n_kv_heads) * c->head_dim;
  size_t off = sizeof(DevStatus);
  auto take = [&](size_t bytes) {
    size_t at = off;
    off = align256(off + bytes);
    return at;
  };
  const Needs nd = step_needs(c, M, n_new);
  AttnPlan ap = plan_attn(c->dtype, nb, c->block, c->n_q_heads, c->n_kv_heads, c->head_dim,
                          max_ctx);
  L.h = take(M * H * 4);
  L.x = take(M * std::max(H, F) * e);
  L.q = take(M * qd * e);
  L.kb = take(M * kvd * e);
  L.vb = take(M * kvd * e);
  L.attn = take(M * qd * e);
  L.act = take(M * F * e);
  // per-layer fused contexts [D][N][H]; the FC variant keeps one [N][H]
  // context behind its fp32 product [N][H] in the same region
  L.fused = take(std::max(static_cast<size_t>(c->n_draft_layers) * e, 4 + e) * n_new * H);
  L.partial = take(nd.partial_floats * 4);
  // fewer blocks can mean more splits (and more partials): size for all
  size_t attn_bytes = 0;
  for (int b = 1; b <= nb; ++b)
    attn_bytes = std::max(
        attn_bytes, attn_ws_bytes(plan_attn(c->dtype, b, c->block, c->n_q_heads, c->n_kv_heads,
                                            c->head_dim, max_ctx),
                                  b, c->block, c->n_q_heads, c->head_dim));
  (void)ap;
  L.attn_ws = take(attn_bytes);
  const size_t ncount = nd.counters;
  // the context branch runs on a second stream: its own split-K scratch
  Needs side;
  if (n_new > 0) {
    side.take(plan_gemm(job_kv(c, nullptr, n_new, nullptr, nullptr, 0, 0, 0, 0)));
    side.take(plan_gemm(job_fc(c, nullptr, n_new, nullptr, nullptr)));
  }
  L.partial_side = take(side.partial_floats * 4);
  L.zero = off;
  L.keys = take(M * 8);
  L.counters = take(ncount * 4);
  L.counters_side = take(side.counters * 4);
  L.zero_bytes = off - L.zero;
  L.blk_pos = take(M * 4);
  L.new_pos = take(n_new * 4);
  L.new_dst = take(n_new * 8);
  // (fewer tokens can mean more, narrower vocabulary tiles: size for both)
  const int64_t Ms = std::min<int64_t>(M, 64);
  L.lse = take(std::max(static_cast<size_t>(lmhead_tiles(c->dtype, c->vocab, M)) * M,
                        static_cast<size_t>(lmhead_tiles(c->dtype, c->vocab, Ms)) * Ms) * 8);
  L.row_lse = take(M * 4);   // temperature-1 mode: logsumexp of each logit row
  // per (draft layer, new row) partial sums of squares of the unnormalised
  // bf16 fusion
  L.rss = take(static_cast<size_t>(c->n_draft_layers) * n_new * fuse_unnorm_parts(c->hidden) * 4);
  L.rope_len = static_cast<int>(max_ctx + c->block);
  L.rope = take(static_cast<size_t>(L.rope_len) * (c->head_dim / 2) * 8);
  L.total = off;
  return L;
}

template <typename P>
P* at(void* ws, size_t off) {
  return reinterpret_cast<P*>(static_cast<uint8_t*>(ws) + off);
}
uint32_t* status_word(void* ws) { return static_cast<uint32_t*>(ws); }

dflash_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  DFL_CHECK(ws != nullptr, DFLASH_EINVAL, "workspace is NULL");
  DFL_CHECK((reinterpret_cast<uintptr_t>(ws) & 255u) == 0, DFLASH_EINVAL,
            "workspace must be 256-byte aligned");
  DFL_CHECK(ws_bytes >= need, DFLASH_EINVAL, "workspace too small: %zu bytes, need %zu",
            ws_bytes, need);
  return DFLASH_OK;
}

// A second stream (per host thread and device) for the context branch of a
// draft step: fusion and the context K/V projections of every layer depend
// only on the new context rows, not on the block path, so they run beside
// the weight-streaming block GEMMs; layer i's attention waits for its
// context K/V through an event.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr;
  cudaEvent_t done[kMaxLayers] = {};
};
constexpr int kSideDevices = 16;
thread_local SideStream t_side[kSideDevices];

dflash_status side_stream(SideStream** out) {
  *out = nullptr;
  int dev = 0;
  DFL_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  if (dev < 0 || dev >= kSideDevices) return DFLASH_OK;   // run the branch in order instead
  SideStream& r = t_side[dev];
  if (r.stream == nullptr) {
    DFL_CUDA(cudaStreamCreateWithFlags(&r.stream, cudaStreamNonBlocking), "side stream");
    DFL_CUDA(cudaEventCreateWithFlags(&r.fork, cudaEventDisableTiming), "side event");
    for (int i = 0; i < kMaxLayers; ++i)
      DFL_CUDA(cudaEventCreateWithFlags(&r.done[i], cudaEventDisableTiming), "side event");
  }
  *out = &r;
  return DFLASH_OK;
}

dflash_status run_job(const GemmJob& j, float* partial, uint32_t* counters, uint32_t* status,
                      cudaStream_t st, const char* what) {
  const GemmPlan pl = plan_gemm(j);
  DFL_CUDA(launch_gemm(j, pl, partial, counters, status, st), what);
  return DFLASH_OK;
}

}  // namespace
}  // namespace dfl

using namespace dfl;

extern "C" {

const char* dflash_version(void) { return "dflash-b200 0.1 (sm_100a)"; }

const char* dflash_last_error(void) { return t_err.c_str(); }

uint64_t dflash_launch_count(void) { return g_launches.load(); }

size_t dflash_workspace_size(const dflash_config* cfg, int32_t n_req, int32_t n_blocks,
                             int64_t n_ctx_new, int64_t max_ctx_len) {
  if (check_config(cfg) != DFLASH_OK || n_req < 0 || n_blocks < 0 || n_ctx_new < 0 ||
      max_ctx_len < 0)
    return 0;
  return make_layout(cfg, n_req, n_blocks, n_ctx_new, max_ctx_len).total;
}

dflash_status dflash_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  DFL_CHECK(ws != nullptr, DFLASH_EINVAL, "workspace is NULL");
  DFL_CHECK(ws_bytes >= sizeof(DevStatus), DFLASH_EINVAL, "workspace smaller than its header");
  DFL_CUDA(cudaMemsetAsync(ws, 0, sizeof(DevStatus), static_cast<cudaStream_t>(stream)),
           "workspace init");
  return DFLASH_OK;
}

dflash_status dflash_check(void* ws, void* stream) {
  DFL_CHECK(ws != nullptr, DFLASH_EINVAL, "workspace is NULL");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DFL_CUDA(cudaStreamSynchronize(st), "stream synchronize");
  uint32_t hdr[2] = {0, 0};
  DFL_CUDA(cudaMemcpy(hdr, ws, sizeof(hdr), cudaMemcpyDeviceToHost), "read status");
  if (hdr[0] != 0) {
    DFL_CUDA(cudaMemset(ws, 0, sizeof(hdr)), "clear status");
    const char* what = hdr[0] == DFLASH_ETIMEOUT ? "a bounded device wait ran out"
                       : hdr[0] == DFLASH_ENUMERIC ? "non-finite logit"
                       : hdr[0] == DFLASH_EBOUNDS  ? "device index out of its buffer"
                                                   : "device error";
    return fail(static_cast<dflash_status>(hdr[0]), "%s (kernel tag %u)", what, hdr[1]);
  }
  return DFLASH_OK;
}

dflash_status dflash_fuse_ctx(const dflash_config* cfg, const void* states, int64_t n_rows,
                              const float* w_fuse, const float* const* g_fuse, void* fused,
                              void* stream) {
  dflash_status s = check_config(cfg);
  if (s != DFLASH_OK) return s;
  DFL_CHECK(n_rows >= 0, DFLASH_EINVAL, "n_rows must be >= 0");
  if (n_rows == 0) return DFLASH_OK;
  DFL_PTR(states, "states");
  DFL_PTR(fused, "fused");
  DFL_CHECK(w_fuse != nullptr, DFLASH_EINVAL, "w_fuse is NULL");
  DFL_CHECK(g_fuse != nullptr, DFLASH_EINVAL, "g_fuse is NULL");
  for (int i = 0; i < cfg->n_draft_layers; ++i) DFL_PTR(g_fuse[i], "g_fuse[i]");
  DFL_CUDA(launch_fuse(cfg->dtype, states, n_rows, cfg->n_target_layers, cfg->hidden,
                       cfg->n_draft_layers, w_fuse, g_fuse, fused, cfg->rms_eps, nullptr,
                       static_cast<cudaStream_t>(stream)),
           "fusion kernel");
  return DFLASH_OK;
}

int32_t dflash_fuse_rss_parts(int32_t hidden) { return hidden > 0 ? fuse_unnorm_parts(hidden) : 0; }

dflash_status dflash_fuse_ctx_rss(const dflash_config* cfg, const void* states, int64_t n_rows,
                                  const float* w_fuse, const float* const* g_fuse, void* fused,
                                  float* rss, void* ws, size_t ws_bytes, void* stream) {
  dflash_status s = check_config(cfg);
  if (s != DFLASH_OK) return s;
  DFL_CHECK(cfg->dtype == DFLASH_BF16, DFLASH_EUNSUPPORTED, "the split fusion is bf16 only");
  DFL_CHECK(n_rows >= 0, DFLASH_EINVAL, "n_rows must be >= 0");
  if ((s = check_ws(ws, ws_bytes, sizeof(DevStatus))) != DFLASH_OK) return s;
  if (n_rows == 0) return DFLASH_OK;
  DFL_PTR(states, "states");
  DFL_PTR(fused, "fused");
  DFL_CHECK(rss != nullptr, DFLASH_EINVAL, "rss is NULL");
  DFL_ALIGNED(rss, 4, "rss");
  DFL_CHECK(w_fuse != nullptr, DFLASH_EINVAL, "w_fuse is NULL");
  DFL_CHECK(g_fuse != nullptr, DFLASH_EINVAL, "g_fuse is NULL");
  for (int i = 0; i < cfg->n_draft_layers; ++i) DFL_PTR(g_fuse[i], "g_fuse[i]");
  DFL_CUDA(launch_fuse_unnorm(states, n_rows, cfg->n_target_layers, cfg->hidden,
                              cfg->n_draft_layers, w_fuse, g_fuse, fused, rss, status_word(ws),
                              static_cast<cudaStream_t>(stream)),
           "fusion kernel");
  return DFLASH_OK;
}

dflash_status dflash_fc_fuse_ctx(const dflash_config* cfg, const void* states, int64_t n_rows,
                                 const void* w_fc, const float* g_fc, void* fused, void* ws,
                                 size_t ws_bytes, void* stream) {
  dflash_status s = check_config(cfg);
  if (s != DFLASH_OK) return s;
  DFL_CHECK(n_rows >= 0 && n_rows < (int64_t(1) << 31), DFLASH_EINVAL, "n_rows out of range");
  if (n_rows == 0) return DFLASH_OK;
  DFL_PTR(states, "states");
  DFL_PTR(w_fc, "w_fc");
  DFL_PTR(g_fc, "g_fc");
  DFL_PTR(fused, "fused");
  const int H = cfg->hidden;
  const size_t off_u = sizeof(DevStatus);
  const GemmJob j = job_fc(cfg, states, n_rows, w_fc, at<float>(ws, off_u));
  const GemmPlan pl = plan_gemm(j);
  const size_t off_part = align256(off_u + static_cast<size_t>(n_rows) * H * 4);
  const size_t off_cnt = align256(off_part + pl.partial_floats * 4);
  const size_t need = off_cnt + pl.counters * 4;
  if ((s = check_ws(ws, ws_bytes, need)) != DFLASH_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DFL_CUDA(launch_zero(at<void>(ws, off_cnt), pl.counters * 4, st), "counter reset");
  DFL_CUDA(launch_gemm(j, pl, at<float>(ws, off_part), at<uint32_t>(ws, off_cnt),
                       status_word(ws), st),
           "FC fusion GEMM");
  DFL_CUDA(launch_rmsnorm(cfg->dtype, at<float>(ws, off_u), n_rows, H, g_fc, cfg->rms_eps, fused,
                          st),
           "FC fusion rmsnorm");
  return DFLASH_OK;
}

dflash_status dflash_kv_project(const dflash_config* cfg, const void* x, int64_t M,
                                const int32_t* pos, const int64_t* dst_row, const void* w_k,
                                const void* w_v, void* k_out, void* v_out, void* ws,
                                size_t ws_bytes, void* stream) {
  dflash_status s = check_config(cfg);
  if (s != DFLASH_OK) return s;
  DFL_CHECK(M >= 0 && M < (int64_t(1) << 31), DFLASH_EINVAL, "M out of range");
  if (M == 0) return DFLASH_OK;
  DFL_PTR(x, "x");
  DFL_PTR(w_k, "w_k");
  DFL_PTR(w_v, "w_v");
  DFL_PTR(k_out, "k_out");
  DFL_PTR(v_out, "v_out");
  DFL_CHECK(pos != nullptr, DFLASH_EINVAL, "pos is NULL");
  DFL_ALIGNED(pos, 4, "pos");
  DFL_ALIGNED(dst_row, 8, "dst_row");
  const GemmJob j = job_kv(cfg, x, M, pos, dst_row, w_k, w_v, k_out, v_out);
  const GemmPlan pl = plan_gemm(j);
  const size_t off_cnt = align256(sizeof(DevStatus) + pl.partial_floats * 4);
  const size_t need = off_cnt + pl.counters * 4;
  if ((s = check_ws(ws, ws_bytes, need)) != DFLASH_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DFL_CUDA(launch_zero(at<void>(ws, off_cnt), pl.counters * 4, st), "counter reset");
  DFL_CUDA(launch_gemm(j, pl, at<float>(ws, sizeof(DevStatus)), at<uint32_t>(ws, off_cnt),
                       status_word(ws), st),
           "kv projection GEMM");
  return DFLASH_OK;
}

dflash_status dflash_block_attn(const dflash_config* cfg, int32_t n_blocks, const void* q,
                                const void* k_blk, const void* v_blk, const void* k_ctx,
                                const void* v_ctx, const int64_t* ctx_off,
                                const int32_t* block_req, int64_t max_ctx_len, void* out,
                                void* ws, size_t ws_bytes, void* stream) {
  dflash_status s = check_config(cfg);
  if (s != DFLASH_OK) return s;
  DFL_CHECK(n_blocks >= 0 && max_ctx_len >= 0, DFLASH_EINVAL, "negative size");
  if (n_blocks == 0) return DFLASH_OK;
  DFL_PTR(q, "q");
  DFL_PTR(k_blk, "k_blk");
  DFL_PTR(v_blk, "v_blk");
  DFL_PTR(out, "out");
  DFL_CHECK(ctx_off != nullptr && block_req != nullptr, DFLASH_EINVAL,
            "ctx_off / block_req is NULL");
  DFL_ALIGNED(ctx_off, 8, "ctx_off");
  DFL_ALIGNED(block_req, 4, "block_req");
  if (max_ctx_len > 0) {
    DFL_PTR(k_ctx, "k_ctx");
    DFL_PTR(v_ctx, "v_ctx");
  }
  AttnPlan ap = plan_attn(cfg->dtype, n_blocks, cfg->block, cfg->n_q_heads, cfg->n_kv_heads,
                          cfg->head_dim, max_ctx_len);
  const size_t need =
      sizeof(DevStatus) + attn_ws_bytes(ap, n_blocks, cfg->block, cfg->n_q_heads, cfg->head_dim);
  if ((s = check_ws(ws, ws_bytes, need)) != DFLASH_OK) return s;
  DFL_CUDA(launch_attn(cfg->dtype, ap, n_blocks, cfg->block, cfg->n_q_heads, cfg->n_kv_heads,
                       cfg->head_dim, q, k_blk, v_blk, k_ctx, v_ctx, ctx_off, block_req, out,
                       at<float>(ws, sizeof(DevStatus)), status_word(ws),
                       static_cast<cudaStream_t>(stream)),
           "attention kernel");
  return DFLASH_OK;
}

dflash_status dflash_mlp(const dflash_config* cfg, int64_t M, float* h, const float* g_mlp,
                         const void* w_gate, const void* w_up, const void* w_down, void* ws,
                         size_t ws_bytes, void* stream) {
  dflash_status s = check_config(cfg);
  if (s != DFLASH_OK) return s;
  DFL_CHECK(M >= 0 && M < (int64_t(1) << 31), DFLASH_EINVAL, "M out of range");
  if (M == 0) return DFLASH_OK;
  DFL_PTR(h, "h");
  DFL_PTR(g_mlp, "g_mlp");
  DFL_PTR(w_gate, "w_gate");
  DFL_PTR(w_up, "w_up");
  DFL_PTR(w_down, "w_down");
  const size_t e = esize(cfg);
  const int H = cfg->hidden, F = cfg->ffn;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t off_x = sizeof(DevStatus);
  const size_t off_act = align256(off_x + M * H * e);
  const GemmJob j1 = job_swiglu(cfg, w_gate, w_up, at<void>(ws, off_x), M, at<void>(ws, off_act));
  const GemmJob j2 = job_resid(cfg, w_down, at<void>(ws, off_act), M, F, h);
  const GemmPlan p1 = plan_gemm(j1), p2 = plan_gemm(j2);
  const size_t off_part = align256(off_act + M * F * e);
  const size_t off_cnt =
      align256(off_part + std::max(p1.partial_floats, p2.partial_floats) * 4);
  const size_t ncnt = std::max(p1.counters, p2.counters);
  if ((s = check_ws(ws, ws_bytes, off_cnt + ncnt * 4)) != DFLASH_OK) return s;
  float* part = at<float>(ws, off_part);
  uint32_t* cnt = at<uint32_t>(ws, off_cnt);
  DFL_CUDA(launch_zero(cnt, ncnt * 4, st), "counter reset");
  DFL_CUDA(launch_rmsnorm(cfg->dtype, h, M, H, g_mlp, cfg->rms_eps, at<void>(ws, off_x), st),
           "mlp rmsnorm");
  DFL_CUDA(launch_gemm(j1, p1, part, cnt, status_word(ws), st), "gate/up GEMM");
  DFL_CUDA(launch_gemm(j2, p2, part, cnt, status_word(ws), st), "down GEMM");
  return DFLASH_OK;
}

dflash_status dflash_lmhead_argmax(const dflash_config* cfg, int64_t M, const void* x,
                                   const void* w_lm, int32_t* tok, float* max_logit, float* conf,
                                   void* ws, size_t ws_bytes, void* stream) {
  dflash_status s = check_config(cfg);
  if (s != DFLASH_OK) return s;
  DFL_CHECK(M >= 0 && M < (int64_t(1) << 31), DFLASH_EINVAL, "M out of range");
  if (M == 0) return DFLASH_OK;
  DFL_PTR(x, "x");
  DFL_PTR(w_lm, "w_lm");
  DFL_CHECK(tok != nullptr, DFLASH_EINVAL, "tok is NULL");
  DFL_ALIGNED(tok, 4, "tok");
  DFL_ALIGNED(max_logit, 4, "max_logit");
  DFL_ALIGNED(conf, 4, "conf");
  const GemmPlan pl = plan_lmhead(cfg->dtype, cfg->vocab, M, cfg->hidden);
  const size_t off_keys = sizeof(DevStatus);
  const size_t off_cnt = align256(off_keys + M * 8);
  const size_t off_part = align256(off_cnt + pl.counters * 4);
  const int lt = lmhead_tiles(cfg->dtype, cfg->vocab, M);
  const size_t off_lse = align256(off_part + pl.partial_floats * 4);
  const size_t need = off_lse + (conf ? static_cast<size_t>(lt) * M * 8 : 0);
  if ((s = check_ws(ws, ws_bytes, need)) != DFLASH_OK) return s;
  float2* lse = conf ? at<float2>(ws, off_lse) : nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  auto* keys = at<unsigned long long>(ws, off_keys);
  // keys and tile counters start at zero
  DFL_CUDA(launch_zero(keys, off_part - off_keys, st), "argmax key reset");
  DFL_CUDA(launch_lmhead_argmax(cfg->dtype, w_lm, cfg->vocab, x, M, cfg->hidden, keys,
                                status_word(ws), st,
                                pl.stream_k ? at<float>(ws, off_part) : nullptr,
                                pl.stream_k ? at<uint32_t>(ws, off_cnt) : nullptr, lse),
           "LM head argmax");
  DFL_CUDA(launch_argmax_finish(keys, M, cfg->block, nullptr, nullptr, tok, max_logit, st, lse,
                                lt, conf),
           "argmax finish");
  return DFLASH_OK;
}

dflash_status dflash_lmhead_logits(const dflash_config* cfg, int64_t M, const void* x,
                                   const void* w_lm, float* logits, void* ws, size_t ws_bytes,
                                   void* stream) {
  dflash_status s = check_config(cfg);
  if (s != DFLASH_OK) return s;
  DFL_CHECK(M >= 0 && M < (int64_t(1) << 31), DFLASH_EINVAL, "M out of range");
  if (M == 0) return DFLASH_OK;
  DFL_PTR(x, "x");
  DFL_PTR(w_lm, "w_lm");
  DFL_PTR(logits, "logits");
  const GemmJob j = job_logits(cfg, x, M, w_lm, logits);
  const GemmPlan pl = plan_gemm(j);
  const size_t off_part = sizeof(DevStatus);
  const size_t off_cnt = align256(off_part + pl.partial_floats * 4);
  if ((s = check_ws(ws, ws_bytes, off_cnt + pl.counters * 4)) != DFLASH_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DFL_CUDA(launch_zero(at<void>(ws, off_cnt), pl.counters * 4, st), "counter reset");
  DFL_CUDA(launch_gemm(j, pl, at<float>(ws, off_part), at<uint32_t>(ws, off_cnt),
                       status_word(ws), st),
           "LM head logits GEMM");
  return DFLASH_OK;
}

dflash_status dflash_sample(const dflash_config* cfg, int64_t M, const float* logits,
                            uint64_t seed, uint32_t offset, int32_t* tok, float* logq, float* lse,
                            void* stream) {
  dflash_status s = check_config(cfg);
  if (s != DFLASH_OK) return s;
  DFL_CHECK(M >= 0 && M < (int64_t(1) << 31), DFLASH_EINVAL, "M out of range");
  if (M == 0) return DFLASH_OK;
  DFL_CHECK(logits != nullptr && tok != nullptr, DFLASH_EINVAL, "logits / tok is NULL");
  DFL_ALIGNED(logits, 4, "logits");
  DFL_ALIGNED(tok, 4, "tok");
  DFL_ALIGNED(logq, 4, "logq");
  DFL_ALIGNED(lse, 4, "lse");
  DFL_CUDA(launch_sample_rows(logits, M, cfg->vocab, seed, offset, cfg->block, nullptr, nullptr,
                              tok, logq, lse, nullptr, static_cast<cudaStream_t>(stream)),
           "sampling kernel");
  return DFLASH_OK;
}

dflash_status dflash_accept_stochastic(int32_t R, int32_t B, int32_t V, const int32_t* draft,
                                       const float* draft_logits, const float* draft_lse,
                                       const float* target_logp, uint64_t seed, uint32_t offset,
                                       int32_t* n_acc, int32_t* out_tok, void* ws,
                                       size_t ws_bytes, void* stream) {
  DFL_CHECK(R >= 0, DFLASH_EINVAL, "R must be >= 0");
  DFL_CHECK(B >= 1 && B <= kMaxBlock, DFLASH_EINVAL, "B must be in [1, %d], got %d", kMaxBlock, B);
  DFL_CHECK(V >= 2, DFLASH_EINVAL, "V must be >= 2, got %d", V);
  if (R == 0) return DFLASH_OK;
  DFL_CHECK(R < (1 << 26), DFLASH_EINVAL, "R too large for the random-number counters");
  DFL_CHECK(draft && draft_logits && draft_lse && target_logp && n_acc && out_tok, DFLASH_EINVAL,
            "a pointer argument is NULL");
  DFL_ALIGNED(draft, 4, "draft");
  DFL_ALIGNED(draft_logits, 4, "draft_logits");
  DFL_ALIGNED(draft_lse, 4, "draft_lse");
  DFL_ALIGNED(target_logp, 4, "target_logp");
  DFL_ALIGNED(n_acc, 4, "n_acc");
  DFL_ALIGNED(out_tok, 4, "out_tok");
  dflash_status s = check_ws(ws, ws_bytes, sizeof(DevStatus) + static_cast<size_t>(R) * 8);
  if (s != DFLASH_OK) return s;
  DFL_CUDA(launch_accept_stochastic(R, B, V, draft, draft_logits, draft_lse, target_logp, seed,
                                    offset, n_acc, out_tok,
                                    at<unsigned long long>(ws, sizeof(DevStatus)),
                                    status_word(ws), static_cast<cudaStream_t>(stream)),
           "stochastic accept");
  return DFLASH_OK;
}

dflash_status dflash_accept(int32_t R, int32_t K, int32_t B, const int32_t* draft,
                            const int32_t* target, int32_t* n_acc, int32_t* best_k,
                            int32_t* out_tok, void* stream) {
  DFL_CHECK(R >= 0, DFLASH_EINVAL, "R must be >= 0");
  DFL_CHECK(K >= 1 && K <= 32, DFLASH_EINVAL, "K must be in [1, 32], got %d", K);
  DFL_CHECK(B >= 1 && B <= kMaxBlock, DFLASH_EINVAL, "B must be in [1, %d], got %d", kMaxBlock, B);
  if (R == 0) return DFLASH_OK;
  DFL_CHECK(draft && target && n_acc && best_k && out_tok, DFLASH_EINVAL,
            "a pointer argument is NULL");
  DFL_ALIGNED(draft, 4, "draft");
  DFL_ALIGNED(target, 4, "target");
  DFL_ALIGNED(n_acc, 4, "n_acc");
  DFL_ALIGNED(best_k, 4, "best_k");
  DFL_ALIGNED(out_tok, 4, "out_tok");
  DFL_CUDA(launch_accept(R, K, B, draft, target, n_acc, best_k, out_tok,
                         static_cast<cudaStream_t>(stream)),
           "accept kernel");
  return DFLASH_OK;
}

dflash_status dflash_d2sd_candidates(int32_t R, int32_t B, int32_t K, int32_t mask_token_id,
                                     const int32_t* base_tokens, const float* conf,
                                     int32_t* known_len, int32_t* cand_tokens,
                                     int32_t* block_req, void* stream) {
  DFL_CHECK(R >= 0, DFLASH_EINVAL, "R must be >= 0");
  DFL_CHECK(B >= 2 && B <= kMaxBlock, DFLASH_EINVAL, "B must be in [2, %d], got %d", kMaxBlock, B);
  DFL_CHECK(K >= 1 && K <= B - 1, DFLASH_EINVAL, "K must be in [1, B-1], got %d", K);
  if (R == 0) return DFLASH_OK;
  DFL_CHECK(base_tokens && conf && known_len && cand_tokens, DFLASH_EINVAL,
            "a pointer argument is NULL");
  DFL_ALIGNED(base_tokens, 4, "base_tokens");
  DFL_ALIGNED(conf, 4, "conf");
  DFL_ALIGNED(known_len, 4, "known_len");
  DFL_ALIGNED(cand_tokens, 4, "cand_tokens");
  DFL_ALIGNED(block_req, 4, "block_req");
  DFL_CUDA(launch_d2sd(R, B, K, mask_token_id, base_tokens, conf, known_len, cand_tokens,
                       block_req, static_cast<cudaStream_t>(stream)),
           "D2SD cut kernel");
  return DFLASH_OK;
}

dflash_status dflash_advance(const dflash_config* cfg, int32_t R, int32_t K, const int32_t* n_acc,
                             const int32_t* best_k, const int32_t* out_tok,
                             const void* verify_states, int32_t* ctx_len, const int64_t* ctx_off,
                             void* new_states, int32_t* new_count, int32_t* block_tokens,
                             int32_t* known_len, void* ws, size_t ws_bytes, void* stream) {
  dflash_status s = check_config(cfg);
  if (s != DFLASH_OK) return s;
  DFL_CHECK(R >= 0, DFLASH_EINVAL, "R must be >= 0");
  DFL_CHECK(K >= 1 && K <= 32, DFLASH_EINVAL, "K must be in [1, 32], got %d", K);
  if (R == 0) return DFLASH_OK;
  DFL_CHECK(n_acc && out_tok && ctx_len && ctx_off && new_count && block_tokens && known_len,
            DFLASH_EINVAL, "a pointer argument is NULL");
  DFL_PTR(verify_states, "verify_states");
  DFL_PTR(new_states, "new_states");
  DFL_ALIGNED(n_acc, 4, "n_acc");
  DFL_ALIGNED(best_k, 4, "best_k");
  DFL_ALIGNED(out_tok, 4, "out_tok");
  DFL_ALIGNED(ctx_len, 4, "ctx_len");
  DFL_ALIGNED(ctx_off, 8, "ctx_off");
  DFL_ALIGNED(new_count, 4, "new_count");
  DFL_ALIGNED(block_tokens, 4, "block_tokens");
  DFL_ALIGNED(known_len, 4, "known_len");
  if ((s = check_ws(ws, ws_bytes, sizeof(DevStatus))) != DFLASH_OK) return s;
  const int64_t row_bytes = static_cast<int64_t>(cfg->n_target_layers) * cfg->hidden * esize(cfg);
  DFL_CUDA(launch_advance(R, K, cfg->block, row_bytes, n_acc, best_k, out_tok, verify_states,
                          ctx_len, ctx_off, new_states, new_count, block_tokens, known_len,
                          cfg->mask_token_id, status_word(ws), static_cast<cudaStream_t>(stream)),
           "advance kernel");
  return DFLASH_OK;
}

dflash_status dflash_selftest_wait_timeout(void* ws, size_t ws_bytes, int64_t limit_ns,
                                           void* stream) {
  dflash_status s = check_ws(ws, ws_bytes, sizeof(DevStatus));
  if (s != DFLASH_OK) return s;
  DFL_CHECK(limit_ns > 0 && limit_ns <= 2000000000ll, DFLASH_EINVAL,
            "limit_ns must be in (0, 2e9]");
  DFL_CUDA(launch_wait_selftest(status_word(ws), limit_ns, static_cast<cudaStream_t>(stream)),
           "wait self test");
  return DFLASH_OK;
}

dflash_status dflash_draft_step(const dflash_config* c, const dflash_weights* w,
                                const dflash_step_args* a, void* ws, size_t ws_bytes,
                                void* stream) {
  dflash_status s = check_config(c);
  if (s != DFLASH_OK) return s;
  DFL_CHECK(w != nullptr && a != nullptr, DFLASH_EINVAL, "weights / args is NULL");
  DFL_CHECK(a->n_req >= 1 && a->n_blocks >= 1, DFLASH_EINVAL, "n_req and n_blocks must be >= 1");
  DFL_CHECK(a->n_ctx_new >= 0 && a->max_ctx_len >= 0, DFLASH_EINVAL, "negative context size");
  DFL_CHECK(a->n_ctx_new < (int64_t(1) << 31), DFLASH_EINVAL, "n_ctx_new too large");
  const int64_t M = static_cast<int64_t>(a->n_blocks) * c->block;
  DFL_CHECK(a->block_req && a->block_tokens && a->ctx_off && a->draft_tokens, DFLASH_EINVAL,
            "block_req / block_tokens / ctx_off / draft_tokens is NULL");
  DFL_CHECK(a->k_cache && a->v_cache, DFLASH_EINVAL, "k_cache / v_cache is NULL");
  DFL_ALIGNED(a->block_req, 4, "block_req");
  DFL_ALIGNED(a->block_tokens, 4, "block_tokens");
  DFL_ALIGNED(a->known_len, 4, "known_len");
  DFL_ALIGNED(a->ctx_off, 8, "ctx_off");
  DFL_ALIGNED(a->new_off, 8, "new_off");
  DFL_ALIGNED(a->ctx_cached, 4, "ctx_cached");
  DFL_ALIGNED(a->draft_tokens, 4, "draft_tokens");
  DFL_ALIGNED(a->max_logit, 4, "max_logit");
  DFL_ALIGNED(a->confidence, 4, "confidence");
  DFL_ALIGNED(a->target_tokens, 4, "target_tokens");
  DFL_ALIGNED(a->n_acc, 4, "n_acc");
  DFL_ALIGNED(a->best_k, 4, "best_k");
  DFL_ALIGNED(a->out_tok, 4, "out_tok");
  if (a->n_ctx_new > 0) DFL_PTR(a->new_states, "new_states");
  DFL_CHECK(w->layers, DFLASH_EINVAL, "layers is NULL");
  const bool fc = w->w_fc != nullptr;
  if (fc) {
    DFL_PTR(w->w_fc, "w_fc");
    DFL_PTR(w->g_fc, "g_fc");
  } else {
    DFL_CHECK(w->w_fuse != nullptr, DFLASH_EINVAL, "w_fuse is NULL");
  }
  DFL_PTR(w->embed, "embed");
  DFL_PTR(w->lm_head, "lm_head");
  DFL_PTR(w->g_final, "g_final");
  const int D = c->n_draft_layers;
  for (int i = 0; i < D; ++i) {
    const dflash_layer_weights& l = w->layers[i];
    DFL_PTR(l.w_q, "w_q");
    DFL_PTR(l.w_kt, "w_kt");
    DFL_PTR(l.w_vt, "w_vt");
    DFL_PTR(l.w_kd, "w_kd");
    DFL_PTR(l.w_vd, "w_vd");
    DFL_PTR(l.w_o, "w_o");
    DFL_PTR(l.w_gate, "w_gate");
    DFL_PTR(l.w_up, "w_up");
    DFL_PTR(l.w_down, "w_down");
    if (!fc) DFL_PTR(l.g_fuse, "g_fuse");
    DFL_PTR(l.g_attn, "g_attn");
    DFL_PTR(l.g_mlp, "g_mlp");
    if (a->max_ctx_len > 0) {
      DFL_PTR(a->k_cache[i], "k_cache[i]");
      DFL_PTR(a->v_cache[i], "v_cache[i]");
    }
  }
  DFL_ALIGNED(a->ctx_len, 4, "ctx_len");
  DFL_ALIGNED(a->new_count, 4, "new_count");
  if (a->new_count) {
    DFL_CHECK(a->ctx_len != nullptr, DFLASH_EINVAL, "new_count needs ctx_len");
    DFL_CHECK(a->n_ctx_new == static_cast<int64_t>(a->n_req) * c->block, DFLASH_EINVAL,
              "with new_count, n_ctx_new must be n_req * block (%lld != %d * %d)",
              static_cast<long long>(a->n_ctx_new), a->n_req, c->block);
  }
  DFL_CHECK(a->sample == 0 || a->sample == 1, DFLASH_EINVAL, "sample must be 0 or 1");
  const bool sampling = a->sample == 1;
  if (sampling) {
    DFL_CHECK(a->draft_logits != nullptr, DFLASH_EINVAL, "sample = 1 needs draft_logits");
    DFL_ALIGNED(a->draft_logits, 16, "draft_logits");
    DFL_ALIGNED(a->draft_logq, 4, "draft_logq");
    DFL_ALIGNED(a->target_logp, 4, "target_logp");
    if (a->target_logp) {
      DFL_CHECK(a->n_cand == 1 && a->n_blocks == a->n_req, DFLASH_EINVAL,
                "stochastic verification takes one candidate per request (n_cand = 1)");
      DFL_CHECK(a->n_acc && a->out_tok, DFLASH_EINVAL, "n_acc / out_tok is NULL");
      DFL_CHECK(a->n_req < (1 << 26), DFLASH_EINVAL, "n_req too large for the counters");
    }
  }
  if (a->target_tokens && !sampling) {
    DFL_CHECK(a->n_cand >= 1 && a->n_cand <= 32 && a->n_blocks == a->n_req * a->n_cand,
              DFLASH_EINVAL, "verification needs n_blocks == n_req * n_cand (n_cand in [1,32])");
    DFL_CHECK(a->n_acc && a->best_k && a->out_tok, DFLASH_EINVAL,
              "n_acc / best_k / out_tok is NULL");
  }
  const Layout L = make_layout(c, a->n_req, a->n_blocks, a->n_ctx_new, a->max_ctx_len);
  if ((s = check_ws(ws, ws_bytes, L.total)) != DFLASH_OK) return s;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t* status = status_word(ws);
  const int dt = c->dtype;
  const int H = c->hidden, qd = c->n_q_heads * c->head_dim;
  const size_t e = esize(c);
  float* h = at<float>(ws, L.h);
  void* x = at<void>(ws, L.x);
  void* q = at<void>(ws, L.q);
  void* kb = at<void>(ws, L.kb);
  void* vb = at<void>(ws, L.vb);
  void* attn = at<void>(ws, L.attn);
  void* act = at<void>(ws, L.act);
  uint8_t* fused = at<uint8_t>(ws, L.fused);
  float* partial = at<float>(ws, L.partial);
  int32_t* blk_pos = at<int32_t>(ws, L.blk_pos);
  int32_t* new_pos = at<int32_t>(ws, L.new_pos);
  int64_t* new_dst = at<int64_t>(ws, L.new_dst);
  auto* keys = at<unsigned long long>(ws, L.keys);
  uint32_t* counters = at<uint32_t>(ws, L.counters);

  // positions, cache rows, and zeroed argmax keys / tile counters
  DFL_CUDA(launch_prep_rows(a->n_req, a->n_blocks, c->block, a->block_req, a->ctx_off,
                            a->new_off, a->ctx_cached, a->ctx_len, a->new_count, a->n_ctx_new,
                            blk_pos, new_pos, new_dst,
                            at<uint32_t>(ws, L.zero), static_cast<int64_t>(L.zero_bytes / 4),
                            status, st),
           "row bookkeeping");
  float2* rope_tab = at<float2>(ws, L.rope);
  DFL_CUDA(launch_rope_table(rope_tab, L.rope_len, c->head_dim, c->rope_theta, st), "RoPE table");
  // context branch: fusion + every layer's context K/V projection
  SideStream* side = nullptr;
  if (a->n_ctx_new > 0) {
    if ((s = side_stream(&side)) != DFLASH_OK) return s;
    cudaStream_t cs = st;
    if (side) {
      DFL_CUDA(cudaEventRecord(side->fork, st), "fork");
      DFL_CUDA(cudaStreamWaitEvent(side->stream, side->fork, 0), "fork");
      cs = side->stream;
    }
    float* part_c = side ? at<float>(ws, L.partial_side) : partial;
    uint32_t* cnt_c = side ? at<uint32_t>(ws, L.counters_side) : counters;
    // FC variant: fp32 product at the start of the fused region, the one
    // shared context right behind it
    uint8_t* fc_ctx = fused + static_cast<size_t>(a->n_ctx_new) * H * 4;
    // bf16: the fusion leaves the norm's per-row scale to the K/V epilogue
    const bool unnorm = !fc && dt == DFLASH_BF16;
    float* rss = at<float>(ws, L.rss);
    const int rss_parts = fuse_unnorm_parts(H);
    if (fc) {
      s = run_job(job_fc(c, a->new_states, a->n_ctx_new, w->w_fc, reinterpret_cast<float*>(fused)),
                  part_c, cnt_c, status, cs, "FC fusion GEMM");
      if (s != DFLASH_OK) return s;
      DFL_CUDA(launch_rmsnorm(dt, reinterpret_cast<float*>(fused), a->n_ctx_new, H, w->g_fc,
                              c->rms_eps, fc_ctx, cs),
               "FC fusion rmsnorm");
    } else {
      const float* gf[kMaxLayers];
      for (int i = 0; i < D; ++i) gf[i] = w->layers[i].g_fuse;
      if (unnorm)
        DFL_CUDA(launch_fuse_unnorm(a->new_states, a->n_ctx_new, c->n_target_layers, H, D,
                                    w->w_fuse, gf, fused, rss, status, cs),
                 "fusion kernel");
      else
        DFL_CUDA(launch_fuse(dt, a->new_states, a->n_ctx_new, c->n_target_layers, H, D,
                             w->w_fuse, gf, fused, c->rms_eps, status, cs),
                 "fusion kernel");
    }
    for (int i = 0; i < D; ++i) {
      const dflash_layer_weights& l = w->layers[i];
      const void* ctx_i = fc ? static_cast<const void*>(fc_ctx)
                             : fused + static_cast<size_t>(i) * a->n_ctx_new * H * e;
      GemmJob jc = job_kv(c, ctx_i, a->n_ctx_new, new_pos, new_dst, l.w_kt, l.w_vt,
                          a->k_cache[i], a->v_cache[i]);
      jc.rope_tab = rope_tab;
      jc.rope_len = L.rope_len;
      if (unnorm) {   // the fusion's RMSNorm, applied per row in the epilogue
        jc.rss = rss + static_cast<size_t>(i) * a->n_ctx_new * rss_parts;
        jc.rss_parts = rss_parts;
        jc.rss_inv = 1.f / static_cast<float>(H);
        jc.rss_eps = c->rms_eps;
      }
      s = run_job(jc, part_c, cnt_c, status, cs, "context K/V GEMM");
      if (s != DFLASH_OK) return s;
      if (side) DFL_CUDA(cudaEventRecord(side->done[i], side->stream), "context done");
    }
  }
  DFL_CUDA(launch_embed(dt, w->embed, H, a->n_blocks, c->block, a->block_tokens, a->known_len,
                        c->mask_token_id, c->vocab, h, status, st),
           "slot embedding");
  const AttnPlan ap = plan_attn(dt, a->n_blocks, c->block, c->n_q_heads, c->n_kv_heads,
                                c->head_dim, a->max_ctx_len);
  for (int i = 0; i < D; ++i) {
    const dflash_layer_weights& l = w->layers[i];
    // block: RMSNorm -> Q (RoPE), K^d (RoPE), V^d
    DFL_CUDA(launch_rmsnorm(dt, h, M, H, l.g_attn, c->rms_eps, x, st), "attention rmsnorm");
    GemmJob jq = job_qkv(c, l, x, M, blk_pos, q, kb, vb);
    jq.rope_tab = rope_tab;
    jq.rope_len = L.rope_len;
    if ((s = run_job(jq, partial, counters, status, st, "QKV GEMM")) != DFLASH_OK) return s;
    if (side) DFL_CUDA(cudaStreamWaitEvent(st, side->done[i], 0), "join context");
    DFL_CUDA(launch_attn(dt, ap, a->n_blocks, c->block, c->n_q_heads, c->n_kv_heads,
                         c->head_dim, q, kb, vb, a->k_cache[i], a->v_cache[i], a->ctx_off,
                         a->block_req, attn, at<float>(ws, L.attn_ws), status, st, a->ctx_len),
             "attention");
    if ((s = run_job(job_resid(c, l.w_o, attn, M, qd, h), partial, counters, status, st,
                     "O GEMM")) != DFLASH_OK)
      return s;
    DFL_CUDA(launch_rmsnorm(dt, h, M, H, l.g_mlp, c->rms_eps, x, st), "mlp rmsnorm");
    if ((s = run_job(job_swiglu(c, l.w_gate, l.w_up, x, M, act), partial, counters, status, st,
                     "gate/up GEMM")) != DFLASH_OK)
      return s;
    if ((s = run_job(job_resid(c, l.w_down, act, M, c->ffn, h), partial, counters, status, st,
                     "down GEMM")) != DFLASH_OK)
      return s;
  }
  DFL_CUDA(launch_rmsnorm(dt, h, M, H, w->g_final, c->rms_eps, x, st), "final rmsnorm");
  if (sampling) {
    // temperature 1: logits to the caller's buffer, a Gumbel-max draw per
    // slot, then (optionally) stochastic verification
    float* row_lse = at<float>(ws, L.row_lse);
    s = run_job(job_logits(c, x, M, w->lm_head, a->draft_logits), partial, counters, status, st,
                "LM head logits GEMM");
    if (s != DFLASH_OK) return s;
    DFL_CUDA(launch_sample_rows(a->draft_logits, M, c->vocab, a->seed, a->rng_offset, c->block,
                                a->block_tokens, a->known_len, a->draft_tokens, a->draft_logq,
                                row_lse, status, st),
             "sampling kernel");
    if (a->target_logp) {
      DFL_CUDA(launch_accept_stochastic(a->n_req, c->block, c->vocab, a->draft_tokens,
                                        a->draft_logits, row_lse, a->target_logp, a->seed,
                                        a->rng_offset, a->n_acc, a->out_tok, keys, status, st),
               "stochastic accept");
    }
    return DFLASH_OK;
  }
  float2* lse = a->confidence ? at<float2>(ws, L.lse) : nullptr;
  DFL_CUDA(launch_lmhead_argmax(dt, w->lm_head, c->vocab, x, M, H, keys, status, st, partial,
                                counters, lse),
           "LM head argmax");
  DFL_CUDA(launch_argmax_finish(keys, M, c->block, a->block_tokens, a->known_len,
                                a->draft_tokens, a->max_logit, st, lse,
                                lmhead_tiles(dt, c->vocab, M), a->confidence),
           "argmax finish");
  if (a->target_tokens) {
    DFL_CUDA(launch_accept(a->n_req, a->n_cand, c->block, a->draft_tokens, a->target_tokens,
                           a->n_acc, a->best_k, a->out_tok, st),
             "accept kernel");
  }
  return DFLASH_OK;
}

}  // extern "C"

// ===========================================================================
// LM-head argmax for callers that cannot allocate device memory
// ===========================================================================
// Some callers cannot call cudaMalloc or hand us a workspace: a plugin loaded
// into a serving process whose device memory is owned by that process's
// caching allocator, or a latency-critical loop that is not allowed to
// allocate after start-up.  This variant keeps its only scratch -- one
// 64-bit argmax key per token -- in a fixed array that lives in the module's
// global memory for as long as the library is loaded, on every GPU that
// loads it.
namespace dfl {
namespace {

constexpr int64_t kNoAllocMaxTokens = 4096;       // 32 KiB of keys per device
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned long long g_noalloc_keys[kNoAllocMaxTokens];

std::mutex g_noalloc_mu;
unsigned long long* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_keys on the current device.  In host code the
// array's name is only a stand-in, so the address is looked up once per
// device (with that device current) and cached.
dflash_status noalloc_scratch(unsigned long long** out) {
  int dev = 0;
  DFL_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  DFL_CHECK(dev >= 0 && dev < kNoAllocMaxDevices, DFLASH_EUNSUPPORTED,
            "device ordinal %d beyond %d", dev, kNoAllocMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    DFL_CUDA(cudaGetSymbolAddress(&p, g_noalloc_keys), "cudaGetSymbolAddress");
    g_noalloc_ptr[dev] = static_cast<unsigned long long*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return DFLASH_OK;
}

}  // namespace
}  // namespace dfl

extern "C" dflash_status dflash_lmhead_argmax_noalloc(const dflash_config* cfg, int64_t M,
                                                      const void* x, const void* w_lm,
                                                      int32_t* tok, float* max_logit,
                                                      void* stream) {
  dflash_status s = check_config(cfg);
  if (s != DFLASH_OK) return s;
  DFL_CHECK(M >= 0 && M <= kNoAllocMaxTokens, DFLASH_EINVAL,
            "M = %lld exceeds the %lld tokens this allocation-free variant can hold",
            static_cast<long long>(M), static_cast<long long>(kNoAllocMaxTokens));
  if (M == 0) return DFLASH_OK;
  DFL_PTR(x, "x");
  DFL_PTR(w_lm, "w_lm");
  DFL_CHECK(tok != nullptr, DFLASH_EINVAL, "tok is NULL");
  DFL_ALIGNED(tok, 4, "tok");
  DFL_ALIGNED(max_logit, 4, "max_logit");
  unsigned long long* keys = nullptr;
  if ((s = noalloc_scratch(&keys)) != DFLASH_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the array keeps the previous call's contents: the keys must start at zero
  DFL_CUDA(launch_zero(keys, static_cast<size_t>(M) * 8, st), "argmax key reset");
  DFL_CUDA(launch_lmhead_argmax(cfg->dtype, w_lm, cfg->vocab, x, M, cfg->hidden, keys, nullptr,
                                st),
           "LM head argmax");
  DFL_CUDA(launch_argmax_finish(keys, M, cfg->block, nullptr, nullptr, tok, max_logit, st),
           "argmax finish");
  return DFLASH_OK;
}
