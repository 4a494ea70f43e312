// Block attention with KV injection (DFLARE summary, section 2.2): the B
// block queries of every head attend, without a mask, to the keys of
// [request context ; this block], GQA group G = Hq / Hkv.
//
// Split-KV (flash-decoding): the grid is (block x kv head, split, query-row
// chunk).  A split streams its slice of the request's packed context K/V
// (split 0 also takes the B block keys) and keeps an fp32 online softmax
// (running max m, sum l, unnormalised output o) per query row; a combine
// kernel merges the splits in a fixed order.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dfl {

struct AttnParams {
  const void* q;
  const void* kb;
  const void* vb;
  const void* kc;
  const void* vc;
  const int64_t* ctx_off;
  const int32_t* block_req;
  int B, Hq, Hkv, G;
  int splits, chunk, rows_per_cta;
  float scale;
  float* part_o;   // [nb*B*Hq][splits][d]
  float* part_ml;  // [nb*B*Hq][splits][2]
};

constexpr int kAttnWarps = 4;
constexpr int kAttnRowsPerWarp = 8;
constexpr int kAttnKeyTile = 32;

template <typename T, int D>
__global__ void __launch_bounds__(kAttnWarps * 32) attn_simt_kernel(const AttnParams p) {
  extern __shared__ float sm[];
  constexpr int NO = D / 32;
  const int rows_cta = kAttnWarps * kAttnRowsPerWarp;
  float* qs = sm;                              // [rows_cta][D]
  float* ks = qs + rows_cta * D;               // [32][D+1]
  float* vs = ks + kAttnKeyTile * (D + 1);     // [32][D]
  const int b = blockIdx.x / p.Hkv, g = blockIdx.x % p.Hkv;
  const int split = blockIdx.y;
  const int r = p.block_req[b];
  const int64_t c_begin = p.ctx_off[r];
  const int64_t L = p.ctx_off[r + 1] - c_begin;
  const int64_t k_lo = static_cast<int64_t>(split) * p.chunk;
  const int n_ctx = static_cast<int>(std::max<int64_t>(0, std::min<int64_t>(L, k_lo + p.chunk) - k_lo));
  const int n_blk = split == 0 ? p.B : 0;
  const int total = n_ctx + n_blk;
  const int nrows_all = p.B * p.G;
  const int row0 = blockIdx.z * rows_cta;
  const int nrows = min(rows_cta, nrows_all - row0);
  const T* Q = static_cast<const T*>(p.q);
  const T* KB = static_cast<const T*>(p.kb);
  const T* VB = static_cast<const T*>(p.vb);
  const T* KC = static_cast<const T*>(p.kc);
  const T* VC = static_cast<const T*>(p.vc);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  for (int e = tid; e < nrows * D; e += blockDim.x) {
    const int rr = row0 + e / D;
    const int s = rr / p.G, j = rr % p.G;
    qs[e] = to_f(Q[((static_cast<size_t>(b) * p.B + s) * p.Hq + g * p.G + j) * D + e % D]);
  }
  float o[kAttnRowsPerWarp][NO];
  float m[kAttnRowsPerWarp], l[kAttnRowsPerWarp];
#pragma unroll
  for (int i = 0; i < kAttnRowsPerWarp; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
#pragma unroll
    for (int x = 0; x < NO; ++x) o[i][x] = 0.f;
  }
  for (int t0 = 0; t0 < total; t0 += kAttnKeyTile) {
    __syncthreads();
    for (int e = tid; e < kAttnKeyTile * D; e += blockDim.x) {
      const int kk = e / D, dd = e % D;
      const int key = t0 + kk;
      float kv = 0.f, vv = 0.f;
      if (key < n_ctx) {
        const size_t src = ((c_begin + k_lo + key) * p.Hkv + g) * D + dd;
        kv = to_f(KC[src]);
        vv = to_f(VC[src]);
      } else if (key < total) {
        const size_t src = ((static_cast<size_t>(b) * p.B + (key - n_ctx)) * p.Hkv + g) * D + dd;
        kv = to_f(KB[src]);
        vv = to_f(VB[src]);
      }
      ks[kk * (D + 1) + dd] = kv;
      vs[kk * D + dd] = vv;
    }
    __syncthreads();
    const int nvalid = min(kAttnKeyTile, total - t0);
#pragma unroll
    for (int i = 0; i < kAttnRowsPerWarp; ++i) {
      const int row = warp * kAttnRowsPerWarp + i;
      if (row >= nrows) break;
      const float* qr = qs + row * D;
      const float* kr = ks + lane * (D + 1);
      float s = 0.f;
#pragma unroll 8
      for (int dd = 0; dd < D; ++dd) s = fmaf(qr[dd], kr[dd], s);
      s = lane < nvalid ? s * p.scale : -INFINITY;
      const float mnew = fmaxf(m[i], warp_max(s));
      const float corr = expf(m[i] - mnew);
      const float pr = expf(s - mnew);
      l[i] = l[i] * corr + warp_sum(pr);
#pragma unroll
      for (int x = 0; x < NO; ++x) o[i][x] *= corr;
      for (int kk = 0; kk < nvalid; ++kk) {
        const float pk = __shfl_sync(0xffffffffu, pr, kk);
#pragma unroll
        for (int x = 0; x < NO; ++x) o[i][x] = fmaf(pk, vs[kk * D + lane + 32 * x], o[i][x]);
      }
      m[i] = mnew;
    }
  }
#pragma unroll
  for (int i = 0; i < kAttnRowsPerWarp; ++i) {
    const int row = warp * kAttnRowsPerWarp + i;
    if (row >= nrows) break;
    const int rr = row0 + row;
    const int s = rr / p.G, j = rr % p.G;
    const size_t pr = (static_cast<size_t>(b) * p.B + s) * p.Hq + g * p.G + j;
    float* po = p.part_o + (pr * p.splits + split) * D;
#pragma unroll
    for (int x = 0; x < NO; ++x) po[lane + 32 * x] = o[i][x];
    if (lane == 0) {
      p.part_ml[(pr * p.splits + split) * 2 + 0] = m[i];
      p.part_ml[(pr * p.splits + split) * 2 + 1] = l[i];
    }
  }
}

// out[pr][dd] = sum_s o_s e^{m_s - M} / sum_s l_s e^{m_s - M}
template <typename T>
__global__ void attn_combine_kernel(const float* __restrict__ part_o,
                                    const float* __restrict__ part_ml, int64_t n_rows, int splits,
                                    int D, T* __restrict__ out) {
  const int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (idx >= n_rows * D) return;
  const int64_t pr = idx / D;
  const int dd = static_cast<int>(idx % D);
  const float* ml = part_ml + pr * splits * 2;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s)
    if (ml[2 * s + 1] > 0.f) M = fmaxf(M, ml[2 * s]);
  float num = 0.f, den = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float ls = ml[2 * s + 1];
    if (ls > 0.f) {
      const float w = expf(ml[2 * s] - M);
      den = fmaf(ls, w, den);
      num = fmaf(part_o[(pr * splits + s) * D + dd], w, num);
    }
  }
  out[idx] = from_f<T>(num / den);
}

// Opt every attention kernel into large dynamic shared memory once (on the
// first call, which must come before any stream capture).
static cudaError_t allow_smem() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    const int bytes = 200 * 1024;
    const void* ks[4] = {reinterpret_cast<const void*>(attn_simt_kernel<float, 64>),
                         reinterpret_cast<const void*>(attn_simt_kernel<float, 128>),
                         reinterpret_cast<const void*>(attn_simt_kernel<__nv_bfloat16, 64>),
                         reinterpret_cast<const void*>(attn_simt_kernel<__nv_bfloat16, 128>)};
    for (const void* k : ks) {
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (e != cudaSuccess && err == cudaSuccess) err = e;
    }
  });
  return err;
}

AttnPlan plan_attn(int dtype, int nb, int B, int Hq, int Hkv, int d, int64_t max_ctx_len) {
  (void)dtype;
  (void)d;
  AttnPlan p{};
  p.rows_per_cta = kAttnWarps * kAttnRowsPerWarp;
  const int G = Hq / Hkv;
  p.row_chunks = (B * G + p.rows_per_cta - 1) / p.rows_per_cta;
  const int64_t base = static_cast<int64_t>(nb) * Hkv * p.row_chunks;
  if (max_ctx_len <= 0) {
    p.splits = 1;
    p.chunk = 64;
    return p;
  }
  const int64_t max_splits = std::min<int64_t>(64, (max_ctx_len + 63) / 64);
  int64_t want = (2 * kNumSMs + base - 1) / base;
  int64_t splits = std::max<int64_t>(1, std::min(want, max_splits));
  int64_t chunk = (max_ctx_len + splits - 1) / splits;
  chunk = (chunk + 63) / 64 * 64;
  p.chunk = static_cast<int>(chunk);
  p.splits = static_cast<int>((max_ctx_len + chunk - 1) / chunk);
  return p;
}

size_t attn_ws_bytes(const AttnPlan& p, int nb, int B, int Hq, int d) {
  const size_t rows = static_cast<size_t>(nb) * B * Hq;
  return rows * p.splits * (d + 2) * sizeof(float);
}

cudaError_t launch_attn(int dtype, const AttnPlan& plan, int nb, int B, int Hq, int Hkv, int d,
                        const void* q, const void* kb, const void* vb, const void* kc,
                        const void* vc, const int64_t* ctx_off, const int32_t* block_req,
                        void* out, float* ws, uint32_t* status, cudaStream_t st) {
  (void)status;
  if (nb <= 0) return cudaSuccess;
  AttnParams p{};
  p.q = q; p.kb = kb; p.vb = vb; p.kc = kc; p.vc = vc;
  p.ctx_off = ctx_off;
  p.block_req = block_req;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv;
  p.splits = plan.splits;
  p.chunk = plan.chunk;
  p.rows_per_cta = plan.rows_per_cta;
  p.scale = 1.0f / sqrtf(static_cast<float>(d));
  const int64_t n_rows = static_cast<int64_t>(nb) * B * Hq;
  p.part_o = ws;
  p.part_ml = ws + static_cast<size_t>(n_rows) * plan.splits * d;
  dim3 grid(nb * Hkv, plan.splits, plan.row_chunks);
  const size_t smem = (static_cast<size_t>(plan.rows_per_cta) * d +
                       kAttnKeyTile * (d + 1) + kAttnKeyTile * d) * sizeof(float);
  cudaError_t e = cudaSuccess;
#define DFL_ATTN(T, DD)                                                                    \
  do {                                                                                     \
    if ((e = allow_smem()) != cudaSuccess) return e;                                       \
    attn_simt_kernel<T, DD><<<grid, kAttnWarps * 32, smem, st>>>(p);                       \
  } while (0)
  if (dtype == DFLASH_BF16) {
    if (d == 64) DFL_ATTN(__nv_bfloat16, 64); else DFL_ATTN(__nv_bfloat16, 128);
  } else {
    if (d == 64) DFL_ATTN(float, 64); else DFL_ATTN(float, 128);
  }
#undef DFL_ATTN
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t total = n_rows * d;
  const unsigned cgrid = static_cast<unsigned>((total + 255) / 256);
  if (dtype == DFLASH_BF16)
    attn_combine_kernel<__nv_bfloat16><<<cgrid, 256, 0, st>>>(
        p.part_o, p.part_ml, n_rows, plan.splits, d, static_cast<__nv_bfloat16*>(out));
  else
    attn_combine_kernel<float><<<cgrid, 256, 0, st>>>(p.part_o, p.part_ml, n_rows, plan.splits,
                                                      d, static_cast<float*>(out));
  count_launch();
  return cudaGetLastError();
}

}  // namespace dfl
