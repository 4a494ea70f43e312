// Temperature-1 drafting and stochastic speculative acceptance.
//
// DFlash summary, methodology step 3: the target checks the drafted block
// with the standard speculative acceptance test (a comparison of log
// probabilities); accepted tokens are emitted and the first rejected slot is
// filled by the target's own generation.  DFLARE summary, section 4: the
// loop also runs with stochastic decoding at temperature 1.
//
//   sample_rows_kernel   one CTA per token row: logsumexp of the row's
//                        stored logits and the Gumbel-max draw
//                        argmax_v (z_v + G_v) in one pass;
//   accept_decide_kernel one warp per request: slot j is accepted while
//                        log U_j < log p_j(d_j) - log q_j(d_j) (ballot);
//   resid_draw_kernel    many CTAs per request: the Gumbel-max draw from
//                        norm(max(0, p - q)) at the first rejected slot (or
//                        from the target's next-slot distribution when every
//                        slot passed), merged with 64-bit atomicMax keys;
//   accept_finish_kernel writes the drawn token and re-arms the keys.
//
// Every uniform is a Philox4x32-10 draw from (seed, counter): draft noise of
// row m, id v: (v >> 2, m, offset, DRFT) word v & 3; acceptance uniform of
// request r, slot j: (j, r, offset, ACPT) word 0; residual / next-slot noise
// of request r at slot j, id v: (v >> 2, 64 r + j, offset, RESD) word v & 3.
#include <algorithm>
#include <cmath>

#include "common.cuh"
#include "internal.h"

namespace dfl {

namespace {

__device__ __forceinline__ uint32_t word_of(const uint4& w, int e) {
  return e == 0 ? w.x : e == 1 ? w.y : e == 2 ? w.z : w.w;
}

// (max, sum exp(z - max)) merge of two partial log-sum-exp states
__device__ __forceinline__ void lse_merge(float& m, float& s, float m2, float s2) {
  if (m2 > m) {
    s = s * __expf(m - m2) + s2;
    m = m2;
  } else if (m2 > -INFINITY) {
    s += s2 * __expf(m2 - m);
  }
}

constexpr int kSampleThreads = 512;

}  // namespace

// ---------------------------------------------------------------------------
// Gumbel-max draw of every token row from its stored logits.  Known-prefix
// slots (s < known_len of their block) keep their input token.
// ---------------------------------------------------------------------------
template <bool VEC4>
__global__ void __launch_bounds__(kSampleThreads) sample_rows_kernel(
    const float* __restrict__ logits, int V, uint32_t k0, uint32_t k1, uint32_t offset, int B,
    const int32_t* __restrict__ block_tokens, const int32_t* __restrict__ known_len,
    int32_t* __restrict__ tok, float* __restrict__ logq, float* __restrict__ lse_out,
    uint32_t* status) {
  __shared__ unsigned long long s_key[kSampleThreads / 32];
  __shared__ float s_m[kSampleThreads / 32], s_s[kSampleThreads / 32];
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int64_t m = blockIdx.x;
  const float* row = logits + m * V;
  unsigned long long best = 0ull;
  float mx = -INFINITY, se = 0.f;
  const int nq = (V + 3) >> 2;
  for (int q = threadIdx.x; q < nq; q += blockDim.x) {
    float z[4];
    if (VEC4) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(row) + q);
      z[0] = v.x; z[1] = v.y; z[2] = v.z; z[3] = v.w;
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) z[e] = 4 * q + e < V ? __ldg(row + 4 * q + e) : -INFINITY;
    }
    const uint4 w = philox4x32_10(make_uint4(static_cast<uint32_t>(q), static_cast<uint32_t>(m),
                                             offset, kRngDraft), k0, k1);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int v = 4 * q + e;
      if (v >= V) break;
      const unsigned long long k = argmax_key(z[e] + gumbel_from_word(word_of(w, e)),
                                              static_cast<uint32_t>(v));
      best = k > best ? k : best;
      lse_merge(mx, se, z[e], 1.f);
    }
  }
  best = warp_max_u64(best);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, mx, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, se, o);
    lse_merge(mx, se, m2, s2);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    s_key[warp] = best;
    s_m[warp] = mx;
    s_s[warp] = se;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const int nw = blockDim.x >> 5;
    unsigned long long k = s_key[0];
    float M = s_m[0], S = s_s[0];
    for (int i = 1; i < nw; ++i) {   // fixed order: deterministic
      k = s_key[i] > k ? s_key[i] : k;
      lse_merge(M, S, s_m[i], s_s[i]);
    }
    const float lse = M + logf(S);
    int32_t t = static_cast<int32_t>(key_index(k));
    if (block_tokens != nullptr) {
      const int64_t b = m / B;
      const int kl = known_len ? known_len[b] : 1;
      if (m % B < kl) t = block_tokens[m];
    }
    if (!DFL_BOUNDS(t >= 0 && t < V, status, 89)) t = 0;
    tok[m] = t;
    if (logq) logq[m] = row[t] - lse;
    if (lse_out) lse_out[m] = lse;
  }
}

cudaError_t launch_sample_rows(const float* logits, int64_t M, int V, uint64_t seed,
                               uint32_t offset, int B, const int32_t* block_tokens,
                               const int32_t* known_len, int32_t* tok, float* logq,
                               float* lse, uint32_t* status, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  const bool vec = (V % 4) == 0 && (reinterpret_cast<uintptr_t>(logits) & 15u) == 0;
  const dim3 grid(static_cast<unsigned>(M));
  if (vec)
    return launch_k(sample_rows_kernel<true>, grid, dim3(kSampleThreads), 0, st, logits, V, k0,
                    k1, offset, B, block_tokens, known_len, tok, logq, lse, status);
  return launch_k(sample_rows_kernel<false>, grid, dim3(kSampleThreads), 0, st, logits, V, k0,
                  k1, offset, B, block_tokens, known_len, tok, logq, lse, status);
}

// ---------------------------------------------------------------------------
// Stochastic acceptance, one candidate block per request.
// draft [R][B]; draft_logits [R][B][V] with per-row logsumexp draft_lse
// [R][B]; target_logp [R][B][V], row j = log p(. | slots 0..j) (the target's
// distribution for slot j + 1).
// ---------------------------------------------------------------------------
__global__ void accept_decide_kernel(int R, int B, int V, const int32_t* __restrict__ draft,
                                     const float* __restrict__ draft_logits,
                                     const float* __restrict__ draft_lse,
                                     const float* __restrict__ target_logp, uint32_t k0,
                                     uint32_t k1, uint32_t offset, int32_t* __restrict__ n_acc,
                                     int32_t* __restrict__ out_tok,
                                     unsigned long long* __restrict__ keys, uint32_t* status) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  bool ok = false;
  if (lane >= 1 && lane < B) {
    const size_t row = static_cast<size_t>(r) * B + lane;
    int32_t d = draft[row];
    if (!DFL_BOUNDS(d >= 0 && d < V, status, 88)) d = 0;
    const float lq = draft_logits[row * V + d] - draft_lse[row];
    const float lp = target_logp[(row - 1) * V + d];
    const uint4 w = philox4x32_10(make_uint4(static_cast<uint32_t>(lane),
                                             static_cast<uint32_t>(r), offset, kRngAccept),
                                  k0, k1);
    ok = logf(uniform_from_word(w.x)) < lp - lq;
  }
  const uint32_t bits = __ballot_sync(0xffffffffu, ok) >> 1;   // bit j-1 <-> slot j
  const int n = __ffs(~bits) - 1;                                // leading run of passes
  if (lane < B) {
    const size_t row = static_cast<size_t>(r) * B;
    out_tok[row + lane] = lane < n ? draft[row + lane + 1] : -1;
  }
  if (lane == 0) {
    n_acc[r] = n;
    keys[r] = 0ull;
  }
}

// Gumbel-max over the residual max(0, p - q) at slot n + 1 (or over p at the
// slot after the block); grid (R, chunks of the vocabulary).
__global__ void __launch_bounds__(256) resid_draw_kernel(
    int R, int B, int V, const float* __restrict__ draft_logits,
    const float* __restrict__ draft_lse, const float* __restrict__ target_logp, uint32_t k0,
    uint32_t k1, uint32_t offset, const int32_t* __restrict__ n_acc,
    unsigned long long* __restrict__ keys) {
  __shared__ unsigned long long s_key[8];
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int r = blockIdx.x;
  const int n = n_acc[r];
  const int slot = n + 1;
  const bool resid = slot < B;
  const float* tp = target_logp + (static_cast<size_t>(r) * B + n) * V;
  const float* dl = resid ? draft_logits + (static_cast<size_t>(r) * B + slot) * V : nullptr;
  const float dlse = resid ? draft_lse[static_cast<size_t>(r) * B + slot] : 0.f;
  const uint32_t c1 = static_cast<uint32_t>(r) * 64u + static_cast<uint32_t>(slot);
  const int nq = (V + 3) >> 2;
  unsigned long long best = 0ull;
  for (int q = blockIdx.y * blockDim.x + threadIdx.x; q < nq; q += gridDim.y * blockDim.x) {
    const uint4 w = philox4x32_10(make_uint4(static_cast<uint32_t>(q), c1, offset, kRngResid),
                                  k0, k1);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int v = 4 * q + e;
      if (v >= V) break;
      float key;
      if (resid) {
        const float res = __expf(tp[v]) - __expf(dl[v] - dlse);
        if (!(res > 0.f)) continue;
        key = logf(res);
      } else {
        key = tp[v];
      }
      const unsigned long long k =
          argmax_key(key + gumbel_from_word(word_of(w, e)), static_cast<uint32_t>(v));
      best = k > best ? k : best;
    }
  }
  best = warp_max_u64(best);
  if ((threadIdx.x & 31) == 0) s_key[threadIdx.x >> 5] = best;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long k = s_key[0];
    for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i) k = s_key[i] > k ? s_key[i] : k;
    if (k) atomicMax(keys + r, k);
  }
}

__global__ void accept_finish_kernel(int R, int B, const int32_t* __restrict__ n_acc,
                                     unsigned long long* __restrict__ keys,
                                     int32_t* __restrict__ out_tok) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= R) return;
  out_tok[static_cast<size_t>(r) * B + n_acc[r]] = static_cast<int32_t>(key_index(keys[r]));
  keys[r] = 0ull;
}

cudaError_t launch_accept_stochastic(int R, int B, int V, const int32_t* draft,
                                     const float* draft_logits, const float* draft_lse,
                                     const float* target_logp, uint64_t seed, uint32_t offset,
                                     int32_t* n_acc, int32_t* out_tok,
                                     unsigned long long* keys, uint32_t* status,
                                     cudaStream_t st) {
  if (R <= 0) return cudaSuccess;
  const uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  const int wpb = 4;
  cudaError_t e = launch_k(accept_decide_kernel, dim3((R + wpb - 1) / wpb), dim3(wpb * 32), 0,
                           st, R, B, V, draft, draft_logits, draft_lse, target_logp, k0, k1,
                           offset, n_acc, out_tok, keys, status);
  if (e != cudaSuccess) return e;
  // enough CTAs to stream the two rows of every request at full bandwidth
  const int nq = (V + 3) / 4;
  const int chunks = std::max(1, std::min((nq + 255) / 256, (2 * kNumSMs + R - 1) / R));
  e = launch_k(resid_draw_kernel, dim3(R, chunks), dim3(256), 0, st, R, B, V, draft_logits,
               draft_lse, target_logp, k0, k1, offset, n_acc, keys);
  if (e != cudaSuccess) return e;
  return launch_k(accept_finish_kernel, dim3((R + 127) / 128), dim3(128), 0, st, R, B, n_acc,
                  keys, out_tok);
}

}  // namespace dfl
