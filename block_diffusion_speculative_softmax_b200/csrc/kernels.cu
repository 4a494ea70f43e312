// Bandwidth- and latency-bound kernels of the draft step.
#include <algorithm>
#include <cstdlib>
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dfl {

// ===========================================================================
// Adaptive layer fusion + RMSNorm (DFLARE summary, section 2.1)
//
// Persistent CTAs walk the context rows.  A row's T target states are
// contiguous ([T][H]), so thread 0 streams whole rows into a shared-memory
// ring with cp.async.bulk (one copy per row, completion on an mbarrier).
// Thread t owns one 16-byte vector of columns: it reads that vector of the
// T states once and accumulates, in registers, the fused vectors of all D
// draft layers  u_i = sum_j alpha_ij h_j  (alpha_i = softmax(W_fuse[i])) and
// their sums of squares; one block barrier per row combines the sums, and
// f_i = u_i * rsqrt(mean(u_i^2) + eps) * g_i is stored straight from the
// registers.  The states are read from HBM exactly once.
// ===========================================================================
struct FuseGains {
  const float* g[kMaxLayers];
};

// Paired fp32 arithmetic (one instruction for two lanes of a .b64 pair):
// d = a * b + d and d = a * b, elementwise on (0, 1).
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0,
                                      float b1) {
  asm("{.reg .b64 A, B, D;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\t"
      "mov.b64 D, {%0, %1};\n\tfma.rn.f32x2 D, A, B, D;\n\tmov.b64 {%0, %1}, D;}"
      : "+f"(d0), "+f"(d1) : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}
__device__ __forceinline__ void fmul2(float& d0, float& d1, float b0, float b1) {
  asm("{.reg .b64 B, D;\n\tmov.b64 B, {%2, %3};\n\tmov.b64 D, {%0, %1};\n\t"
      "mul.rn.f32x2 D, D, B;\n\tmov.b64 {%0, %1}, D;}"
      : "+f"(d0), "+f"(d1) : "f"(b0), "f"(b1));
}

constexpr int kFuseThreads = 512;
constexpr int kFuseSmemBudget = 221 * 1024;

template <typename T, int MAXD>
__global__ void __launch_bounds__(kFuseThreads) fuse_rows_kernel(
    const T* __restrict__ states, int64_t N, int nT, int H, int D,
    const float* __restrict__ w_fuse, const FuseGains gains, T* __restrict__ fused, float eps,
    int slots, uint32_t* status) {
  using V = Vec16<T>;
  constexpr int VE = V::N;
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ __align__(8) uint64_t full[8];
  __shared__ __align__(16) float alpha[kMaxTargetLayers][MAXD];   // [j][i], zero past D
  __shared__ __align__(16) float red[2][MAXD][32];   // per-warp partial sums, layer-major
  __shared__ volatile int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nwarps = (blockDim.x + 31) >> 5;
  const uint32_t row_bytes = static_cast<uint32_t>(nT) * H * sizeof(T);
  pdl_wait();
  if (tid == 0) pdl_launch();
  if (tid == 0) {
    for (int s = 0; s < slots; ++s) mbar_init(&full[s], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < MAXD) {
    if (tid < D) {
      float mx = -INFINITY;
      for (int j = 0; j < nT; ++j) mx = fmaxf(mx, w_fuse[tid * nT + j]);
      float sum = 0.f;
      for (int j = 0; j < nT; ++j) {
        const float e = expf(w_fuse[tid * nT + j] - mx);
        alpha[j][tid] = e;
        sum += e;
      }
      for (int j = 0; j < nT; ++j) alpha[j][tid] /= sum;
    } else {
      for (int j = 0; j < nT; ++j) alpha[j][tid] = 0.f;
    }
  }
  __syncthreads();
  // rows of this CTA: blockIdx.x, blockIdx.x + gridDim.x, ...
  const int64_t my_rows = N > blockIdx.x ? (N - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  if (tid == 0) {
    for (int k = 0; k < slots && k < my_rows; ++k) {
      const int64_t n = blockIdx.x + k * static_cast<int64_t>(gridDim.x);
      mbar_arrive_expect_tx(&full[k], row_bytes);
      bulk_load(ring + static_cast<size_t>(k) * row_bytes, states + n * nT * H, row_bytes,
                &full[k]);
    }
  }
  const int nvec = H / VE;
  const bool active = tid < nvec;
  const int col = tid * VE;
  int64_t k = 0;
  for (; k < my_rows; ++k) {
    const int slot = static_cast<int>(k % slots);
    const int64_t n = blockIdx.x + k * static_cast<int64_t>(gridDim.x);
    if (!mbar_wait(&full[slot], static_cast<uint32_t>((k / slots) & 1), status, 21)) {
      abort_flag = 1;
    }
    float u[MAXD][VE];
    float ss[MAXD];
#pragma unroll
    for (int i = 0; i < MAXD; ++i) {
      ss[i] = 0.f;
#pragma unroll
      for (int e = 0; e < VE; ++e) u[i][e] = 0.f;
    }
    if (active && !abort_flag) {
      const T* row = reinterpret_cast<const T*>(ring + static_cast<size_t>(slot) * row_bytes);
      for (int j = 0; j < nT; ++j) {
        float h[VE];
        const uint4 raw = *reinterpret_cast<const uint4*>(row + static_cast<size_t>(j) * H + col);
        if constexpr (VE == 8) {
          const __nv_bfloat162* hp = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(hp[q]);
            h[2 * q] = f.x;
            h[2 * q + 1] = f.y;
          }
        } else {
          const float* fp = reinterpret_cast<const float*>(&raw);
#pragma unroll
          for (int q = 0; q < VE; ++q) h[q] = fp[q];
        }
        // alpha[j][0..MAXD) as float4 loads, paired FMAs over column pairs
        float a[MAXD];
#pragma unroll
        for (int q = 0; q < MAXD / 4; ++q) {
          const float4 av = *reinterpret_cast<const float4*>(&alpha[j][4 * q]);
          a[4 * q] = av.x; a[4 * q + 1] = av.y; a[4 * q + 2] = av.z; a[4 * q + 3] = av.w;
        }
#pragma unroll
        for (int i = 0; i < MAXD; ++i) {
          if (i < D) {
#pragma unroll
            for (int e = 0; e < VE; e += 2) ffma2(u[i][e], u[i][e + 1], a[i], a[i], h[e], h[e + 1]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < MAXD; ++i) {
        float s0 = 0.f, s1 = 0.f;
#pragma unroll
        for (int e = 0; e < VE; e += 2) ffma2(s0, s1, u[i][e], u[i][e + 1], u[i][e], u[i][e + 1]);
        ss[i] = s0 + s1;
      }
    }
    const int par = static_cast<int>(k & 1);
#pragma unroll
    for (int i = 0; i < MAXD; ++i) {
      if (i < D) {
        const float v = warp_sum(ss[i]);
        if (lane == 0) red[par][i][warp] = v;
      }
    }
    // the gain does not enter the norm: apply it now, so its loads overlap
    // the reductions and the barrier instead of following them
    if (active && !abort_flag) {
#pragma unroll
      for (int i = 0; i < MAXD; ++i) {
        if (i < D) {
          const float4* g4 = reinterpret_cast<const float4*>(gains.g[i] + col);
#pragma unroll
          for (int q = 0; q < VE / 4; ++q) {
            const float4 gv = __ldg(g4 + q);
            fmul2(u[i][4 * q], u[i][4 * q + 1], gv.x, gv.y);
            fmul2(u[i][4 * q + 2], u[i][4 * q + 3], gv.z, gv.w);
          }
        }
      }
    }
    __syncthreads();   // the slot is consumed and the per-warp sums are visible
    if (tid == 0 && !abort_flag && k + slots < my_rows) {
      const int64_t n2 = blockIdx.x + (k + slots) * static_cast<int64_t>(gridDim.x);
      mbar_arrive_expect_tx(&full[slot], row_bytes);
      bulk_load(ring + static_cast<size_t>(slot) * row_bytes, states + n2 * nT * H, row_bytes,
                &full[slot]);
    }
    if (abort_flag) break;
    if (active) {
#pragma unroll
      for (int i = 0; i < MAXD; ++i) {
        if (i < D) {
          // the per-warp partials of layer i as float4 loads (warps past
          // nwarps wrote nothing: their slots are masked), then a short tree
          const float4* r4 = reinterpret_cast<const float4*>(red[par][i]);
          float4 acc4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
          for (int w4 = 0; w4 < 8; ++w4) {
            if (4 * w4 < nwarps) {
              float4 t = r4[w4];
              if (4 * w4 + 1 >= nwarps) t.y = 0.f;
              if (4 * w4 + 2 >= nwarps) t.z = 0.f;
              if (4 * w4 + 3 >= nwarps) t.w = 0.f;
              acc4.x += t.x; acc4.y += t.y; acc4.z += t.z; acc4.w += t.w;
            }
          }
          const float sc = rsqrtf(((acc4.x + acc4.y) + (acc4.z + acc4.w)) /
                                  static_cast<float>(H) + eps);
          float o[VE];
#pragma unroll
          for (int e = 0; e < VE; e += 2) {
            o[e] = u[i][e];
            o[e + 1] = u[i][e + 1];
            fmul2(o[e], o[e + 1], sc, sc);
          }
          V::store(fused + (static_cast<size_t>(i) * N + n) * H + col, o);
        }
      }
    }
  }
  if (abort_flag && tid == 0) {
    // let copies still in flight land before the CTA's shared memory goes away
    for (int64_t q = k; q < my_rows && q < k + slots; ++q)
      mbar_wait(&full[q % slots], static_cast<uint32_t>((q / slots) & 1), status, 22);
  }
}

// Sums each of NV values over the warp (NV a power of two <= 32): afterwards
// v[0] of lane l holds the warp total of value l / (32 / NV).  Each halving
// step exchanges half of the values still held, so NV values take
// NV - 1 + log2(32 / NV) shuffles instead of 5 NV.
template <int NV>
__device__ __forceinline__ void warp_sum_multi(float (&v)[NV], int lane) {
#pragma unroll
  for (int cnt = NV, off = 16; cnt > 1; cnt >>= 1, off >>= 1) {
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int k = 0; k < cnt / 2; ++k) {
      const float send = up ? v[k] : v[k + cnt / 2];
      const float keep = up ? v[k + cnt / 2] : v[k];
      v[k] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
#pragma unroll
  for (int off = 16 / NV; off >= 1; off >>= 1) v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
}

// ---------------------------------------------------------------------------
// Fusion for the draft step's context branch, without the norm.  RMSNorm is
// a per-row scale: f_i = (u_i * g_i) * rsqrt(mean(u_i^2) + eps).  This
// variant stores v_i = u_i * g_i and adds each warp's share of sum(u_i^2)
// to rss[i][n][w] (one slot per consumer warp w, so the sum's order is
// fixed); the context K/V GEMM applies the row's rsqrt(sum / H + eps) to its
// accumulator row in the epilogue (K and V are
// linear in f, and RoPE commutes with a scalar).  With no cross-warp
// reduction per row, warps never wait for one another: the last warp done
// reading a ring slot (a shared counter) issues the slot's next row.
// ---------------------------------------------------------------------------
template <typename T, int MAXD>
__global__ void __launch_bounds__(kFuseThreads) fuse_rows_unnorm_kernel(
    const T* __restrict__ states, int64_t N, int nT, int H, int D,
    const float* __restrict__ w_fuse, const FuseGains gains, T* __restrict__ fused,
    float* __restrict__ rss, int slots, uint32_t* status) {
  using V = Vec16<T>;
  constexpr int VE = V::N;
  extern __shared__ __align__(128) uint8_t ring[];
  __shared__ __align__(8) uint64_t full[8];
  __shared__ int done_cnt[8];      // warps done with the slot's current row
  __shared__ int64_t last_k[8];    // latest row loaded into the slot
  __shared__ __align__(16) float alpha[kMaxTargetLayers][MAXD];
  __shared__ volatile int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ncw = blockDim.x >> 5;
  const uint32_t row_bytes = static_cast<uint32_t>(nT) * H * sizeof(T);
  pdl_wait();
  if (tid == 0) pdl_launch();
  if (tid == 0) {
    for (int s = 0; s < slots; ++s) {
      mbar_init(&full[s], 1);
      done_cnt[s] = 0;
      last_k[s] = -1;
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < MAXD) {
    if (tid < D) {
      float mx = -INFINITY;
      for (int j = 0; j < nT; ++j) mx = fmaxf(mx, w_fuse[tid * nT + j]);
      float sum = 0.f;
      for (int j = 0; j < nT; ++j) {
        const float e = expf(w_fuse[tid * nT + j] - mx);
        alpha[j][tid] = e;
        sum += e;
      }
      for (int j = 0; j < nT; ++j) alpha[j][tid] /= sum;
    } else {
      for (int j = 0; j < nT; ++j) alpha[j][tid] = 0.f;
    }
  }
  __syncthreads();
  const int64_t my_rows = N > blockIdx.x ? (N - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  auto issue = [&](int64_t k) {   // row k of this CTA into slot k % slots
    const int slot = static_cast<int>(k % slots);
    const int64_t n = blockIdx.x + k * static_cast<int64_t>(gridDim.x);
    last_k[slot] = k;
    mbar_arrive_expect_tx(&full[slot], row_bytes);
    bulk_load(ring + static_cast<size_t>(slot) * row_bytes, states + n * nT * H, row_bytes,
              &full[slot]);
  };
  if (tid == 0)
    for (int64_t k = 0; k < slots && k < my_rows; ++k) issue(k);
  const int nvec = H / VE;
  const bool active = tid < nvec;
  const int col = tid * VE;
  constexpr int GW = 3;   // layers whose gains are in flight ahead of their use
  auto load_gain = [&](float4 (&g)[VE / 4], int i) {
#pragma unroll
    for (int q = 0; q < VE / 4; ++q)
      g[q] = (active && i < D) ? __ldg(reinterpret_cast<const float4*>(gains.g[i] + col) + q)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
  };
  for (int64_t k = 0; k < my_rows; ++k) {
    const int slot = static_cast<int>(k % slots);
    const int64_t n = blockIdx.x + k * static_cast<int64_t>(gridDim.x);
    // the gains are the same for every row: the first GW layers' load while
    // the row arrives and is summed
    float4 gq[GW][VE / 4];
#pragma unroll
    for (int w = 0; w < GW; ++w) load_gain(gq[w], w);
    const bool ok = mbar_wait(&full[slot], static_cast<uint32_t>((k / slots) & 1), status, 26);
    if (!ok) abort_flag = 1;
    float u[MAXD][VE];
#pragma unroll
    for (int i = 0; i < MAXD; ++i)
#pragma unroll
      for (int e = 0; e < VE; ++e) u[i][e] = 0.f;
    if (active && ok) {
      const T* row = reinterpret_cast<const T*>(ring + static_cast<size_t>(slot) * row_bytes);
      for (int j = 0; j < nT; ++j) {
        float h[VE];
        const uint4 raw = *reinterpret_cast<const uint4*>(row + static_cast<size_t>(j) * H + col);
        if constexpr (VE == 8) {
          const __nv_bfloat162* hp = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(hp[q]);
            h[2 * q] = f.x;
            h[2 * q + 1] = f.y;
          }
        } else {
          const float* fp = reinterpret_cast<const float*>(&raw);
#pragma unroll
          for (int q = 0; q < VE; ++q) h[q] = fp[q];
        }
        float a[MAXD];
#pragma unroll
        for (int q = 0; q < MAXD / 4; ++q) {
          const float4 av = *reinterpret_cast<const float4*>(&alpha[j][4 * q]);
          a[4 * q] = av.x; a[4 * q + 1] = av.y; a[4 * q + 2] = av.z; a[4 * q + 3] = av.w;
        }
#pragma unroll
        for (int i = 0; i < MAXD; ++i) {
          if (i < D) {
#pragma unroll
            for (int e = 0; e < VE; e += 2) ffma2(u[i][e], u[i][e + 1], a[i], a[i], h[e], h[e + 1]);
          }
        }
      }
    }
    // this warp is done with the slot: the last warp to finish refills it
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      if (atomicAdd(&done_cnt[slot], 1) == ncw - 1) {
        done_cnt[slot] = 0;
        __threadfence_block();
        if (abort_flag == 0 && k + slots < my_rows) issue(k + slots);
      }
    }
    if (__any_sync(0xffffffffu, abort_flag != 0)) break;
    // this warp's share of every layer's sum of squares (u_i = 0 past D),
    // all layers reduced over the warp together
    float ss[MAXD];
#pragma unroll
    for (int i = 0; i < MAXD; ++i) {
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int e = 0; e < VE; e += 2) ffma2(s0, s1, u[i][e], u[i][e + 1], u[i][e], u[i][e + 1]);
      ss[i] = s0 + s1;
    }
    warp_sum_multi<MAXD>(ss, lane);
    {
      constexpr int per = 32 / MAXD;
      const int li = lane / per;
      if (lane % per == 0 && li < D) rss[(static_cast<size_t>(li) * N + n) * ncw + warp] = ss[0];
    }
    // v_i = u_i * g_i, with layer i + GW's gains loading meanwhile
#pragma unroll
    for (int i = 0; i < MAXD; ++i) {
      if (i < D) {
        float4 gv[VE / 4];
#pragma unroll
        for (int q = 0; q < VE / 4; ++q) gv[q] = gq[i % GW][q];
        if (i + GW < D) load_gain(gq[i % GW], i + GW);
        if (active) {
#pragma unroll
          for (int q = 0; q < VE / 4; ++q) {
            fmul2(u[i][4 * q], u[i][4 * q + 1], gv[q].x, gv[q].y);
            fmul2(u[i][4 * q + 2], u[i][4 * q + 3], gv[q].z, gv[q].w);
          }
          V::store(fused + (static_cast<size_t>(i) * N + n) * H + col, u[i]);
        }
      }
    }
  }
  // after a wait that ran out, let the loads still in flight land before the
  // CTA's shared memory goes away (the latest load of each slot)
  __syncthreads();
  if (abort_flag && tid == 0)
    for (int s = 0; s < slots; ++s)
      if (last_k[s] >= 0)
        mbar_wait(&full[s], static_cast<uint32_t>((last_k[s] / slots) & 1), status, 27);
}

// Ring depth: rows of up to ~96 KB in flight per CTA (two CTAs per SM fit
// when the ring is small), never fewer than two rows.
template <typename T>
static int fuse_slots(int nT, int H) {
  const int rb = nT * H * static_cast<int>(sizeof(T));
  const int two_per_sm = (96 * 1024) / rb;          // rows that keep two CTAs per SM
  if (two_per_sm >= 2) return std::min(8, two_per_sm);
  // one CTA per SM anyway: as many rows in flight as the budget holds
  return std::max(2, std::min(8, kFuseSmemBudget / rb));
}

template <typename T, int MAXD>
static cudaError_t fuse_go(const void* states, int64_t N, int nT, int H, int D,
                           const float* w_fuse, const FuseGains& g, void* fused, float eps,
                           uint32_t* status, cudaStream_t st) {
  const int nvec = H / Vec16<T>::N;
  const int threads = ((nvec + 31) / 32) * 32;
  const int slots = fuse_slots<T>(nT, H);
  const size_t smem = static_cast<size_t>(slots) * nT * H * sizeof(T);
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(fuse_rows_kernel<T, MAXD>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kFuseSmemBudget);
  });
  if (attr != cudaSuccess) return attr;
  // two CTAs per SM when the ring is small enough
  const int per_sm = smem <= 100 * 1024 && threads <= 512 ? 2 : 1;
  const int grid = static_cast<int>(std::min<int64_t>(N, kNumSMs * per_sm));
  return launch_k(fuse_rows_kernel<T, MAXD>, dim3(grid), dim3(threads), smem, st,
                  static_cast<const T*>(states), N, nT, H, D, w_fuse, g,
                  static_cast<T*>(fused), eps, slots, status);
}

// Largest hidden size the fusion kernel covers (one 16-byte vector per
// thread, at most kFuseThreads threads, at least one row in the ring).
template <typename T>
static int fuse_max_hidden(int nT) {
  const int by_threads = kFuseThreads * (16 / static_cast<int>(sizeof(T)));
  const int by_smem = kFuseSmemBudget / 2 / (nT * static_cast<int>(sizeof(T)));
  return std::min(by_threads, by_smem / 16 * 16);
}

template <typename T>
static cudaError_t launch_fuse_t(const void* states, int64_t N, int nT, int H, int D,
                                 const float* w_fuse, const FuseGains& g, void* fused, float eps,
                                 uint32_t* status, cudaStream_t st) {
  if (H > fuse_max_hidden<T>(nT)) return cudaErrorInvalidValue;
  if (D <= 4) return fuse_go<T, 4>(states, N, nT, H, D, w_fuse, g, fused, eps, status, st);
  if (D <= 8) return fuse_go<T, 8>(states, N, nT, H, D, w_fuse, g, fused, eps, status, st);
  return fuse_go<T, 16>(states, N, nT, H, D, w_fuse, g, fused, eps, status, st);
}

template <int MAXD>
static cudaError_t fuse_unnorm_go(const void* states, int64_t N, int nT, int H, int D,
                                  const float* w_fuse, const FuseGains& g, void* fused,
                                  float* rss, uint32_t* status, cudaStream_t st) {
  using T = __nv_bfloat16;
  const int nvec = H / Vec16<T>::N;
  const int threads = ((nvec + 31) / 32) * 32;
  const int rb = nT * H * static_cast<int>(sizeof(T));
  int slots = fuse_slots<T>(nT, H);
  size_t smem = static_cast<size_t>(slots) * rb;
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(fuse_rows_unnorm_kernel<T, MAXD>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kFuseSmemBudget);
  });
  if (attr != cudaSuccess) return attr;
  // two CTAs per SM when registers and the small ring allow it; otherwise
  // one, with as many rows in flight as the shared-memory budget holds
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, fuse_rows_unnorm_kernel<T, MAXD>, threads, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 2) {
    per_sm = 1;
    slots = std::max(2, std::min(8, kFuseSmemBudget / rb));
    smem = static_cast<size_t>(slots) * rb;
  } else {
    per_sm = 2;
  }
  const int grid = static_cast<int>(std::min<int64_t>(N, kNumSMs * per_sm));
  return launch_k(fuse_rows_unnorm_kernel<T, MAXD>, dim3(grid), dim3(threads), smem, st,
                  static_cast<const T*>(states), N, nT, H, D, w_fuse, g, static_cast<T*>(fused),
                  rss, slots, status);
}

int fuse_unnorm_parts(int H) { return (H / Vec16<__nv_bfloat16>::N + 31) / 32; }

cudaError_t launch_fuse_unnorm(const void* states, int64_t N, int nT, int H, int D,
                               const float* w_fuse, const float* const* g_fuse, void* fused,
                               float* rss, uint32_t* status, cudaStream_t st) {
  if (N <= 0) return cudaSuccess;
  if (H > fuse_max_hidden<__nv_bfloat16>(nT)) return cudaErrorInvalidValue;
  FuseGains g{};
  for (int i = 0; i < D; ++i) g.g[i] = g_fuse[i];
  if (D <= 4) return fuse_unnorm_go<4>(states, N, nT, H, D, w_fuse, g, fused, rss, status, st);
  if (D <= 8) return fuse_unnorm_go<8>(states, N, nT, H, D, w_fuse, g, fused, rss, status, st);
  return fuse_unnorm_go<16>(states, N, nT, H, D, w_fuse, g, fused, rss, status, st);
}

int fuse_hidden_limit(int dtype, int nT) {
  return dtype == DFLASH_BF16 ? fuse_max_hidden<__nv_bfloat16>(nT) : fuse_max_hidden<float>(nT);
}

cudaError_t launch_fuse(int dtype, const void* states, int64_t N, int nT, int H, int D,
                        const float* w_fuse, const float* const* g_fuse, void* fused, float eps,
                        uint32_t* status, cudaStream_t st) {
  if (N <= 0) return cudaSuccess;
  FuseGains g{};
  for (int i = 0; i < D; ++i) g.g[i] = g_fuse[i];
  if (dtype == DFLASH_BF16)
    return launch_fuse_t<__nv_bfloat16>(states, N, nT, H, D, w_fuse, g, fused, eps, status, st);
  return launch_fuse_t<float>(states, N, nT, H, D, w_fuse, g, fused, eps, status, st);
}

// ===========================================================================
// Slot embeddings: h[b*B + s] = embed[s < known_len[b] ? tok[b][s] : mask]
// ===========================================================================
template <typename T>
__global__ void embed_kernel(const T* __restrict__ embed, int H, int B,
                             const int32_t* __restrict__ block_tokens,
                             const int32_t* __restrict__ known_len, int mask_id, int vocab,
                             float* __restrict__ h, uint32_t* status) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int m = blockIdx.x;
  const int b = m / B, s = m % B;
  const int kl = known_len ? known_len[b] : 1;
  int tok = s < kl ? block_tokens[m] : mask_id;
  if (!DFL_BOUNDS(tok >= 0 && tok < vocab, status, 87)) tok = mask_id;
  const T* src = embed + static_cast<size_t>(tok) * H;
  for (int c = threadIdx.x; c < H; c += blockDim.x)
    h[static_cast<size_t>(m) * H + c] = to_f(src[c]);
}

cudaError_t launch_embed(int dtype, const void* embed, int H, int nb, int B,
                         const int32_t* block_tokens, const int32_t* known_len, int mask_id,
                         int vocab, float* h, uint32_t* status, cudaStream_t st) {
  if (nb <= 0) return cudaSuccess;
  if (dtype == DFLASH_BF16)
    return launch_k(embed_kernel<__nv_bfloat16>, dim3(nb * B), dim3(256), 0, st,
                    static_cast<const __nv_bfloat16*>(embed), H, B, block_tokens, known_len,
                    mask_id, vocab, h, status);
  return launch_k(embed_kernel<float>, dim3(nb * B), dim3(256), 0, st,
                  static_cast<const float*>(embed), H, B, block_tokens, known_len, mask_id, vocab,
                  h, status);
}

// ===========================================================================
// RMSNorm of the fp32 residual stream into the GEMM input dtype.  One CTA
// per row; every thread holds up to two float4 of the row in registers, so
// the row is read once with all loads in flight.
// ===========================================================================
template <typename T>
__global__ void __launch_bounds__(1024) rmsnorm_kernel(const float* __restrict__ h, int H,
                                                       const float* __restrict__ g, float eps,
                                                       T* __restrict__ x) {
  __shared__ float red[32];
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int64_t m = blockIdx.x;
  const int nv = H >> 2;
  const int i0 = threadIdx.x, i1 = threadIdx.x + blockDim.x;
  const float4* row = reinterpret_cast<const float4*>(h + m * H);
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4 a = i0 < nv ? row[i0] : z;
  const float4 b = i1 < nv ? row[i1] : z;
  float ss = a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w + b.x * b.x + b.y * b.y + b.z * b.z +
             b.w * b.w;
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = rsqrtf(v / static_cast<float>(H) + eps);
  }
  __syncthreads();
  const float sc = red[0];
  const float4* gv = reinterpret_cast<const float4*>(g);
  T* out = x + m * H;
  if (i0 < nv) {
    const float4 q = __ldg(gv + i0);
    const float o[4] = {a.x * sc * q.x, a.y * sc * q.y, a.z * sc * q.z, a.w * sc * q.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) out[4 * i0 + e] = from_f<T>(o[e]);
  }
  if (i1 < nv) {
    const float4 q = __ldg(gv + i1);
    const float o[4] = {b.x * sc * q.x, b.y * sc * q.y, b.z * sc * q.z, b.w * sc * q.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) out[4 * i1 + e] = from_f<T>(o[e]);
  }
}

cudaError_t launch_rmsnorm(int dtype, const float* h, int64_t M, int H, const float* g, float eps,
                           void* x, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  const int nv = H / 4;
  const int threads = std::min(1024, ((nv + 1) / 2 + 31) / 32 * 32);
  if (2 * threads < nv || H % 4) return cudaErrorInvalidValue;
  if (dtype == DFLASH_BF16)
    return launch_k(rmsnorm_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(M)), dim3(threads),
                    0, st, h, H, g, eps, static_cast<__nv_bfloat16*>(x));
  return launch_k(rmsnorm_kernel<float>, dim3(static_cast<unsigned>(M)), dim3(threads), 0, st, h,
                  H, g, eps, static_cast<float*>(x));
}

// ===========================================================================
// Row bookkeeping: RoPE positions of block slots and of new context rows,
// and the cache row each new context row is written to.
// ===========================================================================
__global__ void prep_rows_kernel(int R, int nb, int B, const int32_t* __restrict__ block_req,
                                 const int64_t* __restrict__ ctx_off,
                                 const int64_t* __restrict__ new_off,
                                 const int32_t* __restrict__ ctx_cached,
                                 const int32_t* __restrict__ ctx_len,
                                 const int32_t* __restrict__ new_count, int64_t n_new,
                                 int32_t* __restrict__ blk_pos, int32_t* __restrict__ new_pos,
                                 int64_t* __restrict__ new_dst, uint32_t* __restrict__ zero,
                                 int64_t n_zero, uint32_t* status) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int64_t tid = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = tid; i < n_zero; i += stride) zero[i] = 0u;
  for (int64_t m = tid; m < static_cast<int64_t>(nb) * B; m += stride) {
    const int r = block_req[m / B];
    if (!DFL_BOUNDS(r >= 0 && r < R, status, 81)) {
      blk_pos[m] = 0;
      continue;
    }
    const int64_t L = ctx_len ? static_cast<int64_t>(ctx_len[r]) : ctx_off[r + 1] - ctx_off[r];
    (void)DFL_BOUNDS(L >= 0 && L <= ctx_off[r + 1] - ctx_off[r], status, 82);
    blk_pos[m] = static_cast<int32_t>(L + m % B);
  }
  if (new_count != nullptr) {
    // fixed slots: B per request, the first new_count[r] are the last rows
    // of its context; the others are skipped (destination -1)
    for (int64_t n = tid; n < n_new; n += stride) {
      const int r = static_cast<int>(n / B), j = static_cast<int>(n % B);
      const int c = new_count[r];
      const int64_t p = static_cast<int64_t>(ctx_len[r]) - c + j;
      if (j < c &&
          DFL_BOUNDS(c <= B && p >= 0 && ctx_off[r] + p < ctx_off[r + 1], status, 83)) {
        new_pos[n] = static_cast<int32_t>(p);
        new_dst[n] = ctx_off[r] + p;
      } else {
        new_pos[n] = 0;
        new_dst[n] = -1;
      }
    }
    return;
  }
  const int64_t* off = new_off ? new_off : ctx_off;
  for (int64_t n = tid; n < n_new; n += stride) {
    int lo = 0, hi = R - 1;       // last r with off[r] <= n
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (off[mid] <= n) lo = mid; else hi = mid - 1;
    }
    const int64_t p = (ctx_cached ? ctx_cached[lo] : 0) + (n - off[lo]);
    const bool in = DFL_BOUNDS(p >= 0 && ctx_off[lo] + p < ctx_off[lo + 1], status, 84);
    new_pos[n] = in ? static_cast<int32_t>(p) : 0;
    new_dst[n] = in ? ctx_off[lo] + p : -1;
  }
}

cudaError_t launch_prep_rows(int R, int nb, int B, const int32_t* block_req,
                             const int64_t* ctx_off, const int64_t* new_off,
                             const int32_t* ctx_cached, const int32_t* ctx_len,
                             const int32_t* new_count, int64_t n_new, int32_t* blk_pos,
                             int32_t* new_pos, int64_t* new_dst, uint32_t* zero, int64_t n_zero,
                             uint32_t* status, cudaStream_t st) {
  const int64_t work =
      std::max(std::max<int64_t>(static_cast<int64_t>(nb) * B, n_new), n_zero);
  if (work <= 0) return cudaSuccess;
  const int grid = static_cast<int>(std::min<int64_t>((work + 255) / 256, kNumSMs * 8));
  return launch_k(prep_rows_kernel, dim3(grid), dim3(256), 0, st, R, nb, B, block_req, ctx_off,
                  new_off, ctx_cached, ctx_len, new_count, n_new, blk_pos, new_pos, new_dst, zero,
                  n_zero, status);
}

struct InvFreq {
  double v[64];
};

__global__ void rope_table_kernel(float2* __restrict__ tab, int len, int half, const InvFreq f) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int64_t n = static_cast<int64_t>(len) * half;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int pos = static_cast<int>(e / half), i = static_cast<int>(e % half);
    double ang = static_cast<double>(pos) * f.v[i];
    ang -= 6.283185307179586 * rint(ang * 0.15915494309189535);
    float sn, cs;
    sincosf(static_cast<float>(ang), &sn, &cs);
    tab[e] = make_float2(cs, sn);
  }
}

cudaError_t launch_rope_table(float2* tab, int len, int head_dim, double theta,
                              cudaStream_t st) {
  const int half = head_dim / 2;
  const int64_t n = static_cast<int64_t>(len) * half;
  if (n <= 0) return cudaSuccess;
  InvFreq f{};
  for (int i = 0; i < half && i < 64; ++i) f.v[i] = std::pow(theta, -2.0 * i / head_dim);
  const int grid = static_cast<int>(std::min<int64_t>((n + 255) / 256, kNumSMs * 8));
  return launch_k(rope_table_kernel, dim3(grid), dim3(256), 0, st, tab, len, half, f);
}

__global__ void zero_kernel(uint32_t* __restrict__ p, int64_t n) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = 0u;
}

cudaError_t launch_zero(void* p, size_t bytes, cudaStream_t st) {
  const int64_t n = static_cast<int64_t>(bytes / 4);
  if (n <= 0) return cudaSuccess;
  const int grid = static_cast<int>(std::min<int64_t>((n + 255) / 256, kNumSMs * 8));
  return launch_k(zero_kernel, dim3(grid), dim3(256), 0, st, static_cast<uint32_t*>(p), n);
}

// ===========================================================================
// argmax keys -> tokens (+ max logit); known slots keep their input token
// ===========================================================================
// Confidence of the draft's argmax token: p = exp(max - lse) = 1 / S with
// S = sum over vocabulary tiles of sumexp_t * exp(max_t - max), one warp per
// token (lanes take tiles in a fixed stride, then a fixed-order tree).
__global__ void confidence_kernel(const float2* __restrict__ lse, int tiles, int64_t M,
                                  float* __restrict__ conf) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int64_t m = (blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (m >= M) return;
  float mx = -INFINITY;
  for (int t = lane; t < tiles; t += 32) mx = fmaxf(mx, lse[static_cast<size_t>(t) * M + m].x);
  mx = warp_max(mx);
  float s = 0.f;
  for (int t = lane; t < tiles; t += 32) {
    const float2 v = lse[static_cast<size_t>(t) * M + m];
    if (v.y > 0.f) s += v.y * __expf(v.x - mx);
  }
  s = warp_sum(s);
  if (lane == 0) conf[m] = 1.f / s;
}

__global__ void argmax_finish_kernel(unsigned long long* __restrict__ keys, int64_t M,
                                     int B, const int32_t* __restrict__ block_tokens,
                                     const int32_t* __restrict__ known_len,
                                     int32_t* __restrict__ tok, float* __restrict__ max_logit) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int64_t m = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (m >= M) return;
  const unsigned long long k = keys[m];
  keys[m] = 0ull;   // re-armed for the next LM-head launch
  int32_t t = static_cast<int32_t>(key_index(k));
  if (block_tokens) {
    const int64_t b = m / B;
    const int kl = known_len ? known_len[b] : 1;
    if (m % B < kl) t = block_tokens[m];
  }
  tok[m] = t;
  if (max_logit) max_logit[m] = key_value(k);
}

cudaError_t launch_argmax_finish(unsigned long long* keys, int64_t M, int B,
                                 const int32_t* block_tokens, const int32_t* known_len,
                                 int32_t* tok, float* max_logit, cudaStream_t st,
                                 const float2* lse, int lse_tiles, float* conf) {
  if (M <= 0) return cudaSuccess;
  cudaError_t e = launch_k(argmax_finish_kernel, dim3(static_cast<unsigned>((M + 255) / 256)),
                           dim3(256), 0, st, keys, M, B, block_tokens, known_len, tok, max_logit);
  if (e != cudaSuccess || conf == nullptr || lse == nullptr) return e;
  return launch_k(confidence_kernel, dim3(static_cast<unsigned>((M * 32 + 255) / 256)), dim3(256),
                  0, st, lse, lse_tiles, M, conf);
}

// ===========================================================================
// Greedy acceptance: one warp per request; lane j compares draft[k][j]
// with target[k][j-1] and a ballot gives the accepted prefix of candidate k
// as the run of ones starting at slot 1.
// ===========================================================================
__global__ void accept_kernel(int R, int K, int B, const int32_t* __restrict__ draft,
                              const int32_t* __restrict__ target, int32_t* __restrict__ n_acc,
                              int32_t* __restrict__ best_k, int32_t* __restrict__ out_tok) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  int best_n = -1, best = 0;
  for (int k = 0; k < K; ++k) {
    const int32_t* d = draft + (static_cast<size_t>(r) * K + k) * B;
    const int32_t* t = target + (static_cast<size_t>(r) * K + k) * B;
    const bool eq = lane >= 1 && lane < B && d[lane] == t[lane - 1];
    const uint32_t bits = __ballot_sync(0xffffffffu, eq) >> 1;   // bit j-1 <-> slot j
    const int n = __ffs(~bits) - 1;                               // leading run of ones
    if (n > best_n) { best_n = n; best = k; }
  }
  const int32_t* d = draft + (static_cast<size_t>(r) * K + best) * B;
  const int32_t* t = target + (static_cast<size_t>(r) * K + best) * B;
  if (lane < B) {
    int32_t v = -1;
    if (lane < best_n) v = d[lane + 1];
    else if (lane == best_n) v = t[best_n];
    out_tok[static_cast<size_t>(r) * B + lane] = v;
  }
  if (lane == 0) {
    n_acc[r] = best_n;
    best_k[r] = best;
  }
}

cudaError_t launch_accept(int R, int K, int B, const int32_t* draft, const int32_t* target,
                          int32_t* n_acc, int32_t* best_k, int32_t* out_tok, cudaStream_t st) {
  if (R <= 0) return cudaSuccess;
  const int wpb = 4;
  return launch_k(accept_kernel, dim3((R + wpb - 1) / wpb), dim3(wpb * 32), 0, st, R, K, B, draft,
                  target, n_acc, best_k, out_tok);
}

// ===========================================================================
// D2SD cuts: one warp per request; lane j (1 <= j < B) ranks its confidence
// against every other slot (ties: lower slot first); ranks < K are the cuts,
// ordered by slot through a ballot prefix count.
// ===========================================================================
__global__ void d2sd_kernel(int R, int B, int K, int mask_id, const int32_t* __restrict__ base,
                            const float* __restrict__ conf, int32_t* __restrict__ known_len,
                            int32_t* __restrict__ cand, int32_t* __restrict__ block_req) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= R) return;
  const float c = (lane >= 1 && lane < B) ? conf[static_cast<size_t>(r) * B + lane] : 0.f;
  int rank = 0;
  for (int i = 1; i < B; ++i) {
    const float ci = __shfl_sync(0xffffffffu, c, i);
    if (lane >= 1 && lane < B && (ci < c || (ci == c && i < lane))) ++rank;
  }
  const bool sel = lane >= 1 && lane < B && rank < K;
  const uint32_t mask = __ballot_sync(0xffffffffu, sel);
  if (sel) {
    const int k = __popc(mask & ((1u << lane) - 1u));   // order by slot
    known_len[static_cast<size_t>(r) * K + k] = lane;
    if (block_req) block_req[static_cast<size_t>(r) * K + k] = r;
  }
  // candidate tokens: slot s of candidate k is base[s] if s < p_k else mask
  const int32_t tok = lane < B ? base[static_cast<size_t>(r) * B + lane] : 0;
  uint32_t rest = mask;
  for (int k = 0; k < K; ++k) {
    const int p = __ffs(rest) - 1;
    rest &= rest - 1;
    if (lane < B) cand[(static_cast<size_t>(r) * K + k) * B + lane] = lane < p ? tok : mask_id;
  }
}

cudaError_t launch_d2sd(int R, int B, int K, int mask_id, const int32_t* base, const float* conf,
                        int32_t* known_len, int32_t* cand, int32_t* block_req, cudaStream_t st) {
  if (R <= 0) return cudaSuccess;
  const int wpb = 4;
  return launch_k(d2sd_kernel, dim3((R + wpb - 1) / wpb), dim3(wpb * 32), 0, st, R, B, K, mask_id,
                  base, conf, known_len, cand, block_req);
}

// ===========================================================================
// Roll the speculative window forward on the device (DFlash summary,
// methodology step 4): request r accepted n = n_acc[r] drafted tokens of
// candidate k = best_k[r]; the target states of that block's slots 0..n
// (anchor + accepted tokens, from the target's verification pass) become the
// newest context rows, the context grows by n + 1 and the emitted token
// out_tok[r][n] is the next anchor.  Grid (R, B): CTA (r, j) copies slot j.
// ===========================================================================
__global__ void advance_kernel(int R, int K, int B, int64_t row_bytes,
                               const int32_t* __restrict__ n_acc,
                               const int32_t* __restrict__ best_k,
                               const int32_t* __restrict__ out_tok,
                               const uint8_t* __restrict__ verify_states,
                               int32_t* __restrict__ ctx_len, const int64_t* __restrict__ ctx_off,
                               uint8_t* __restrict__ new_states, int32_t* __restrict__ new_count,
                               int32_t* __restrict__ block_tokens, int32_t* __restrict__ known_len,
                               int mask_id, uint32_t* status) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int r = blockIdx.x, j = blockIdx.y;
  const int n = n_acc[r];
  const int k = best_k ? best_k[r] : 0;
  if (j <= n) {
    const uint4* src = reinterpret_cast<const uint4*>(
        verify_states + ((static_cast<int64_t>(r) * K + k) * B + j) * row_bytes);
    uint4* dst = reinterpret_cast<uint4*>(new_states + (static_cast<int64_t>(r) * B + j) * row_bytes);
    for (int64_t i = threadIdx.x; i < row_bytes / 16; i += blockDim.x) dst[i] = __ldg(src + i);
  }
  if (threadIdx.x == 0) {
    block_tokens[static_cast<int64_t>(r) * B + j] =
        j == 0 ? out_tok[static_cast<int64_t>(r) * B + n] : mask_id;
    if (j == 0) {
      const int64_t cap = ctx_off[r + 1] - ctx_off[r];
      int64_t L = static_cast<int64_t>(ctx_len[r]) + n + 1;
      if (L > cap) {   // the caller's capacity is exhausted: keep what fits
        report(status, DFLASH_EINVAL, 61);
        L = cap;
      }
      new_count[r] = static_cast<int32_t>(min(static_cast<int64_t>(n + 1), L - ctx_len[r]));
      ctx_len[r] = static_cast<int32_t>(L);
      known_len[r] = 1;
    }
  }
}

cudaError_t launch_advance(int R, int K, int B, int64_t row_bytes, const int32_t* n_acc,
                           const int32_t* best_k, const int32_t* out_tok, const void* verify_states,
                           int32_t* ctx_len, const int64_t* ctx_off, void* new_states,
                           int32_t* new_count, int32_t* block_tokens, int32_t* known_len,
                           int mask_id, uint32_t* status, cudaStream_t st) {
  if (R <= 0) return cudaSuccess;
  return launch_k(advance_kernel, dim3(R, B), dim3(256), 0, st, R, K, B, row_bytes, n_acc, best_k,
                  out_tok, static_cast<const uint8_t*>(verify_states), ctx_len, ctx_off,
                  static_cast<uint8_t*>(new_states), new_count, block_tokens, known_len, mask_id,
                  status);
}

// ===========================================================================
// Failure-detection self test: wait on a barrier that nothing completes.
// ===========================================================================
__global__ void wait_selftest_kernel(uint32_t* status, int64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  pdl_wait();
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, status, 99, static_cast<uint64_t>(limit_ns));
  __syncthreads();
}

cudaError_t launch_wait_selftest(uint32_t* status, int64_t limit_ns, cudaStream_t st) {
  return launch_k(wait_selftest_kernel, dim3(1), dim3(32), 0, st, status, limit_ns);
}

}  // namespace dfl
