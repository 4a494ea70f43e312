// Persistent weight-streaming "layer chain" for small token counts (bf16,
// M <= 64 block rows).
//
// Between two attentions a draft layer is a chain of weight-streaming GEMMs
// whose only coupling is through small activations:
//
//   O (h += attn W_o^T) -> RMSNorm_mlp -> gate/up (act = silu(g) * u)
//     -> down (h += act W_down^T) -> RMSNorm_attn of the next layer
//     -> next layer's Q / K^d / V^d (RoPE)            [or the final RMSNorm]
//
// Launched once per layer, one CTA per SM, this kernel streams every weight
// byte of the chain.  Each GEMM is a "stage" cut stream-K style into equal
// contiguous shares of (128-row weight tile x 64-wide k-block) units, one
// share per CTA, so every SM streams the same number of bytes per stage.
//
//   warp 0 lane 0 : weight producer -- TMA of the CTA's weight tiles of ALL
//                   stages in order, gated only by ring space, so the next
//                   GEMM's weights stream while the current one finishes;
//   warp 1 lane 0 : activation producer -- TMA of the [BN tokens x 64] input
//                   tiles, stage s only after stage s's input is complete
//                   (a device flag, bounded wait);
//   warp 2 lane 0 : tcgen05.mma issuer (TMEM accumulator, double-buffered);
//   warps 3..6    : epilogue -- TMEM -> registers; a tile shared by several
//                   CTAs is summed by its last contributor from fp32 partial
//                   slots in CTA order (deterministic), then the stage's op
//                   (residual add / SwiGLU / RoPE store) runs.  The CTA that
//                   completes a stage's last tile runs the RMSNorm that the
//                   next stage reads (if any) and releases the next stage.
//
// The flags are per launch (zeroed with the step's scratch words), counters
// are re-armed by whoever consumes them, and every wait is bounded: on
// timeout the kernel records DFLASH_ETIMEOUT and winds down.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dfl {
namespace chain {

constexpr int BM = 128;          // weight rows per tile (UMMA M)
constexpr int BK = 64;           // k per unit: one 128-byte swizzle row of bf16
constexpr int UK = 16;           // k per tcgen05.mma
constexpr int W_BYTES = BM * BK * 2;
constexpr int SROW = BM + 4;     // fp32 staging row
constexpr int EPI = 128;         // epilogue threads
constexpr int THREADS = 96 + EPI;

struct Seg {
  int tile_begin;    // first weight tile of the segment within its stage
  int map;           // weight tensor map (a SwiGLU pair uses map and map + 1)
  int rows;          // output features
  int pair;          // SwiGLU: 64 gate rows over the same 64 up rows per tile
  int op;            // EPI_STORE (optionally RoPE) / EPI_RESID / EPI_SWIGLU
  int rope;
  int64_t out_stride;
  void* out;
};

struct Stage {
  Seg seg[3];
  int nseg;
  int map_x;         // activation tensor map [M][K]
  int kbt;           // k-blocks
  int tiles;         // weight tiles
  int max_slots;     // partial slots reserved per tile
  float* partial;    // [tiles][max_slots][BN][BM]
  uint32_t* counters;   // [tiles], zero between uses
  const float* norm_g;  // after the stage: x = RMSNorm_{norm_g}(h) (nullptr: none)
};

constexpr int kMaxStages = kChainMaxStages;
constexpr int kMaxMaps = 12;

struct Params {
  CUtensorMap tm[kMaxMaps];
  int nmaps;
  Stage st[kMaxStages];
  int nst;
  int M;
  int grid;
  uint32_t* done;     // [nst] completed tiles per stage (zero at launch)
  uint32_t* ready;    // [nst] stage input complete (stage 0: at launch)
  float* h;           // residual stream [M][H] fp32
  int H;
  float eps;
  __nv_bfloat16* x;   // normed rows [M][H] written by the stage post-norm
  const int32_t* pos;      // RoPE positions [M]
  const float2* rope_tab;  // (cos, sin) [rope_len][head_dim / 2]
  int rope_len;
  int head_dim;
  uint32_t* status;
};

__device__ __forceinline__ int64_t u_begin(int64_t units, int grid, int c) {
  return (static_cast<int64_t>(c) * units) / grid;
}
__device__ __forceinline__ int cta_of(int64_t units, int grid, int64_t u) {
  return static_cast<int>(((u + 1) * grid - 1) / units);
}
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void mbar_arrive_local(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// TMA reads of data other CTAs wrote with ordinary stores
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ float2 rope_cs(const Params& p, int pos, int fi) {
  if (p.rope_tab != nullptr && pos < p.rope_len)
    return __ldg(p.rope_tab + static_cast<size_t>(pos) * (p.head_dim >> 1) + fi);
  return make_float2(1.f, 0.f);   // the host guarantees the table covers every position
}

template <int BN, int WST, int XST>
__global__ void __launch_bounds__(THREADS, 1) chain_kernel(const __grid_constant__ Params p) {
  constexpr int X_BYTES = BN * BK * 2;
  constexpr uint32_t ACC_COLS = BN < 32 ? 32 : BN;
  constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
  constexpr uint32_t IDESC = idesc_bf16(BM, BN);
  static_assert(W_BYTES % 1024 == 0 && X_BYTES % 1024 == 0, "1024-byte aligned ring stages");

  extern __shared__ uint8_t dsm[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm) + 1023) & ~uintptr_t(1023));
  uint8_t* wring = smem;                            // [WST][128 x 64]
  uint8_t* xring = smem + WST * W_BYTES;            // [XST][BN x 64]
  float* stg = reinterpret_cast<float*>(xring + XST * X_BYTES);   // [BN][SROW]
  __shared__ __align__(8) uint64_t wfull[WST], wempty[WST], xfull[XST], xempty[XST];
  __shared__ __align__(8) uint64_t accf[2], acce[2];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ int s_last, s_post;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = p.grid;
  const int c = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < WST; ++i) {
      mbar_init(&wfull[i], 1);
      mbar_init(&wempty[i], 1);
    }
    for (int i = 0; i < XST; ++i) {
      mbar_init(&xfull[i], 1);
      mbar_init(&xempty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf[b], 1);
      mbar_init(&acce[b], EPI);
    }
    abort_flag = 0;
    fence_mbar_init();
    for (int i = 0; i < p.nmaps; ++i) tma_prefetch_desc(&p.tm[i]);
  }
  if (warp == 3) tmem_alloc(&tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (threadIdx.x == 0) pdl_launch();

  auto seg_of = [&](const Stage& S, int tile) {
    int sg = 0;
    while (sg + 1 < S.nseg && tile >= S.seg[sg + 1].tile_begin) ++sg;
    return sg;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- weight producer (all stages, never gated by data)
      const uint64_t pol = policy_evict_first();   // every weight byte is read once
      int s = 0;
      uint32_t ph = 0;
      bool first = true;
      for (int si = 0; si < p.nst && !abort_flag; ++si) {
        const Stage& S = p.st[si];
        const int64_t units = static_cast<int64_t>(S.tiles) * S.kbt;
        const int64_t u0 = u_begin(units, G, c), u1 = u_begin(units, G, c + 1);
        int tile = static_cast<int>(u0 / S.kbt), k = static_cast<int>(u0 % S.kbt);
        for (int64_t u = u0; u < u1; ++u) {
          if (!mbar_wait(&wempty[s], ph ^ 1, p.status, 81)) {
            abort_flag = 1;
            break;
          }
          const Seg& g = S.seg[seg_of(S, tile)];
          const int row0 = (tile - g.tile_begin) * (g.pair ? BM / 2 : BM);
          uint8_t* dst = wring + s * W_BYTES;
          mbar_arrive_expect_tx(&wfull[s], W_BYTES);
          tma_load_2d_hint(dst, &p.tm[g.map], &wfull[s], k * BK, row0, pol);
          if (g.pair)
            tma_load_2d_hint(dst + W_BYTES / 2, &p.tm[g.map + 1], &wfull[s], k * BK, row0, pol);
          if (++k == S.kbt) {
            k = 0;
            ++tile;
          }
          if (++s == WST) {
            s = 0;
            ph ^= 1;
          }
          first = false;
        }
      }
      (void)first;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- activation producer: stage s after its input is ready
      pdl_wait();
      int s = 0;
      uint32_t ph = 0;
      for (int si = 0; si < p.nst && !abort_flag; ++si) {
        const Stage& S = p.st[si];
        const int64_t units = static_cast<int64_t>(S.tiles) * S.kbt;
        const int64_t u0 = u_begin(units, G, c), u1 = u_begin(units, G, c + 1);
        if (u0 == u1) continue;
        if (si > 0) {
          const uint64_t t0 = globaltimer_ns();
          uint32_t it = 0;
          while (ld_acquire(p.ready + si) == 0u) {
            __nanosleep(32);
            if ((++it & 63u) == 0u && globaltimer_ns() - t0 > kWaitLimitNs) {
              report(p.status, DFLASH_ETIMEOUT, 82);
              abort_flag = 1;
              break;
            }
          }
          if (abort_flag) break;
          fence_proxy_async_global();
        }
        int k = static_cast<int>(u0 % S.kbt);
        for (int64_t u = u0; u < u1; ++u) {
          if (!mbar_wait(&xempty[s], ph ^ 1, p.status, 83)) {
            abort_flag = 1;
            break;
          }
          mbar_arrive_expect_tx(&xfull[s], X_BYTES);
          tma_load_2d(xring + s * X_BYTES, &p.tm[S.map_x], &xfull[s], k * BK, 0);
          if (++k == S.kbt) k = 0;
          if (++s == XST) {
            s = 0;
            ph ^= 1;
          }
        }
      }
    }
  } else if (warp == 2) {
    if (lane == 0) {
      // ---------------- MMA issuer: one accumulator buffer per tile run
      int ws = 0, xs = 0, seg_i = 0;
      uint32_t wph = 0, xph = 0;
      for (int si = 0; si < p.nst; ++si) {
        const Stage& S = p.st[si];
        const int64_t units = static_cast<int64_t>(S.tiles) * S.kbt;
        const int64_t u0 = u_begin(units, G, c), u1 = u_begin(units, G, c + 1);
        int k = static_cast<int>(u0 % S.kbt);
        for (int64_t u = u0; u < u1; ++u, ++k) {
          if (k == S.kbt) k = 0;
          const bool first = (u == u0) || (k == 0);
          const bool last = (u == u1 - 1) || (k == S.kbt - 1);
          const int b = seg_i & 1;
          if (first && seg_i >= 2 && !abort_flag &&
              !mbar_wait(&acce[b], ((seg_i >> 1) - 1) & 1, p.status, 84))
            abort_flag = 1;
          if (!abort_flag && !mbar_wait(&wfull[ws], wph, p.status, 85)) abort_flag = 1;
          if (!abort_flag && !mbar_wait(&xfull[xs], xph, p.status, 86)) abort_flag = 1;
          if (!abort_flag) {
            tc_fence_after();
            const uint64_t da = smem_desc_sw128(wring + ws * W_BYTES);
            const uint64_t db = smem_desc_sw128(xring + xs * X_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / UK; ++kk)
              tc_mma_bf16(tmem + b * ACC_COLS, da + 2 * kk, db + 2 * kk, IDESC,
                          (first && kk == 0) ? 0u : 1u);
            tc_commit(&wempty[ws]);
            tc_commit(&xempty[xs]);
          }
          if (++ws == WST) {
            ws = 0;
            wph ^= 1;
          }
          if (++xs == XST) {
            xs = 0;
            xph ^= 1;
          }
          if (last) {
            tc_commit(&accf[b]);   // arrives after an abort too, so nobody waits long
            ++seg_i;
          }
        }
      }
    }
  } else {
    // ---------------- epilogue warps 3..6: tile row = TMEM lane
    const int et = threadIdx.x - 96;                 // 0..127
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;               // row within the weight tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    pdl_wait();
    int seg_i = 0;
    for (int si = 0; si < p.nst; ++si) {
      const Stage& S = p.st[si];
      const int64_t units = static_cast<int64_t>(S.tiles) * S.kbt;
      const int64_t u1 = u_begin(units, G, c + 1);
      int64_t u = u_begin(units, G, c);
      while (u < u1) {
        const int tile = static_cast<int>(u / S.kbt);
        const int kb_begin = static_cast<int>(u % S.kbt);
        const int64_t left = u1 - u;
        const int seg_len = static_cast<int>(left < S.kbt - kb_begin ? left : S.kbt - kb_begin);
        u += seg_len;
        const int b = seg_i & 1;
        const bool ok = mbar_wait(&accf[b], (seg_i >> 1) & 1, p.status, 87);
        tc_fence_after();
        float v[BN];
#pragma unroll
        for (int cc = 0; cc < BN; cc += 16) tmem_ld16(lane_addr + b * ACC_COLS + cc, v + cc);
        tc_fence_before();
        mbar_arrive_local(&acce[b]);
        ++seg_i;
        const bool live = ok && !abort_flag;
        const Seg& g = S.seg[seg_of(S, tile)];
        const int row0 = (tile - g.tile_begin) * (g.pair ? BM / 2 : BM);
        const int c_lo = cta_of(units, G, static_cast<int64_t>(tile) * S.kbt);
        const int c_hi = cta_of(units, G, static_cast<int64_t>(tile + 1) * S.kbt - 1);
        bool do_op = live;
        if (c_hi > c_lo) {
          float* slots = S.partial + static_cast<size_t>(tile) * S.max_slots * BN * BM;
          float* mine = slots + static_cast<size_t>(c - c_lo) * BN * BM;
          if (live) {
#pragma unroll
            for (int j = 0; j < BN; ++j) __stcg(mine + j * BM + r, v[j]);
            __threadfence();
          }
          named_sync(1, EPI);
          if (et == 0) {
            const uint32_t prev = live ? atomicAdd(S.counters + tile, 1u) : 0u;
            s_last = live && prev == static_cast<uint32_t>(c_hi - c_lo);
          }
          named_sync(1, EPI);
          do_op = s_last != 0;
          if (do_op) {
            __threadfence();
            const int nsl = c_hi - c_lo + 1;
            constexpr int ITEMS = BN * (BM / 4);
#pragma unroll 1
            for (int it0 = 0; it0 < ITEMS; it0 += 4 * EPI) {
              float4 acc[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
              for (int sl = 0; sl < nsl; ++sl) {
                const float4* src =
                    reinterpret_cast<const float4*>(slots + static_cast<size_t>(sl) * BN * BM);
                float4 a[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  const int it = it0 + q * EPI + et;
                  a[q] = it < ITEMS ? __ldcg(src + it) : make_float4(0.f, 0.f, 0.f, 0.f);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  acc[q].x += a[q].x; acc[q].y += a[q].y; acc[q].z += a[q].z; acc[q].w += a[q].w;
                }
              }
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int it = it0 + q * EPI + et;
                if (it < ITEMS) {
                  const int j = it / (BM / 4), rq = (it % (BM / 4)) * 4;
                  *reinterpret_cast<float4*>(stg + j * SROW + rq) = acc[q];
                }
              }
            }
            if (et == 0) S.counters[tile] = 0u;
          }
        } else if (do_op) {
#pragma unroll
          for (int j = 0; j < BN; ++j) stg[j * SROW + r] = v[j];
        }
        named_sync(1, EPI);
        if (do_op) {
          if (g.op == EPI_SWIGLU) {
            const int rr = et & 63;
            const int f = row0 + rr;
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(g.out);
#pragma unroll 4
            for (int j = et >> 6; j < BN; j += 2) {
              if (f < g.rows && j < p.M) {
                const float gt = stg[j * SROW + rr], up = stg[j * SROW + rr + 64];
                o[static_cast<int64_t>(j) * g.out_stride + f] =
                    __float2bfloat16_rn(gt / (1.f + __expf(-gt)) * up);
              }
            }
          } else if (g.op == EPI_RESID) {
            // all of the column's residual loads first, then the adds
            const int f = row0 + et;
            float* hp = static_cast<float*>(g.out) + f;
            const bool fv = f < g.rows;
            float hv[BN];
#pragma unroll
            for (int j = 0; j < BN; ++j)
              hv[j] = (fv && j < p.M) ? __ldcg(hp + static_cast<int64_t>(j) * g.out_stride) : 0.f;
#pragma unroll
            for (int j = 0; j < BN; ++j)
              if (fv && j < p.M) hp[static_cast<int64_t>(j) * g.out_stride] = hv[j] + stg[j * SROW + et];
          } else {
            const int f = row0 + et;
            const int half = p.head_dim >> 1;
            const int i = et % p.head_dim;
            const int prt = i < half ? et + half : et - half;
            const int fi = i < half ? i : i - half;
            __nv_bfloat16* o = static_cast<__nv_bfloat16*>(g.out);
            // 16 tokens at a time: their positions, then their (cos, sin),
            // each as one batch of independent loads
#pragma unroll 1
            for (int j0 = 0; j0 < BN; j0 += 16) {
              float2 cs[16];
              if (g.rope) {
                int ps[16];
#pragma unroll
                for (int q = 0; q < 16; ++q) ps[q] = __ldg(p.pos + min(j0 + q, p.M - 1));
#pragma unroll
                for (int q = 0; q < 16; ++q) cs[q] = rope_cs(p, ps[q], fi);
              }
#pragma unroll
              for (int q = 0; q < 16; ++q) {
                const int j = j0 + q;
                if (f >= g.rows || j >= p.M) continue;
                float xv = stg[j * SROW + et];
                if (g.rope) {
                  const float pv = stg[j * SROW + prt];
                  xv = i < half ? xv * cs[q].x - pv * cs[q].y : xv * cs[q].x + pv * cs[q].y;
                }
                o[static_cast<int64_t>(j) * g.out_stride + f] = __float2bfloat16_rn(xv);
              }
            }
          }
          // the next stage reads these outputs through TMA (async proxy)
          fence_proxy_async_global();
        }
        // stage bookkeeping: the tile is final; the CTA that completes the
        // stage runs its post-norm and releases the next stage
        named_sync(1, EPI);
        if (et == 0) {
          s_post = 0;
          if (do_op) {
            __threadfence();
            const uint32_t prev = atomicAdd(p.done + si, 1u);
            s_post = prev == static_cast<uint32_t>(S.tiles - 1);
          }
        }
        named_sync(1, EPI);
        if (s_post) {
          __threadfence();
          if (S.norm_g != nullptr) {
            // x[m] = h[m] / sqrt(mean(h[m]^2) + eps) * g: one warp per row,
            // float4 loads (the row is read twice, from L2)
            const int nv = p.H >> 2;
            const float4* g4 = reinterpret_cast<const float4*>(S.norm_g);
            for (int m = et >> 5; m < p.M; m += EPI / 32) {
              const float4* hr = reinterpret_cast<const float4*>(p.h + static_cast<int64_t>(m) * p.H);
              float ss = 0.f;
#pragma unroll 4
              for (int e = lane; e < nv; e += 32) {
                const float4 hv = __ldcg(hr + e);
                ss = fmaf(hv.x, hv.x, fmaf(hv.y, hv.y, fmaf(hv.z, hv.z, fmaf(hv.w, hv.w, ss))));
              }
              ss = warp_sum(ss);
              const float sc = rsqrtf(ss / static_cast<float>(p.H) + p.eps);
              uint2* xr = reinterpret_cast<uint2*>(p.x + static_cast<int64_t>(m) * p.H);
#pragma unroll 4
              for (int e = lane; e < nv; e += 32) {
                const float4 hv = __ldcg(hr + e);
                const float4 gv = __ldg(g4 + e);
                __nv_bfloat162 lo = __floats2bfloat162_rn(hv.x * sc * gv.x, hv.y * sc * gv.y);
                __nv_bfloat162 hi = __floats2bfloat162_rn(hv.z * sc * gv.z, hv.w * sc * gv.w);
                uint2 pk;
                pk.x = *reinterpret_cast<uint32_t*>(&lo);
                pk.y = *reinterpret_cast<uint32_t*>(&hi);
                xr[e] = pk;
              }
            }
            fence_proxy_async_global();
            named_sync(1, EPI);
          }
          if (et == 0) {
            __threadfence();
            if (si + 1 < p.nst) st_release(p.ready + si + 1, 1u);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 3) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace chain

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
namespace {

template <int BN, int WST, int XST>
constexpr int chain_smem() {
  return WST * chain::W_BYTES + XST * BN * chain::BK * 2 + BN * chain::SROW * 4 + 1024;
}

template <int BN, int WST, int XST>
cudaError_t chain_go(const chain::Params& p, cudaStream_t st) {
  constexpr int SMEM = chain_smem<BN, WST, XST>();
  static std::once_flag once;
  static cudaError_t attr = cudaSuccess;
  std::call_once(once, [] {
    attr = cudaFuncSetAttribute(chain::chain_kernel<BN, WST, XST>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  });
  if (attr != cudaSuccess) return attr;
  return launch_k(chain::chain_kernel<BN, WST, XST>, dim3(p.grid), dim3(chain::THREADS), SMEM,
                  st, p);
}

int cdiv(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

}  // namespace

int chain_bn(int64_t M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 0; }

// Partial slots and counters the chain stages need (floats, words).
static int stage_tiles(const ChainStageJob& sj) {
  int tiles = 0;
  for (int g = 0; g < sj.nseg; ++g)
    tiles += sj.seg[g].op == EPI_SWIGLU ? cdiv(sj.seg[g].rows, chain::BM / 2)
                                        : cdiv(sj.seg[g].rows, chain::BM);
  return tiles;
}

// one CTA per SM, never more CTAs than the smallest stage has units
static int chain_grid(const ChainJob& job) {
  int64_t mu = kNumSMs;
  for (int s = 0; s < job.nst; ++s)
    mu = std::min<int64_t>(mu, static_cast<int64_t>(stage_tiles(job.st[s])) *
                                   cdiv(job.st[s].K, chain::BK));
  return static_cast<int>(std::max<int64_t>(1, mu));
}

void chain_needs(const ChainJob& job, size_t* partial_floats, size_t* counters) {
  const int bn = chain_bn(job.M);
  const int G = chain_grid(job);
  size_t pf = 0, cn = 0;
  for (int s = 0; s < job.nst; ++s) {
    const ChainStageJob& sj = job.st[s];
    const int tiles = stage_tiles(sj);
    const int kbt = cdiv(sj.K, chain::BK);
    const int64_t units = static_cast<int64_t>(tiles) * kbt;
    int slots = 1;
    for (int t = 0; t < tiles; ++t) {
      auto cta = [&](int64_t u) { return static_cast<int>(((u + 1) * G - 1) / units); };
      slots = std::max(slots, cta(static_cast<int64_t>(t + 1) * kbt - 1) -
                                  cta(static_cast<int64_t>(t) * kbt) + 1);
    }
    pf += static_cast<size_t>(tiles) * slots * bn * chain::BM;
    cn += tiles;
  }
  *partial_floats = pf;
  *counters = cn;
}

cudaError_t launch_chain(const ChainJob& job, float* partial, uint32_t* counters,
                         uint32_t* flags, uint32_t* status, cudaStream_t st) {
  const int bn = chain_bn(job.M);
  if (bn == 0 || job.nst < 1 || job.nst > chain::kMaxStages) return cudaErrorInvalidValue;
  chain::Params p{};
  int maps = 0;
  int64_t min_units = INT64_MAX;
  for (int s = 0; s < job.nst; ++s) {
    const ChainStageJob& sj = job.st[s];
    chain::Stage& S = p.st[s];
    int tiles = 0;
    for (int g = 0; g < sj.nseg; ++g) {
      const GemmOut& o = sj.seg[g];
      chain::Seg& G = S.seg[g];
      G.tile_begin = tiles;
      G.map = maps;
      G.rows = o.rows;
      G.pair = o.op == EPI_SWIGLU;
      G.op = o.op;
      G.rope = o.rope;
      G.out_stride = o.out_stride;
      G.out = o.out;
      const int box = G.pair ? chain::BM / 2 : chain::BM;
      if (maps + (G.pair ? 2 : 1) > chain::kMaxMaps) return cudaErrorInvalidValue;
      if (!encode_tmap_bf16_2d(&p.tm[maps++], o.w0, sj.K, o.rows, chain::BK, box))
        return cudaErrorInvalidValue;
      if (G.pair && !encode_tmap_bf16_2d(&p.tm[maps++], o.w1, sj.K, o.rows, chain::BK, box))
        return cudaErrorInvalidValue;
      tiles += cdiv(o.rows, box);
    }
    if (maps + 1 > chain::kMaxMaps) return cudaErrorInvalidValue;
    S.map_x = maps;
    if (!encode_tmap_bf16_2d(&p.tm[maps++], sj.x, sj.K, job.M, chain::BK, bn))
      return cudaErrorInvalidValue;
    S.nseg = sj.nseg;
    S.kbt = cdiv(sj.K, chain::BK);
    S.tiles = tiles;
    S.norm_g = sj.norm_g;
    min_units = std::min<int64_t>(min_units, static_cast<int64_t>(tiles) * S.kbt);
  }
  p.nmaps = maps;
  p.nst = job.nst;
  p.M = static_cast<int>(job.M);
  p.grid = chain_grid(job);
  (void)min_units;
  // partial slots per stage (same geometry as chain_needs, with this grid)
  size_t off = 0, coff = 0;
  for (int s = 0; s < job.nst; ++s) {
    chain::Stage& S = p.st[s];
    const int64_t units = static_cast<int64_t>(S.tiles) * S.kbt;
    int slots = 1;
    for (int t = 0; t < S.tiles; ++t) {
      auto cta = [&](int64_t u) { return static_cast<int>(((u + 1) * p.grid - 1) / units); };
      slots = std::max(slots, cta(static_cast<int64_t>(t + 1) * S.kbt - 1) -
                                  cta(static_cast<int64_t>(t) * S.kbt) + 1);
    }
    S.max_slots = slots;
    S.partial = partial + off;
    S.counters = counters + coff;
    off += static_cast<size_t>(S.tiles) * slots * bn * chain::BM;
    coff += S.tiles;
  }
  p.done = flags;
  p.ready = flags + chain::kMaxStages;
  p.h = job.h;
  p.H = job.H;
  p.eps = job.eps;
  p.x = static_cast<__nv_bfloat16*>(job.x_out);
  p.pos = job.pos;
  p.rope_tab = job.rope_tab;
  p.rope_len = job.rope_len;
  p.head_dim = job.head_dim;
  p.status = status;
  switch (bn) {
    case 16: return chain_go<16, 10, 8>(p, st);
    case 32: return chain_go<32, 10, 8>(p, st);
    default: return chain_go<64, 8, 8>(p, st);
  }
}

}  // namespace dfl
