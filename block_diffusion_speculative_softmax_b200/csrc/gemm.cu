// Weight-streaming GEMMs of the draft step.
//
// Every dense contraction of the draft (Q / K / V / O projections, the
// SwiGLU MLP and the LM head) has the form  Y[m][r] = sum_k X[m][k] W[r][k]
// with W an [out][in] weight matrix and X a handful of token rows (16 at
// batch 1, 512 when 32 blocks are drafted together, up to ~150k context
// rows for the context K/V projection).  The bf16 path puts the WEIGHT rows
// on the tensor core's M dimension (128 rows per tile) and the tokens on N
// (16..256), so one CTA streams a 128-row weight panel through a TMA ->
// shared-memory ring and accumulates in TMEM with tcgen05.mma:
//
//   warp 0 lane 0 : TMA producer (weight tile + token tile per stage)
//   warp 1 lane 0 : tcgen05.mma issuer, commits each stage back to the ring
//   warp 2        : TMEM allocation / release
//   warps 0-3     : epilogue, one TMEM lane (= one tile row) per thread
//
// The epilogue is fused: the accumulator tile is staged in shared memory
// (the drained pipeline ring) and the segment's op is applied there --
// RoPE (pairs i, i + d/2 of a head live in the same tile), scatter into a
// KV cache, residual add, or SwiGLU (a SwiGLU tile stacks 64 rows of W_gate
// over the same 64 rows of W_up, so silu(g) * u is formed inside one CTA).
// With split-K every split writes its fp32 partial tile and the LAST CTA to
// arrive at the tile's counter sums the splits in fixed order (so results
// are deterministic), applies the op and re-arms the counter.
//
// Kernels are launched with programmatic dependent launch: the producer
// streams the first ring stages of WEIGHTS (which no earlier kernel writes)
// before griddepcontrol.wait, so a GEMM's pipeline fill overlaps the tail of
// the kernel before it; activations, partials, counters and outputs are
// only touched after the wait.
//
// The LM-head variant keeps a per-CTA (max, index) per token and merges it
// with one 64-bit atomicMax, so logits never reach global memory.  fp32
// models run on a SIMT FFMA kernel (partials + finish kernel): tensor-core
// tf32 would miss a 1e-4 tolerance.
//
// Three bf16 kernels share this structure:
//   gemm_kernel     weight-major split-K (above), block GEMMs with <= 64 tokens;
//   gemm_sk_kernel  weight-major stream-K: a persistent grid whose CTAs take
//                   equal shares of the (tile, k-block) units, used for the
//                   LM head with <= 64 tokens;
//   gemm_tok_kernel token-major (tokens on M, features on N) for >= 65 tokens,
//                   on CTA pairs (cta_group::2) when tiles are plentiful.
#include <algorithm>
#include <cstdlib>
#include <cmath>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dfl {

namespace {
int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }
}  // namespace

// ===========================================================================
// tcgen05 kernel
// ===========================================================================
namespace tc {

constexpr int BM = 128;          // tile rows (UMMA M)
constexpr int BK = 64;           // bf16 per k-block: one 128-byte swizzle row
constexpr int UK = 16;           // K per tcgen05.mma (kind::f16)
constexpr int A_BYTES = BM * BK * 2;
constexpr int SROW = BM + 4;     // fp32 staging row (tokens x tile rows)

struct Seg {
  int tile_begin;     // first row tile of the segment
  int map;            // index of its (first) weight tensor map
  int rows;           // output features
  int pair;           // SwiGLU pair: 64 features per tile (gate rows over up rows)
  int op;
  int rope;
  int use_dst;
  int64_t out_stride;
  void* out;
};

struct Params {
  CUtensorMap tm[4];                // weights (a SwiGLU pair uses two maps)
  CUtensorMap tm_x;                 // activations [M][K]
  Seg seg[kMaxSegs];
  int nseg;
  int M;
  int kb_total;
  int kb_per_split;
  int splits;
  int row_tiles;
  int tok_fast;                     // token-major grid: token tiles on x (weight tile shared
                                    // by the CTAs that run together), else feature tiles on x
  float* partial;                   // [tiles][splits][BN][BM]
  uint32_t* counters;               // [tiles]
  const int32_t* pos;
  const int64_t* dst;
  int head_dim;
  const float2* rope_tab;           // (cos, sin) [rope_len][head_dim / 2] or null
  int rope_len;
  double inv_freq[64];
  const float* rss;                 // [M][rss_parts] row sums of squares, or null
  int rss_parts;
  float rss_inv;                    // 1 / hidden
  float rss_eps;
  unsigned long long* keys;         // argmax mode: [M]
  float2* lse;                      // argmax mode: per (vocab tile, token) (max, sum exp)
  uint32_t* status;
};

// cos / sin of pos * inv_freq[fi]: from the step's table when the position
// is inside it, else computed (angle reduced mod 2 pi in double first).
__device__ __forceinline__ float2 rope_cs(const Params& p, int pos, int fi) {
  if (p.rope_tab != nullptr && pos < p.rope_len)
    return __ldg(p.rope_tab + static_cast<size_t>(pos) * (p.head_dim >> 1) + fi);
  double ang = static_cast<double>(pos) * p.inv_freq[fi];
  ang -= 6.283185307179586 * rint(ang * 0.15915494309189535);
  float sn, cs;
  sincosf(static_cast<float>(ang), &sn, &cs);
  return make_float2(cs, sn);
}

// RMSNorm scale of token row t when the input rows arrive unnormalised:
// rsqrt(sum of the row's partial sums of squares / hidden + eps), the parts
// added in a fixed order; 1 without one.
__device__ __forceinline__ float rss_scale(const Params& p, int t) {
  if (p.rss == nullptr) return 1.f;
  const float* r = p.rss + static_cast<size_t>(t) * p.rss_parts;
  float s = 0.f;
  for (int w = 0; w < p.rss_parts; ++w) s += __ldg(r + w);
  return rsqrtf(s * p.rss_inv + p.rss_eps);
}

// (cos, sin) of frequencies i0 .. i0 + 15 at `pos`: eight 16-byte table loads
// when the table covers the position (i0 is a multiple of 16).
__device__ __forceinline__ void rope_cs16(const Params& p, int pos, int i0, float2* cs) {
  if (p.rope_tab != nullptr && pos < p.rope_len) {
    const float4* t = reinterpret_cast<const float4*>(
        p.rope_tab + static_cast<size_t>(pos) * (p.head_dim >> 1) + i0);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 v = __ldg(t + q);
      cs[2 * q] = make_float2(v.x, v.y);
      cs[2 * q + 1] = make_float2(v.z, v.w);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 16; ++q) cs[q] = rope_cs(p, pos, i0 + q);
  }
}

template <int BN, int STAGES, bool ARGMAX>
__global__ void __launch_bounds__(128, 1) gemm_kernel(const __grid_constant__ Params p) {
  constexpr int B_BYTES = BN * BK * 2;
  constexpr int STAGE = A_BYTES + B_BYTES;
  constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;
  constexpr uint32_t IDESC = idesc_bf16(BM, BN);
  static_assert(STAGE % 1024 == 0, "stages must stay 1024-byte aligned");
  static_assert(ARGMAX || BN * SROW * 4 <= STAGES * STAGE, "staging tile must fit the ring");

  extern __shared__ uint8_t dsmem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ int s_last;
  __shared__ unsigned long long red[ARGMAX ? 4 : 1][ARGMAX ? BN : 1];
  __shared__ float2 red2[ARGMAX ? 4 : 1][ARGMAX ? BN : 1];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x;

  // Which segment this row tile belongs to.
  const int tile = blockIdx.x;
  int sg = 0;
  while (sg + 1 < p.nseg && tile >= p.seg[sg + 1].tile_begin) ++sg;
  const Seg& S = p.seg[sg];
  const int pair = S.pair;
  const int row0 = (tile - S.tile_begin) * (pair ? BM / 2 : BM);   // first output feature
  const int tok0 = blockIdx.y * BN;
  const int kb0 = blockIdx.z * p.kb_per_split;
  const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
  const int nkb = kb1 - kb0;
  const CUtensorMap* tma = &p.tm[S.map];
  const CUtensorMap* tmb = pair ? &p.tm[S.map + 1] : nullptr;

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(tma);
    if (tmb) tma_prefetch_desc(tmb);
    tma_prefetch_desc(&p.tm_x);
  }
  if (warp == 2) tmem_alloc(&tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (tid == 0) pdl_launch();

  // weights are read once per step: evict them first so L2 keeps what is
  // reused (activations, partial tiles, the K/V caches)
  const uint64_t pol = policy_evict_first();
  auto load_w = [&](int i, uint8_t* sa) {
    const int kc = (kb0 + i) * BK;
    if (pair) {
      tma_load_2d_hint(sa, tma, &full_bar[i % STAGES], kc, row0, pol);
      tma_load_2d_hint(sa + A_BYTES / 2, tmb, &full_bar[i % STAGES], kc, row0, pol);
    } else {
      tma_load_2d_hint(sa, tma, &full_bar[i % STAGES], kc, row0, pol);
    }
  };

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    // weights of the first stages before the dependency wait (no earlier
    // kernel writes weights), activations after it
    const int npre = min(STAGES, nkb);
    for (int i = 0; i < npre; ++i) {
      mbar_arrive_expect_tx(&full_bar[i], STAGE);
      load_w(i, smem + i * STAGE);
    }
    pdl_wait();
    for (int i = 0; i < npre; ++i)
      tma_load_2d(smem + i * STAGE + A_BYTES, &p.tm_x, &full_bar[i], (kb0 + i) * BK, tok0);
    int issued = npre;
    for (int i = npre; i < nkb; ++i) {
      const int s = i % STAGES;
      if (!mbar_wait(&empty_bar[s], ((i / STAGES) & 1) ^ 1, p.status, 11)) {
        abort_flag = 1;
        break;
      }
      if (abort_flag) break;
      uint8_t* sa = smem + s * STAGE;
      mbar_arrive_expect_tx(&full_bar[s], STAGE);
      load_w(i, sa);
      tma_load_2d(sa + A_BYTES, &p.tm_x, &full_bar[s], (kb0 + i) * BK, tok0);
      ++issued;
    }
    if (abort_flag) {
      // let the copies still in flight land before the CTA's smem goes away
      for (int i = max(0, issued - STAGES); i < issued; ++i)
        mbar_wait(&full_bar[i % STAGES], (i / STAGES) & 1, p.status, 12);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    for (int i = 0; i < nkb; ++i) {
      const int s = i % STAGES;
      if (!mbar_wait(&full_bar[s], (i / STAGES) & 1, p.status, 13)) {
        abort_flag = 1;
        break;
      }
      if (abort_flag) break;
      tc_fence_after();
      const uint8_t* sa = smem + s * STAGE;
      const uint64_t da = smem_desc_sw128(sa);
      const uint64_t db = smem_desc_sw128(sa + A_BYTES);
#pragma unroll
      for (int k = 0; k < BK / UK; ++k) {
        // advance 16 elements (32 bytes = 2 descriptor units) along K
        tc_mma_bf16(tmem, da + 2 * k, db + 2 * k, IDESC, (i > 0 || k > 0) ? 1u : 0u);
      }
      tc_commit(&empty_bar[s]);
    }
    tc_commit(&acc_bar);   // fires once every MMA above has completed
  }
  __syncwarp();

  // ---------------- epilogue
  const bool ok = mbar_wait(&acc_bar, 0, p.status, 14);
  tc_fence_after();
  pdl_wait();
  // warp-uniform: the tcgen05.ld below is a warp-wide instruction
  const bool live = __all_sync(0xffffffffu, ok && !abort_flag);
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);

  if constexpr (ARGMAX) {
    const int row = row0 + tid;
    if (live) {
#pragma unroll 1
      for (int c = 0; c < BN; c += 16) {
        float v[16];
        tmem_ld16(lane_addr + c, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          unsigned long long key = 0ull;
          if (row < S.rows && tok0 + c + j < p.M) {
            if (!isfinite(v[j])) report(p.status, DFLASH_ENUMERIC, 15);
            key = argmax_key(v[j], static_cast<uint32_t>(row));
          }
          key = warp_max_u64(key);
          if (lane == 0) red[warp][c + j] = key;
          if (p.lse != nullptr) {
            // this tile's share of the log-sum-exp of token c + j
            const bool in = row < S.rows;
            const float mx = warp_max(in ? v[j] : -INFINITY);
            const float se = warp_sum(in ? __expf(v[j] - mx) : 0.f);
            if (lane == 0) red2[warp][c + j] = make_float2(mx, se);
          }
        }
      }
    }
    __syncthreads();
    if (live) {
      for (int j = tid; j < BN; j += blockDim.x) {
        unsigned long long k = red[0][j];
#pragma unroll
        for (int w = 1; w < 4; ++w) k = red[w][j] > k ? red[w][j] : k;
        const int t = tok0 + j;
        if (t < p.M && k != 0ull) atomicMax(p.keys + t, k);
        if (t < p.M && p.lse != nullptr) {
          float mx = red2[0][j].x;
#pragma unroll
          for (int w = 1; w < 4; ++w) mx = fmaxf(mx, red2[w][j].x);
          float se = 0.f;
#pragma unroll
          for (int w = 0; w < 4; ++w)
            se += red2[w][j].y > 0.f ? red2[w][j].y * __expf(red2[w][j].x - mx) : 0.f;
          p.lse[static_cast<size_t>(blockIdx.x) * p.M + t] = make_float2(mx, se);
        }
      }
    }
  } else {
    float* st = reinterpret_cast<float*>(smem);        // staging [BN][SROW]
    const int tile_lin = blockIdx.y * p.row_tiles + blockIdx.x;
    bool do_op = live;
    if (live) {
      if (p.splits == 1) {
#pragma unroll 1
        for (int c = 0; c < BN; c += 16) {
          float v[16];
          tmem_ld16(lane_addr + c, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) st[(c + j) * SROW + tid] = v[j];
        }
      } else {
        float* mine = p.partial +
                      (static_cast<size_t>(tile_lin) * p.splits + blockIdx.z) * BN * BM;
#pragma unroll 1
        for (int c = 0; c < BN; c += 16) {
          float v[16];
          tmem_ld16(lane_addr + c, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) mine[(c + j) * BM + tid] = v[j];
        }
        __threadfence();
      }
    }
    if (p.splits > 1) {
      __syncthreads();
      if (tid == 0) {
        const uint32_t prev = live ? atomicAdd(p.counters + tile_lin, 1u) : 0u;
        s_last = live && prev == static_cast<uint32_t>(p.splits - 1);
      }
      __syncthreads();
      do_op = s_last != 0;
      if (do_op) {
        __threadfence();
        // the tile's BN x 128 floats as float4 items (token j, rows 4q..4q+3),
        // each summed over the splits in fixed order, straight into staging.
        // A thread owns 4 items and loads 8 splits of each at once (32 float4
        // in flight), so the reduction costs ceil(splits / 8) L2 round trips
        // per 4 items instead of one per split.
        const float4* base = reinterpret_cast<const float4*>(
            p.partial + static_cast<size_t>(tile_lin) * p.splits * BN * BM);
        constexpr int ITEMS = BN * (BM / 4);
        constexpr int NT = 128;
        constexpr int SB = 8;   // splits per batch of loads
#pragma unroll 1
        for (int it0 = 0; it0 < ITEMS; it0 += 4 * NT) {
          float4 acc[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
          for (int sp0 = 0; sp0 < p.splits; sp0 += SB) {
            float4 a[4][SB];
#pragma unroll
            for (int u = 0; u < SB; ++u)
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int it = it0 + q * NT + tid;
                a[q][u] = (it < ITEMS && sp0 + u < p.splits)
                              ? __ldcg(base + static_cast<size_t>(sp0 + u) * ITEMS + it)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
              }
#pragma unroll
            for (int u = 0; u < SB; ++u)
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                if (sp0 + u < p.splits) {
                  acc[q].x += a[q][u].x; acc[q].y += a[q][u].y;
                  acc[q].z += a[q][u].z; acc[q].w += a[q][u].w;
                }
              }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int it = it0 + q * NT + tid;
            if (it < ITEMS) {
              const int j = it / (BM / 4), rq = (it % (BM / 4)) * 4;
              *reinterpret_cast<float4*>(st + j * SROW + rq) = acc[q];
            }
          }
        }
        if (tid == 0) p.counters[tile_lin] = 0u;
      }
    }
    __syncthreads();
    if (do_op) {
      constexpr int JU = BN < 8 ? BN : 8;   // tokens per unrolled group
      if (S.op == EPI_SWIGLU) {
        const int r = tid & 63;
        const int f = row0 + r;
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(S.out);
#pragma unroll 4
        for (int j = tid >> 6; j < BN; j += 2) {
          const int t = tok0 + j;
          if (f < S.rows && t < p.M) {
            const float g = st[j * SROW + r], u = st[j * SROW + r + 64];
            o[static_cast<int64_t>(t) * S.out_stride + f] =
                __float2bfloat16_rn(g / (1.f + __expf(-g)) * u);
          }
        }
      } else if (S.op == EPI_RESID) {
        const int f = row0 + tid;
        float* h = static_cast<float*>(S.out) + f;
#pragma unroll 1
        for (int j0 = 0; j0 < BN; j0 += JU) {
          float hv[JU];
#pragma unroll
          for (int q = 0; q < JU; ++q) {
            const int t = tok0 + j0 + q;
            hv[q] = (f < S.rows && t < p.M) ? h[static_cast<int64_t>(t) * S.out_stride] : 0.f;
          }
#pragma unroll
          for (int q = 0; q < JU; ++q) {
            const int t = tok0 + j0 + q;
            if (f < S.rows && t < p.M)
              h[static_cast<int64_t>(t) * S.out_stride] = hv[q] + st[(j0 + q) * SROW + tid];
          }
        }
      } else {
        const int f = row0 + tid;
        const int half = p.head_dim >> 1;
        const int i = tid % p.head_dim;
        const int prt = i < half ? tid + half : tid - half;
        const int fi = i < half ? i : i - half;
        __nv_bfloat16* o = static_cast<__nv_bfloat16*>(S.out);
#pragma unroll 1
        for (int j0 = 0; j0 < BN; j0 += JU) {
          float2 cs[JU];
          int64_t orow[JU];
          float rs[JU];
#pragma unroll
          for (int q = 0; q < JU; ++q) {
            const int t = min(tok0 + j0 + q, p.M - 1);
            cs[q] = S.rope ? rope_cs(p, p.pos[t], fi) : make_float2(1.f, 0.f);
            orow[q] = S.use_dst ? p.dst[t] : t;
            rs[q] = rss_scale(p, t);
          }
#pragma unroll
          for (int q = 0; q < JU; ++q) {
            const int t = tok0 + j0 + q;
            if (f >= S.rows || t >= p.M || orow[q] < 0) continue;
            float v = st[(j0 + q) * SROW + tid];
            if (S.rope) {
              const float pv = st[(j0 + q) * SROW + prt];
              v = i < half ? v * cs[q].x - pv * cs[q].y : v * cs[q].x + pv * cs[q].y;
            }
            v *= rs[q];
            if (S.op == EPI_STORE_F32)
              static_cast<float*>(S.out)[orow[q] * S.out_stride + f] = v;
            else
              o[orow[q] * S.out_stride + f] = __float2bfloat16_rn(v);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Epilogue of one token row of a token-major tile: thread = token t (valid
// when tv), features f0 .. f0 + BW - 1 of segment S; cols(c, v) yields the
// accumulator columns [c, c + 16) of the row.  ARGMAX: argmax key (and the
// tile's log-sum-exp share); else the segment's op (SwiGLU halves, residual
// row, or a store with optional RoPE over heads and row scatter).
template <int BW, bool ARGMAX, typename ColsFn>
__device__ __forceinline__ void tok_row_epilogue(const Params& p, const Seg& S, int tile, int f0,
                                                 int t, bool tv, ColsFn&& cols) {
  if constexpr (ARGMAX) {
    unsigned long long best = 0ull;
    float mx = -INFINITY, se = 0.f;   // running log-sum-exp share of this tile
#pragma unroll 1
    for (int c = 0; c < BW; c += 16) {
      float v[16];
      cols(c, v);
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        const int f = f0 + c + q;
        if (f < S.rows) {
          if (!isfinite(v[q]) && tv) report(p.status, DFLASH_ENUMERIC, 35);
          const unsigned long long k = argmax_key(v[q], static_cast<uint32_t>(f));
          best = k > best ? k : best;
          if (v[q] > mx) {
            se = se * __expf(mx - v[q]) + 1.f;
            mx = v[q];
          } else {
            se += __expf(v[q] - mx);
          }
        }
      }
    }
    if (tv && best) atomicMax(p.keys + t, best);
    if (tv && p.lse != nullptr) p.lse[static_cast<size_t>(tile) * p.M + t] = make_float2(mx, se);
  } else if (S.op == EPI_SWIGLU) {
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(S.out) + static_cast<int64_t>(t) * S.out_stride;
#pragma unroll 1
    for (int c = 0; c < BW / 2; c += 16) {
      float g[16], u[16];
      cols(c, g);
      cols(BW / 2 + c, u);
      if (tv) {
        alignas(16) __nv_bfloat16 r[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) r[q] = __float2bfloat16_rn(g[q] / (1.f + __expf(-g[q])) * u[q]);
        const int f = f0 + c;
        if (f + 16 <= S.rows) {
          reinterpret_cast<uint4*>(o + f)[0] = reinterpret_cast<const uint4*>(r)[0];
          reinterpret_cast<uint4*>(o + f)[1] = reinterpret_cast<const uint4*>(r)[1];
        } else {
          for (int q = 0; q < 16 && f + q < S.rows; ++q) o[f + q] = r[q];
        }
      }
    }
  } else if (S.op == EPI_RESID) {
    float* h = static_cast<float*>(S.out) + static_cast<int64_t>(t) * S.out_stride;
#pragma unroll 1
    for (int c = 0; c < BW; c += 16) {
      float v[16];
      cols(c, v);
      const int f = f0 + c;
      if (tv) {
        if (f + 16 <= S.rows) {
#pragma unroll
          for (int q = 0; q < 16; q += 4) {
            float4 a = *reinterpret_cast<float4*>(h + f + q);
            a.x += v[q]; a.y += v[q + 1]; a.z += v[q + 2]; a.w += v[q + 3];
            *reinterpret_cast<float4*>(h + f + q) = a;
          }
        } else {
          for (int q = 0; q < 16 && f + q < S.rows; ++q) h[f + q] += v[q];
        }
      }
    }
  } else {   // EPI_STORE, optional RoPE over heads of head_dim
    // a negative destination row marks a token to skip
    const int64_t orow = tv ? (S.use_dst ? p.dst[t] : t) : 0;
    tv = tv && orow >= 0;
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(S.out) + orow * S.out_stride;
    const int d = p.head_dim, half = d >> 1;
    const int pos = (tv && S.rope) ? p.pos[t] : 0;
    const float rs = tv ? rss_scale(p, t) : 1.f;
    auto put16 = [&](int f, float* v) {
      if (p.rss != nullptr) {
#pragma unroll
        for (int q = 0; q < 16; ++q) v[q] *= rs;
      }
      if (S.op == EPI_STORE_F32) {
        float* of = static_cast<float*>(S.out) + orow * S.out_stride;
        if (f + 16 <= S.rows) {
#pragma unroll
          for (int q = 0; q < 16; q += 4)
            *reinterpret_cast<float4*>(of + f + q) = make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]);
        } else {
          for (int q = 0; q < 16 && f + q < S.rows; ++q) of[f + q] = v[q];
        }
        return;
      }
      alignas(16) __nv_bfloat16 r[16];
#pragma unroll
      for (int q = 0; q < 16; ++q) r[q] = __float2bfloat16_rn(v[q]);
      if (f + 16 <= S.rows) {
        reinterpret_cast<uint4*>(o + f)[0] = reinterpret_cast<const uint4*>(r)[0];
        reinterpret_cast<uint4*>(o + f)[1] = reinterpret_cast<const uint4*>(r)[1];
      } else {
        for (int q = 0; q < 16 && f + q < S.rows; ++q) o[f + q] = r[q];
      }
    };
    if (S.rope) {
      // 16 frequencies at a time: one (cos, sin) set serves that chunk of
      // every head in the tile; chunk c of a head's first half pairs with
      // chunk c + d/2
#pragma unroll 1
      for (int i0 = 0; i0 < half; i0 += 16) {
        float2 cs[16];
        if (tv) rope_cs16(p, pos, i0, cs);
#pragma unroll 1
        for (int c = i0; c < BW; c += d) {
          float a[16], b[16];
          cols(c, a);
          cols(c + half, b);
          if (tv) {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const float x1 = a[q], x2 = b[q];
              a[q] = x1 * cs[q].x - x2 * cs[q].y;
              b[q] = x2 * cs[q].x + x1 * cs[q].y;
            }
            put16(f0 + c, a);
            put16(f0 + c + half, b);
          }
        }
      }
    } else {
#pragma unroll 1
      for (int c = 0; c < BW; c += 16) {
        float v[16];
        cols(c, v);
        if (tv) put16(f0 + c, v);
      }
    }
  }
}

// ---------------------------------------------------------------------------
// Token-major variant for M >= 128 tokens (the context K/V projection over
// L rows, and every GEMM when many blocks are drafted together): the TOKENS
// sit on UMMA M (128 per tile) and the weight rows on N (BW = 128 or 256
// features per tile), so each epilogue thread owns one token row of the
// accumulator.  RoPE pairs (i, i + d/2), the gate and up halves of a SwiGLU
// tile, a residual row and an argmax over the tile's vocabulary rows are
// all formed in that thread's registers, straight out of TMEM.
// ---------------------------------------------------------------------------
//
// TWO: a cluster of two CTAs on consecutive token tiles computes one
// 256-token x BW tile with cta_group::2 MMAs.  Each CTA stages its own 128
// token rows and HALF of the tile's BW weight rows (gate rows in the even
// CTA and up rows in the odd one for a SwiGLU tile), so every weight byte
// reaching shared memory feeds 256 tokens instead of 128 and each CTA moves
// 2/3 of the bytes per FLOP of the single-CTA tile.  The even CTA counts
// both CTAs' TMA bytes on its stage barriers and issues the MMAs; their
// commits arrive on the stage and accumulator barriers of both CTAs.
template <int BW, int STAGES, bool ARGMAX, bool TWO = false>
__global__ void __launch_bounds__(128, 1) gemm_tok_kernel(const __grid_constant__ Params p) {
  constexpr int X_BYTES = BM * BK * 2;        // 128 tokens x 64 k
  constexpr int W_ROWS = TWO ? BW / 2 : BW;   // weight rows this CTA stages
  constexpr int W_BYTES = W_ROWS * BK * 2;
  constexpr int STAGE = X_BYTES + W_BYTES;
  constexpr uint32_t TMEM_COLS = BW;
  constexpr uint32_t IDESC = idesc_bf16(TWO ? 2 * BM : BM, BW);
  static_assert(STAGE % 1024 == 0, "stages must stay 1024-byte aligned");
  static_assert(!TWO || BW == 256, "CTA pairs use 256-feature tiles");

  extern __shared__ uint8_t dsmem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ int s_last;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x;

  // the operand with fewer tiles varies fastest, so the CTAs resident
  // together share the larger operand's tile through L2 and it crosses HBM once
  // (CTA pairs: a 1-D grid of clusters of two along x; consecutive CTAs are
  // the two token tiles of one pair, pairs ordered the same way)
  int tile, tok_tile;
  if constexpr (TWO) {
    const int pidx = static_cast<int>(blockIdx.x >> 1);
    const int tok_pairs = static_cast<int>(gridDim.x >> 1) / p.row_tiles;
    int tp;
    if (p.tok_fast) {
      tp = pidx % tok_pairs;
      tile = pidx / tok_pairs;
    } else {
      tile = pidx % p.row_tiles;
      tp = pidx / p.row_tiles;
    }
    tok_tile = 2 * tp + static_cast<int>(blockIdx.x & 1u);
  } else {
    tile = p.tok_fast ? blockIdx.y : blockIdx.x;       // feature tile
    tok_tile = p.tok_fast ? blockIdx.x : blockIdx.y;
  }
  int sg = 0;
  while (sg + 1 < p.nseg && tile >= p.seg[sg + 1].tile_begin) ++sg;
  const Seg& S = p.seg[sg];
  const int pair = S.pair;
  const int f0 = (tile - S.tile_begin) * (pair ? BW / 2 : BW);   // first output feature
  const int tok0 = tok_tile * BM;
  const int kb0 = blockIdx.z * p.kb_per_split;
  const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
  const int nkb = kb1 - kb0;
  const uint32_t rank = TWO ? cluster_rank() : 0u;   // 0: the CTA that issues the MMAs
  const CUtensorMap* tma = &p.tm[S.map];
  const CUtensorMap* tmb = pair ? &p.tm[S.map + 1] : nullptr;
  // The CTAs that share a weight tile start their k loops at different
  // k-blocks, so they do not all request the same L2 lines at once.  The
  // order depends on the token tile only: every feature of a token sums its
  // k-blocks in the same order, so equal weight rows give equal outputs
  // (exact argmax ties stay ties).  Both CTAs of a pair walk the same order.
  const int rot = nkb > 0 ? (TWO ? tok_tile >> 1 : tok_tile) % nkb : 0;
  auto kblk = [&](int i) {
    const int j = i + rot;
    return kb0 + (j >= nkb ? j - nkb : j);
  };

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(tma);
    if (tmb) tma_prefetch_desc(tmb);
    tma_prefetch_desc(&p.tm_x);
  }
  if (warp == 2) {
    if constexpr (TWO) tmem_alloc_pair(&tmem_slot, TMEM_COLS);
    else tmem_alloc(&tmem_slot, TMEM_COLS);
  }
  tc_fence_before();
  __syncthreads();
  // both CTAs' barriers exist before either CTA's copies or commits reach them
  if constexpr (TWO) cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (tid == 0) pdl_launch();

  // stage barrier that counts this CTA's copies: its own, or the even CTA's
  auto full_addr = [&](int s) -> uint32_t {
    const uint32_t a = smem_u32(&full_bar[s]);
    return TWO && rank != 0 ? dsmem_addr(a, 0) : a;
  };
  auto load_x = [&](int i, uint8_t* sx) {
    if constexpr (TWO) tma_load_2d_pair(sx, &p.tm_x, full_addr(i % STAGES), kblk(i) * BK, tok0);
    else tma_load_2d(sx, &p.tm_x, &full_bar[i % STAGES], kblk(i) * BK, tok0);
  };
  // stage layout: [X tile 16 KB][W rows W_ROWS x 128 B]
  auto load_w = [&](int i, uint8_t* sw) {
    const int kc = kblk(i) * BK;
    if constexpr (TWO) {
      const uint32_t bar = full_addr(i % STAGES);
      if (pair) tma_load_2d_pair(sw, rank ? tmb : tma, bar, kc, f0);
      else tma_load_2d_pair(sw, tma, bar, kc, f0 + static_cast<int>(rank) * W_ROWS);
    } else if (pair) {
      tma_load_2d(sw, tma, &full_bar[i % STAGES], kc, f0);
      tma_load_2d(sw + W_BYTES / 2, tmb, &full_bar[i % STAGES], kc, f0);
    } else {
      tma_load_2d(sw, tma, &full_bar[i % STAGES], kc, f0);
    }
  };
  // the even CTA expects both CTAs' bytes of a stage
  auto expect = [&](int s) {
    if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], TWO ? 2 * STAGE : STAGE);
  };

  if (warp == 0 && lane == 0) {
    const int npre = min(STAGES, nkb);
    for (int i = 0; i < npre; ++i) {
      expect(i);
      load_w(i, smem + i * STAGE + X_BYTES);
    }
    pdl_wait();
    for (int i = 0; i < npre; ++i) load_x(i, smem + i * STAGE);
    int issued = npre;
    for (int i = npre; i < nkb; ++i) {
      const int s = i % STAGES;
      if (!mbar_wait(&empty_bar[s], ((i / STAGES) & 1) ^ 1, p.status, 31)) {
        abort_flag = 1;
        break;
      }
      if (abort_flag) break;
      uint8_t* sa = smem + s * STAGE;
      expect(s);
      load_w(i, sa + X_BYTES);
      load_x(i, sa);
      ++issued;
    }
    if (abort_flag && rank == 0) {
      for (int i = max(0, issued - STAGES); i < issued; ++i)
        mbar_wait(&full_bar[i % STAGES], (i / STAGES) & 1, p.status, 32);
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    for (int i = 0; i < nkb; ++i) {
      const int s = i % STAGES;
      if (!mbar_wait(&full_bar[s], (i / STAGES) & 1, p.status, 33)) {
        abort_flag = 1;
        break;
      }
      if (abort_flag) break;
      tc_fence_after();
      const uint8_t* sa = smem + s * STAGE;
      const uint64_t da = smem_desc_sw128(sa);
      const uint64_t db = smem_desc_sw128(sa + X_BYTES);
#pragma unroll
      for (int k = 0; k < BK / UK; ++k) {
        if constexpr (TWO) tc_mma_bf16_pair(tmem, da + 2 * k, db + 2 * k, IDESC, (i > 0 || k > 0) ? 1u : 0u);
        else tc_mma_bf16(tmem, da + 2 * k, db + 2 * k, IDESC, (i > 0 || k > 0) ? 1u : 0u);
      }
      if constexpr (TWO) tc_commit_pair(&empty_bar[s]);
      else tc_commit(&empty_bar[s]);
    }
    if constexpr (TWO) tc_commit_pair(&acc_bar);
    else tc_commit(&acc_bar);
  }
  __syncwarp();

  // ---------------- epilogue: thread = token row tok0 + tid
  const bool ok = mbar_wait(&acc_bar, 0, p.status, 34);
  tc_fence_after();
  pdl_wait();
  // warp-uniform: the tcgen05.ld below is a warp-wide instruction
  const bool live = __all_sync(0xffffffffu, ok && !abort_flag);
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const int t = tok0 + tid;
  const bool tv = t < p.M;
  const int tile_lin = tok_tile * p.row_tiles + tile;

  // split-K: every split parks its fp32 tile, the last one sums them
  bool do_op = live;
  float* mine = nullptr;
  if (p.splits > 1) {
    mine = p.partial + (static_cast<size_t>(tile_lin) * p.splits + blockIdx.z) * BM * BW +
           static_cast<size_t>(tid) * BW;
    if (live) {
#pragma unroll 1
      for (int c = 0; c < BW; c += 16) {
        float v[16];
        tmem_ld16(lane_addr + c, v);
#pragma unroll
        for (int q = 0; q < 16; q += 4)
          __stcg(reinterpret_cast<float4*>(mine + c + q), make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]));
      }
      __threadfence();
    }
    __syncthreads();
    if (tid == 0) {
      const uint32_t prev = live ? atomicAdd(p.counters + tile_lin, 1u) : 0u;
      s_last = live && prev == static_cast<uint32_t>(p.splits - 1);
    }
    __syncthreads();
    do_op = s_last != 0;
    if (do_op) __threadfence();
  }
  const float* rowbase = p.partial + static_cast<size_t>(tile_lin) * p.splits * BM * BW +
                         static_cast<size_t>(tid) * BW;
  // 16 accumulator columns [c, c + 16) of this thread's token row
  auto cols = [&](int c, float* v) {
    if (p.splits == 1) {
      tmem_ld16(lane_addr + c, v);
    } else {
#pragma unroll
      for (int q = 0; q < 16; ++q) v[q] = 0.f;
      for (int s = 0; s < p.splits; ++s) {
        const float4* src = reinterpret_cast<const float4*>(rowbase + static_cast<size_t>(s) * BM * BW + c);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 a = __ldcg(src + q);
          v[4 * q] += a.x; v[4 * q + 1] += a.y; v[4 * q + 2] += a.z; v[4 * q + 3] += a.w;
        }
      }
    }
  };

  if (do_op) {
    tok_row_epilogue<BW, ARGMAX>(p, S, tile, f0, t, tv, cols);
    if (p.splits > 1 && tid == 0) p.counters[tile_lin] = 0u;
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (TWO) {
    // after a timed-out wait, give copies that the other CTA issued against
    // this CTA's barriers time to land (bounded) before the pair tears down
    if (abort_flag) {
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 200000ull) __nanosleep(1000);
    }
    cluster_sync_all();   // neither CTA frees TMEM or exits while the other works
  }
  if (warp == 2) {
    tc_fence_after();
    if constexpr (TWO) tmem_dealloc_pair(tmem, TMEM_COLS);
    else tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Persistent token-major GEMM on CTA pairs (many tiles, no K split).  One
// cluster of two CTAs per pair of SMs walks the pair tiles t = pair,
// pair + pairs, ... (same raster as the non-persistent kernel).  Warp 0
// streams TMA stages through the ring without stopping at tile boundaries,
// warp 1 of the even CTA issues the pair MMAs, and warps 2..5 of both CTAs
// drain the accumulator: TMEM holds TWO 256-column accumulators, so tile
// i's epilogue (tcgen05.ld, RoPE / SwiGLU / residual / argmax, global
// stores) runs while tile i + 1 accumulates in the other buffer.  The
// accumulator-empty barrier lives in the even CTA and counts one arrival
// per CTA (each CTA's 128 epilogue threads meet at a named barrier first).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];"
               ::"r"(bar_cluster_addr) : "memory");
}

template <bool ARGMAX>
__global__ void __launch_bounds__(192, 1) gemm_tokp_kernel(const __grid_constant__ Params p,
                                                           const int n_tiles) {
  constexpr int BW = 256;
  constexpr int STAGES = 6;
  constexpr int X_BYTES = BM * BK * 2;        // 128 tokens x 64 k
  constexpr int W_BYTES = (BW / 2) * BK * 2;  // this CTA's half of the 256 feature rows
  constexpr int STAGE = X_BYTES + W_BYTES;
  constexpr uint32_t TMEM_COLS = 2 * BW;
  constexpr uint32_t IDESC = idesc_bf16(2 * BM, BW);
  constexpr int EPI = 128;
  static_assert(STAGE % 1024 == 0, "stages must stay 1024-byte aligned");

  extern __shared__ uint8_t dsmem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t accf_bar[2];
  __shared__ __align__(8) uint64_t acce_bar[2];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int pairs = static_cast<int>(gridDim.x >> 1);
  const int nkb = p.kb_total;
  const int tok_pairs = static_cast<int>((p.M + 2 * BM - 1) / (2 * BM));

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf_bar[b], 1);
      mbar_init(&acce_bar[b], 2);   // one arrival per CTA of the pair
    }
    abort_flag = 0;
    fence_mbar_init();
    for (int g = 0; g < p.nseg; ++g) {
      tma_prefetch_desc(&p.tm[p.seg[g].map]);
      if (p.seg[g].pair) tma_prefetch_desc(&p.tm[p.seg[g].map + 1]);
    }
    tma_prefetch_desc(&p.tm_x);
  }
  if (warp == 2) tmem_alloc_pair(&tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // both CTAs' barriers exist before copies or commits reach them
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (threadIdx.x == 0) pdl_launch();

  // pair tile -> (feature tile, pair of token tiles)
  auto decode = [&](int t, int& ftile, int& tp) {
    if (p.tok_fast) {
      tp = t % tok_pairs;
      ftile = t / tok_pairs;
    } else {
      ftile = t % p.row_tiles;
      tp = t / p.row_tiles;
    }
  };
  auto seg_of = [&](int ftile) {
    int sg = 0;
    while (sg + 1 < p.nseg && ftile >= p.seg[sg + 1].tile_begin) ++sg;
    return sg;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs): its token rows and its
      // half of the feature rows; the even CTA's stage barrier counts both
      pdl_wait();
      int s = 0;
      uint32_t ph = 0;
      for (int t = pair; t < n_tiles && !abort_flag; t += pairs) {
        int ftile, tp;
        decode(t, ftile, tp);
        const Seg& S = p.seg[seg_of(ftile)];
        const int f0 = (ftile - S.tile_begin) * (S.pair ? BW / 2 : BW);
        const int tok0 = (2 * tp + static_cast<int>(rank)) * BM;
        const CUtensorMap* tmw = S.pair ? &p.tm[S.map + (rank ? 1 : 0)] : &p.tm[S.map];
        const int wrow = S.pair ? f0 : f0 + static_cast<int>(rank) * (BW / 2);
        const int rot = tp % nkb;
        for (int i = 0; i < nkb; ++i) {
          if (!mbar_wait(&empty_bar[s], ph ^ 1, p.status, 51)) {
            abort_flag = 1;
            break;
          }
          int kb = i + rot;
          if (kb >= nkb) kb -= nkb;
          const uint32_t fb = rank ? dsmem_addr(smem_u32(&full_bar[s]), 0)
                                   : smem_u32(&full_bar[s]);
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * STAGE);
          uint8_t* st = smem + s * STAGE;
          tma_load_2d_pair(st + X_BYTES, tmw, fb, kb * BK, wrow);
          tma_load_2d_pair(st, &p.tm_x, fb, kb * BK, tok0);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (even CTA)
      int s = 0;
      uint32_t ph = 0;
      int i = 0;
      for (int t = pair; t < n_tiles; t += pairs, ++i) {
        const int b = i & 1;
        if (!abort_flag && !mbar_wait(&acce_bar[b], ((i >> 1) & 1) ^ 1, p.status, 52))
          abort_flag = 1;
        tc_fence_after();
        for (int k = 0; k < nkb; ++k) {
          if (!abort_flag && !mbar_wait(&full_bar[s], ph, p.status, 53)) abort_flag = 1;
          if (!abort_flag) {
            tc_fence_after();
            const uint8_t* st = smem + s * STAGE;
            const uint64_t da = smem_desc_sw128(st);
            const uint64_t db = smem_desc_sw128(st + X_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / UK; ++kk)
              tc_mma_bf16_pair(tmem + b * BW, da + 2 * kk, db + 2 * kk, IDESC,
                               (k > 0 || kk > 0) ? 1u : 0u);
            tc_commit_pair(&empty_bar[s]);
          }
          if (++s == STAGES) {
            s = 0;
            ph ^= 1;
          }
        }
        tc_commit_pair(&accf_bar[b]);   // also after an abort, so nobody waits long
      }
    }
  } else {
    // ---------------- epilogue warps 2..5 (both CTAs): TMEM lane = token row
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t acce0 = dsmem_addr(smem_u32(&acce_bar[0]), 0);
    const uint32_t acce1 = dsmem_addr(smem_u32(&acce_bar[1]), 0);
    pdl_wait();
    int i = 0;
    for (int t = pair; t < n_tiles; t += pairs, ++i) {
      const int b = i & 1;
      const bool ok = mbar_wait(&accf_bar[b], (i >> 1) & 1, p.status, 54);
      tc_fence_after();
      int ftile, tp;
      decode(t, ftile, tp);
      const Seg& S = p.seg[seg_of(ftile)];
      const int f0 = (ftile - S.tile_begin) * (S.pair ? BW / 2 : BW);
      const int tok = (2 * tp + static_cast<int>(rank)) * BM + r;
      const bool tv = tok < p.M;
      const uint32_t acc = lane_addr + static_cast<uint32_t>(b * BW);
      if (__all_sync(0xffffffffu, ok && !abort_flag)) {   // warp-wide tcgen05.ld below
        auto cols = [&](int c, float* v) { tmem_ld16(acc + c, v); };
        tok_row_epilogue<BW, ARGMAX>(p, S, ftile, f0, tok, tv, cols);
      }
      tc_fence_before();
      named_sync(1, EPI);
      if (threadIdx.x == 64) mbar_arrive_cluster(b ? acce1 : acce0);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (abort_flag) {
    // give copies that the other CTA issued against this CTA's barriers
    // time to land (bounded) before the pair tears down
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) __nanosleep(1000);
  }
  cluster_sync_all();   // neither CTA frees TMEM or exits while the other works
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// Stream-K weight-major variant for M <= 64 tokens (weight streaming at small
// batch).  A persistent grid of one CTA per SM; the (tile, k-block) work
// units of the whole GEMM are cut into G equal contiguous ranges, one per
// CTA, so every SM streams the same number of weight bytes whatever the
// tile count.  Warp 0 issues TMA, warp 1 issues tcgen05.mma, warps 2..5
// drain TMEM; the accumulator is double-buffered in TMEM so a finished
// tile is drained while the next one accumulates.  A tile whose k range is
// shared by several CTAs is reduced by the last contributor, slots summed
// in CTA order (deterministic).
// ---------------------------------------------------------------------------
struct SkGeom {
  int64_t units;     // tiles * kb_total
  int grid;          // G
  int max_slots;     // partial slots reserved per tile
};

__device__ __forceinline__ int64_t sk_u0(int64_t units, int grid, int c) {
  return (static_cast<int64_t>(c) * units) / grid;
}
// CTA owning unit u: the largest c with u0(c) <= u.
__device__ __forceinline__ int sk_cta_of(int64_t units, int grid, int64_t u) {
  return static_cast<int>(((u + 1) * grid - 1) / units);
}


template <int BN, int STAGES, bool ARGMAX>
__global__ void __launch_bounds__(192, 1) gemm_sk_kernel(const __grid_constant__ Params p,
                                                         const SkGeom geo) {
  constexpr int B_BYTES = BN * BK * 2;
  constexpr int STAGE = A_BYTES + B_BYTES;
  constexpr uint32_t ACC_COLS = BN < 32 ? 32 : BN;
  constexpr uint32_t TMEM_COLS = 2 * ACC_COLS;
  constexpr uint32_t IDESC = idesc_bf16(BM, BN);
  constexpr int EPI = 128;                     // epilogue threads (warps 2..5)
  static_assert(STAGE % 1024 == 0, "stages must stay 1024-byte aligned");

  extern __shared__ uint8_t dsmem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  float* st = reinterpret_cast<float*>(smem + STAGES * STAGE);   // staging [BN][SROW]
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t accf_bar[2];
  __shared__ __align__(8) uint64_t acce_bar[2];
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ int s_last;
  __shared__ unsigned long long red[ARGMAX ? 4 : 1][ARGMAX ? BN : 1];
  __shared__ float2 red2[ARGMAX ? 4 : 1][ARGMAX ? BN : 1];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kbt = p.kb_total;
  const int64_t u0 = sk_u0(geo.units, geo.grid, blockIdx.x);
  const int64_t u1 = sk_u0(geo.units, geo.grid, blockIdx.x + 1);
  const int n_units = static_cast<int>(u1 - u0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&accf_bar[b], 1);
      mbar_init(&acce_bar[b], EPI);
    }
    abort_flag = 0;
    fence_mbar_init();
    for (int g = 0; g < p.nseg; ++g) {
      tma_prefetch_desc(&p.tm[p.seg[g].map]);
      if (p.seg[g].pair) tma_prefetch_desc(&p.tm[p.seg[g].map + 1]);
    }
    tma_prefetch_desc(&p.tm_x);
  }
  if (warp == 2) tmem_alloc(&tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (threadIdx.x == 0) pdl_launch();

  // tile -> (segment, first weight row, first token)
  auto tile_info = [&](int tile, int& sg, int& row0, int& tok0) {
    const int rt = tile % p.row_tiles, tt = tile / p.row_tiles;
    sg = 0;
    while (sg + 1 < p.nseg && rt >= p.seg[sg + 1].tile_begin) ++sg;
    row0 = (rt - p.seg[sg].tile_begin) * (p.seg[sg].pair ? BM / 2 : BM);
    tok0 = tt * BN;
  };

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer over this CTA's units
      // walk the units with running (tile, k) counters: no divisions per unit
      struct Cursor {
        int tile, k, sg, row0, tok0;
      };
      auto at_tile = [&](Cursor& c) { tile_info(c.tile, c.sg, c.row0, c.tok0); };
      auto step = [&](Cursor& c) {
        if (++c.k == kbt) {
          c.k = 0;
          ++c.tile;
          at_tile(c);
        }
      };
      const uint64_t pol = policy_evict_first();   // weights are read once
      auto load_w = [&](const Cursor& c, int s, uint8_t* sa) {
        const Seg& S = p.seg[c.sg];
        const int kc = c.k * BK;
        tma_load_2d_hint(sa, &p.tm[S.map], &full_bar[s], kc, c.row0, pol);
        if (S.pair)
          tma_load_2d_hint(sa + A_BYTES / 2, &p.tm[S.map + 1], &full_bar[s], kc, c.row0, pol);
      };
      auto load_x = [&](const Cursor& c, int s, uint8_t* sa) {
        tma_load_2d(sa + A_BYTES, &p.tm_x, &full_bar[s], c.k * BK, c.tok0);
      };
      Cursor cw{static_cast<int>(u0 / kbt), static_cast<int>(u0 % kbt), 0, 0, 0};
      at_tile(cw);
      Cursor cx = cw;
      const int npre = min(STAGES, n_units);
      for (int i = 0; i < npre; ++i) {
        mbar_arrive_expect_tx(&full_bar[i], STAGE);
        load_w(cw, i, smem + i * STAGE);
        step(cw);
      }
      pdl_wait();
      for (int i = 0; i < npre; ++i) {
        load_x(cx, i, smem + i * STAGE);
        step(cx);
      }
      int issued = npre;
      int s = npre % STAGES;
      uint32_t ph = (npre / STAGES) & 1;
      for (int i = npre; i < n_units; ++i) {
        if (!mbar_wait(&empty_bar[s], ph ^ 1, p.status, 41)) {
          abort_flag = 1;
          break;
        }
        if (abort_flag) break;
        uint8_t* sa = smem + s * STAGE;
        mbar_arrive_expect_tx(&full_bar[s], STAGE);
        load_w(cw, s, sa);
        load_x(cw, s, sa);
        step(cw);
        ++issued;
        if (++s == STAGES) {
          s = 0;
          ph ^= 1;
        }
      }
      if (abort_flag) {
        for (int i = max(0, issued - STAGES); i < issued; ++i)
          mbar_wait(&full_bar[i % STAGES], (i / STAGES) & 1, p.status, 42);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer; one accumulator buffer per tile segment
      int seg_i = 0;
      int k = static_cast<int>(u0 % kbt);
      int s = 0;
      uint32_t ph = 0;
      for (int i = 0; i < n_units; ++i, ++k) {
        if (k == kbt) k = 0;
        const bool first = (i == 0) || (k == 0);
        const bool last = (i == n_units - 1) || (k == kbt - 1);
        const int b = seg_i & 1;
        if (first && seg_i >= 2) {
          if (!mbar_wait(&acce_bar[b], ((seg_i >> 1) - 1) & 1, p.status, 43)) {
            abort_flag = 1;
          }
        }
        if (!abort_flag && !mbar_wait(&full_bar[s], ph, p.status, 44)) abort_flag = 1;
        if (!abort_flag) {
          tc_fence_after();
          const uint8_t* sa = smem + s * STAGE;
          const uint64_t da = smem_desc_sw128(sa);
          const uint64_t db = smem_desc_sw128(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk)
            tc_mma_bf16(tmem + b * ACC_COLS, da + 2 * kk, db + 2 * kk, IDESC,
                        (first && kk == 0) ? 0u : 1u);
          tc_commit(&empty_bar[s]);
        }
        if (++s == STAGES) {
          s = 0;
          ph ^= 1;
        }
        if (last) {
          tc_commit(&accf_bar[b]);   // arrives even after an abort, so nobody hangs
          ++seg_i;
        }
      }
    }
  } else {
    // ---------------- epilogue warps 2..5: tile row = TMEM lane
    const int et = threadIdx.x - 64;                  // 0..127
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                // tile row
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    int seg_i = 0;
    int64_t u = u0;
    pdl_wait();
    while (u < u1) {
      const int tile = static_cast<int>(u / kbt);
      const int kb_begin = static_cast<int>(u % kbt);
      const int64_t left = u1 - u;
      const int seg_len = static_cast<int>(left < kbt - kb_begin ? left : kbt - kb_begin);
      u += seg_len;
      const int b = seg_i & 1;
      const bool ok = mbar_wait(&accf_bar[b], (seg_i >> 1) & 1, p.status, 45);
      tc_fence_after();
      float v[BN];
#pragma unroll
      for (int c = 0; c < BN; c += 16) tmem_ld16(lane_addr + b * ACC_COLS + c, v + c);
      tc_fence_before();
      mbar_arrive(&acce_bar[b]);
      ++seg_i;
      const bool live = ok && !abort_flag;
      int sg, row0, tok0;
      tile_info(tile, sg, row0, tok0);
      const Seg& S = p.seg[sg];
      // contributors to this tile
      const int c_lo = sk_cta_of(geo.units, geo.grid, static_cast<int64_t>(tile) * kbt);
      const int c_hi = sk_cta_of(geo.units, geo.grid, static_cast<int64_t>(tile + 1) * kbt - 1);
      bool do_op = live;
      if (c_hi > c_lo) {
        float* slots = p.partial + static_cast<size_t>(tile) * geo.max_slots * BN * BM;
        float* mine = slots + static_cast<size_t>(blockIdx.x - c_lo) * BN * BM;
        if (live) {
#pragma unroll
          for (int j = 0; j < BN; ++j) __stcg(mine + j * BM + r, v[j]);
          __threadfence();
        }
        named_sync(1, EPI);
        if (et == 0) {
          const uint32_t prev = live ? atomicAdd(p.counters + tile, 1u) : 0u;
          s_last = live && prev == static_cast<uint32_t>(c_hi - c_lo);
        }
        named_sync(1, EPI);
        do_op = s_last != 0;
        if (do_op) {
          __threadfence();
          // the tile's BN x 128 floats as float4 items (token j, rows 4q..4q+3),
          // each summed over the slots in CTA order, straight into the staging
          const int nsl = c_hi - c_lo + 1;
          constexpr int ITEMS = BN * (BM / 4);
#pragma unroll 1
          for (int it0 = 0; it0 < ITEMS; it0 += 4 * EPI) {
            float4 acc[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 1
            for (int sl = 0; sl < nsl; ++sl) {
              const float4* src = reinterpret_cast<const float4*>(
                  slots + static_cast<size_t>(sl) * BN * BM);
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
                *reinterpret_cast<float4*>(st + j * SROW + rq) = acc[q];
              }
            }
          }
          if (et == 0) p.counters[tile] = 0u;
        }
      } else if (do_op) {
        // stage [BN][SROW] so RoPE partners and SwiGLU halves meet
#pragma unroll
        for (int j = 0; j < BN; ++j) st[j * SROW + r] = v[j];
      }
      named_sync(1, EPI);
      if constexpr (ARGMAX) {
        if (do_op && c_hi > c_lo) {
#pragma unroll
          for (int j = 0; j < BN; ++j) v[j] = st[j * SROW + r];
        }
      }
      if (do_op) {
        if constexpr (ARGMAX) {
          const int row = row0 + r;
#pragma unroll
          for (int j = 0; j < BN; ++j) {
            unsigned long long key = 0ull;
            if (row < S.rows && tok0 + j < p.M) {
              if (!isfinite(v[j])) report(p.status, DFLASH_ENUMERIC, 46);
              key = argmax_key(v[j], static_cast<uint32_t>(row));
            }
            key = warp_max_u64(key);
            if (lane == 0) red[quarter][j] = key;
            if (p.lse != nullptr) {
              // this tile's share of the log-sum-exp of token j
              const bool in = row < S.rows;
              const float mx = warp_max(in ? v[j] : -INFINITY);
              const float se = warp_sum(in ? __expf(v[j] - mx) : 0.f);
              if (lane == 0) red2[quarter][j] = make_float2(mx, se);
            }
          }
          named_sync(1, EPI);
          for (int j = et; j < BN; j += EPI) {
            unsigned long long k = red[0][j];
#pragma unroll
            for (int w = 1; w < 4; ++w) k = red[w][j] > k ? red[w][j] : k;
            if (tok0 + j < p.M && k != 0ull) atomicMax(p.keys + tok0 + j, k);
            if (p.lse != nullptr && tok0 + j < p.M) {
              float mx = red2[0][j].x;
#pragma unroll
              for (int w = 1; w < 4; ++w) mx = fmaxf(mx, red2[w][j].x);
              float se = 0.f;
#pragma unroll
              for (int w = 0; w < 4; ++w)
                se += red2[w][j].y > 0.f ? red2[w][j].y * __expf(red2[w][j].x - mx) : 0.f;
              const int rt = tile % p.row_tiles;
              p.lse[static_cast<size_t>(rt) * p.M + tok0 + j] = make_float2(mx, se);
            }
          }
        } else if (S.op == EPI_SWIGLU) {
          const int rr = et & 63;
          const int f = row0 + rr;
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(S.out);
#pragma unroll 4
          for (int j = et >> 6; j < BN; j += 2) {
            const int t = tok0 + j;
            if (f < S.rows && t < p.M) {
              const float g = st[j * SROW + rr], uu = st[j * SROW + rr + 64];
              o[static_cast<int64_t>(t) * S.out_stride + f] =
                  __float2bfloat16_rn(g / (1.f + __expf(-g)) * uu);
            }
          }
        } else if (S.op == EPI_RESID) {
          const int f = row0 + et;
          float* h = static_cast<float*>(S.out) + f;
          float hv[BN];
#pragma unroll
          for (int j = 0; j < BN; ++j) {
            const int t = tok0 + j;
            hv[j] = (f < S.rows && t < p.M) ? h[static_cast<int64_t>(t) * S.out_stride] : 0.f;
          }
#pragma unroll
          for (int j = 0; j < BN; ++j) {
            const int t = tok0 + j;
            if (f < S.rows && t < p.M)
              h[static_cast<int64_t>(t) * S.out_stride] = hv[j] + st[j * SROW + et];
          }
        } else {
          const int f = row0 + et;
          const int half = p.head_dim >> 1;
          const int i = et % p.head_dim;
          const int prt = i < half ? et + half : et - half;
          const int fi = i < half ? i : i - half;
          __nv_bfloat16* o = static_cast<__nv_bfloat16*>(S.out);
#pragma unroll 1
          for (int j0 = 0; j0 < BN; j0 += 8) {
            float2 cs[8];
            int64_t orow[8];
            float rs[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int t = min(tok0 + j0 + q, p.M - 1);
              cs[q] = S.rope ? rope_cs(p, p.pos[t], fi) : make_float2(1.f, 0.f);
              orow[q] = S.use_dst ? p.dst[t] : t;
              rs[q] = rss_scale(p, t);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const int t = tok0 + j0 + q;
              if (j0 + q >= BN || f >= S.rows || t >= p.M || orow[q] < 0) continue;
              float x = st[(j0 + q) * SROW + et];
              if (S.rope) {
                const float pv = st[(j0 + q) * SROW + prt];
                x = i < half ? x * cs[q].x - pv * cs[q].y : x * cs[q].x + pv * cs[q].y;
              }
              x *= rs[q];
              if (S.op == EPI_STORE_F32)
                static_cast<float*>(S.out)[orow[q] * S.out_stride + f] = x;
              else
                o[orow[q] * S.out_stride + f] = __float2bfloat16_rn(x);
            }
          }
        }
      }
      named_sync(1, EPI);   // staging buffer free for the next tile
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int BN, int STAGES, bool ARGMAX>
cudaError_t launch(const Params& p, dim3 grid, cudaStream_t st) {
  constexpr int SMEM = STAGES * (A_BYTES + BN * BK * 2) + 1024;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_kernel<BN, STAGES, ARGMAX>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  });
  if (attr_err != cudaSuccess) return attr_err;
  return launch_k(gemm_kernel<BN, STAGES, ARGMAX>, grid, dim3(128), SMEM, st, p);
}

// Ring depth per token tile: small tiles keep two CTAs per SM resident.
template <bool ARGMAX>
cudaError_t dispatch(int bn, const Params& p, dim3 grid, cudaStream_t st) {
  switch (bn) {
    case 16: return launch<16, 6, ARGMAX>(p, grid, st);   // 110 KB: 2 CTAs / SM
    case 32: return launch<32, 5, ARGMAX>(p, grid, st);   // 100 KB: 2 CTAs / SM
    case 64: return launch<64, 4, ARGMAX>(p, grid, st);   //  96 KB: 2 CTAs / SM
    case 128: return launch<128, 6, ARGMAX>(p, grid, st);
    case 256: return launch<256, 4, ARGMAX>(p, grid, st);
    default: return cudaErrorInvalidValue;
  }
}

template <int BN, int STAGES, bool ARGMAX>
cudaError_t launch_sk(const Params& p, const SkGeom& geo, cudaStream_t st) {
  constexpr int SMEM = STAGES * (A_BYTES + BN * BK * 2) + BN * SROW * 4 + 1024;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_sk_kernel<BN, STAGES, ARGMAX>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  });
  if (attr_err != cudaSuccess) return attr_err;
  return launch_k(gemm_sk_kernel<BN, STAGES, ARGMAX>, dim3(geo.grid), dim3(192), SMEM, st, p,
                  geo);
}

// Two CTAs per SM, each with a ~90 KB ring: two independent TMA streams per
// SM measured faster than one persistent CTA with twice the ring.
template <bool ARGMAX>
cudaError_t dispatch_sk(int bn, const Params& p, const SkGeom& geo, cudaStream_t st) {
  switch (bn) {
    case 16: return launch_sk<16, 5, ARGMAX>(p, geo, st);
    case 32: return launch_sk<32, 4, ARGMAX>(p, geo, st);
    case 64: return launch_sk<64, 3, ARGMAX>(p, geo, st);
    default: return cudaErrorInvalidValue;
  }
}

// Stream-K partition of `tiles` x `kbt` units over at most two CTAs per SM:
// the grid and the largest number of CTAs sharing one tile.
inline SkGeom sk_geometry(int tiles, int kbt) {
  SkGeom g{};
  g.units = static_cast<int64_t>(tiles) * kbt;
  g.grid = static_cast<int>(std::min<int64_t>(g.units, kNumSMs * 2));
  g.max_slots = 1;
  auto u0 = [&](int64_t c) { return (c * g.units) / g.grid; };
  auto cta_of = [&](int64_t u) { return static_cast<int>(((u + 1) * g.grid - 1) / g.units); };
  for (int t = 0; t < tiles; ++t) {
    const int n = cta_of(static_cast<int64_t>(t + 1) * kbt - 1) -
                  cta_of(static_cast<int64_t>(t) * kbt) + 1;
    g.max_slots = std::max(g.max_slots, n);
  }
  (void)u0;
  return g;
}

template <int BW, int STAGES, bool ARGMAX>
cudaError_t launch_tok(const Params& p, dim3 grid, cudaStream_t st) {
  constexpr int SMEM = STAGES * (BM * BK * 2 + BW * BK * 2) + 1024;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_tok_kernel<BW, STAGES, ARGMAX>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  });
  if (attr_err != cudaSuccess) return attr_err;
  return launch_k(gemm_tok_kernel<BW, STAGES, ARGMAX>, grid, dim3(128), SMEM, st, p);
}

// CTA-pair token-major launch: 256-feature tiles, a 6-stage ring of 32 KB
// stages, a 1-D grid of (feature tiles x even token tiles) CTAs in clusters
// of two.
template <bool ARGMAX>
cudaError_t launch_tok2(const Params& p, dim3 grid, cudaStream_t st) {
  constexpr int STAGES = 6;
  constexpr int SMEM = STAGES * (BM * BK * 2 + 128 * BK * 2) + 1024;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_tok_kernel<256, STAGES, ARGMAX, true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  });
  if (attr_err != cudaSuccess) return attr_err;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  count_launch();
  return cudaLaunchKernelEx(&cfg, gemm_tok_kernel<256, STAGES, ARGMAX, true>, p);
}

// Persistent CTA-pair launch: one cluster of two CTAs per pair of SMs.
template <bool ARGMAX>
cudaError_t launch_tokp(const Params& p, int n_tiles, cudaStream_t st) {
  constexpr int SMEM = 6 * (BM * BK * 2 + 128 * BK * 2) + 1024;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_tokp_kernel<ARGMAX>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int pairs = std::min(n_tiles, kNumSMs / 2);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  count_launch();
  return cudaLaunchKernelEx(&cfg, gemm_tokp_kernel<ARGMAX>, p, n_tiles);
}

// The persistent kernel pays off once there is more than one wave of pair
// tiles (otherwise every pair runs a single tile anyway).
inline bool use_persistent(int pair_tiles) { return pair_tiles > kNumSMs / 2; }

// Token tiles on grid x when there are fewer of them than feature tiles (and
// the feature tiles fit grid y): the weights then stream from HBM once.
inline bool tok_fast(int tok_tiles, int feature_tiles) {
  return tok_tiles < feature_tiles && feature_tiles <= 65535;
}

template <bool ARGMAX>
cudaError_t dispatch_tok(int bw, const Params& p, dim3 grid, cudaStream_t st) {
  switch (bw) {
    case 128: return launch_tok<128, 6, ARGMAX>(p, grid, st);   // 192 KB ring
    case 256: return launch_tok<256, 4, ARGMAX>(p, grid, st);   // 192 KB ring
    default: return cudaErrorInvalidValue;
  }
}

// Tokens at or above which the token-major kernel is used (the stream-K
// weight-major kernel covers up to 64).
constexpr int64_t kTokMajorMin = 65;

inline int pick_bn(int64_t M) {
  if (M <= 16) return 16;
  if (M <= 32) return 32;
  if (M <= 64) return 64;
  if (M <= 128) return 128;
  return 256;
}
inline int ctas_per_sm(int bn) { return bn <= 64 ? 2 : 1; }

}  // namespace tc

// ===========================================================================
// SIMT kernel (fp32 models): 64 weight rows x 32 tokens per CTA, fp32
// partials reduced by a finish kernel
// ===========================================================================
namespace simt {

constexpr int TR = 64, TT = 32, TK = 32;

struct Params {
  const void* w[2 * kMaxSegs];
  int seg_tile_begin[2 * kMaxSegs + 1];
  int seg_rows[2 * kMaxSegs];
  int seg_col0[2 * kMaxSegs];
  int nseg;
  const void* x;
  int M, K;
  int k_per_split;
  int n_cols;
  float* partial;
  unsigned long long* keys;
  float2* lse;
  uint32_t* status;
};

template <bool ARGMAX>
__global__ void __launch_bounds__(256) gemm_kernel(const __grid_constant__ Params p) {
  __shared__ float ws[TK][TR + 1];
  __shared__ float xs[TK][TT + 1];
  __shared__ unsigned long long red[16][TT];
  __shared__ float2 red2[16][TT];
  const int tile = blockIdx.x;
  int seg = 0;
  while (seg + 1 < p.nseg && tile >= p.seg_tile_begin[seg + 1]) ++seg;
  const int row0 = (tile - p.seg_tile_begin[seg]) * TR;
  const int rows = p.seg_rows[seg];
  const float* W = static_cast<const float*>(p.w[seg]);
  const float* X = static_cast<const float*>(p.x);
  const int tok0 = blockIdx.y * TT;
  const int k0 = blockIdx.z * p.k_per_split;
  const int k1 = min(p.K, k0 + p.k_per_split);
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;   // rows ty + 16i, tokens tx + 16j
  pdl_wait();
  if (tid == 0) pdl_launch();
  float acc[4][2] = {};
  for (int kk = k0; kk < k1; kk += TK) {
    for (int e = tid; e < TR * TK; e += 256) {
      const int r = e / TK, k = e % TK;
      const int gr = row0 + r, gk = kk + k;
      ws[k][r] = (gr < rows && gk < k1) ? W[static_cast<size_t>(gr) * p.K + gk] : 0.f;
    }
    for (int e = tid; e < TT * TK; e += 256) {
      const int t = e / TK, k = e % TK;
      const int gt = tok0 + t, gk = kk + k;
      xs[k][t] = (gt < p.M && gk < k1) ? X[static_cast<size_t>(gt) * p.K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int k = 0; k < TK; ++k) {
      float a[4], b[2];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = ws[k][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 2; ++j) b[j] = xs[k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  if constexpr (!ARGMAX) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int r = row0 + ty + 16 * i, t = tok0 + tx + 16 * j;
        if (r < rows && t < p.M)
          p.partial[(static_cast<size_t>(blockIdx.z) * p.M + t) * p.n_cols + p.seg_col0[seg] + r] =
              acc[i][j];
      }
  } else {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      unsigned long long best = 0ull;
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = row0 + ty + 16 * i, t = tok0 + tx + 16 * j;
        if (r < rows && t < p.M) {
          if (!isfinite(acc[i][j])) report(p.status, DFLASH_ENUMERIC, 16);
          const unsigned long long k = argmax_key(acc[i][j], static_cast<uint32_t>(r));
          best = k > best ? k : best;
          mx = fmaxf(mx, acc[i][j]);
        }
      }
      float se = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = row0 + ty + 16 * i, t = tok0 + tx + 16 * j;
        if (r < rows && t < p.M) se += expf(acc[i][j] - mx);
      }
      red[ty][tx + 16 * j] = best;
      red2[ty][tx + 16 * j] = make_float2(mx, se);
    }
    __syncthreads();
    if (tid < TT) {
      unsigned long long best = 0ull;
      float mx = -INFINITY;
      for (int y = 0; y < 16; ++y) {
        best = red[y][tid] > best ? red[y][tid] : best;
        mx = fmaxf(mx, red2[y][tid].x);
      }
      float se = 0.f;
      for (int y = 0; y < 16; ++y)
        if (red2[y][tid].y > 0.f) se += red2[y][tid].y * expf(red2[y][tid].x - mx);
      if (tok0 + tid < p.M && best) atomicMax(p.keys + tok0 + tid, best);
      if (tok0 + tid < p.M && p.lse != nullptr)
        p.lse[static_cast<size_t>(blockIdx.x) * p.M + tok0 + tid] = make_float2(mx, se);
    }
  }
}

// Fixed-order split reduction + epilogue op over [splits][M][n_cols].
struct FinishSeg {
  int op, rows, col0, rope, use_dst, up_col0;
  int64_t out_stride;
  void* out;
};
struct FinishParams {
  FinishSeg seg[kMaxSegs];
  int nseg;
  int out_cols;
  int64_t M;
  int n_cols;
  int splits;
  const float* partial;
  const int32_t* pos;
  const int64_t* dst;
  int head_dim;
  double inv_freq[64];
};

__global__ void __launch_bounds__(256) finish_kernel(const __grid_constant__ FinishParams p) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int64_t total = p.M * p.out_cols;
  const size_t split_stride = static_cast<size_t>(p.M) * p.n_cols;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = idx / p.out_cols;
    int c = static_cast<int>(idx - m * p.out_cols);
    int s = 0;
    while (c >= p.seg[s].rows) c -= p.seg[s++].rows;
    const FinishSeg& sg = p.seg[s];
    const float* src = p.partial + static_cast<size_t>(m) * p.n_cols + sg.col0;
    float v = 0.f;
    for (int k = 0; k < p.splits; ++k) v += src[k * split_stride + c];
    if (sg.op == EPI_RESID) {
      float* h = static_cast<float*>(sg.out) + m * sg.out_stride + c;
      *h = *h + v;
      continue;
    }
    if (sg.op == EPI_SWIGLU) {
      const float* up = p.partial + static_cast<size_t>(m) * p.n_cols + sg.up_col0;
      float u = 0.f;
      for (int k = 0; k < p.splits; ++k) u += up[k * split_stride + c];
      static_cast<float*>(sg.out)[m * sg.out_stride + c] = v / (1.f + expf(-v)) * u;
      continue;
    }
    if (sg.rope) {
      const int d = p.head_dim, half = d >> 1;
      const int i = c % d;
      const int pc = i < half ? c + half : c - half;
      float pv = 0.f;
      for (int k = 0; k < p.splits; ++k) pv += src[k * split_stride + pc];
      const int fi = i < half ? i : i - half;
      double ang = static_cast<double>(p.pos[m]) * p.inv_freq[fi];
      ang -= 6.283185307179586 * rint(ang * 0.15915494309189535);
      float sn, cs;
      sincosf(static_cast<float>(ang), &sn, &cs);
      v = i < half ? v * cs - pv * sn : v * cs + pv * sn;
    }
    const int64_t orow = sg.use_dst ? p.dst[m] : m;
    if (orow >= 0) static_cast<float*>(sg.out)[orow * sg.out_stride + c] = v;
  }
}

}  // namespace simt

// ===========================================================================
// host side
// ===========================================================================
namespace {

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(f);
  });
  return fn;
}

void fill_inv_freq(double theta, int d, double* inv) {
  for (int i = 0; i < d / 2 && i < 64; ++i) inv[i] = std::pow(theta, -2.0 * i / d);
}

}  // namespace

bool encode_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t inner,
                         uint64_t outer, uint32_t box_inner, uint32_t box_outer) {
  EncodeFn fn = get_encode();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1,
                         uint64_t d2, uint32_t b0, uint32_t b1, uint32_t b2) {
  EncodeFn fn = get_encode();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

GemmPlan plan_gemm(const GemmJob& job) {
  GemmPlan pl{};
  const int64_t M = job.M;
  int n_cols = 0;
  if (job.dtype == DFLASH_BF16) {
    const int kb_total = ceil_div(job.K, tc::BK);
    auto feature_tiles = [&](int per_tile) {
      int n = 0;
      for (int s = 0; s < job.nseg; ++s)
        n += job.seg[s].op == EPI_SWIGLU ? ceil_div(job.seg[s].rows, per_tile / 2)
                                         : ceil_div(job.seg[s].rows, per_tile);
      return n;
    };
    int splits = 1;
    if (M >= tc::kTokMajorMin) {
      // token-major: 128 tokens x BW features per tile, tensor-bound
      pl.tok_major = 1;
      pl.tok_tiles = ceil_div(M, tc::BM);
      pl.bn = 256;
      pl.row_tiles = feature_tiles(256);
      if (pl.row_tiles * pl.tok_tiles * 2 < kNumSMs) {   // under half the SMs busy
        pl.bn = 128;
        pl.row_tiles = feature_tiles(128);
      }
      const int tiles = pl.row_tiles * pl.tok_tiles;
      if (tiles * 2 < kNumSMs) splits = std::min(kb_total, kNumSMs / tiles);
      // pairs of token tiles share each weight tile's shared-memory traffic
      pl.two = pl.bn == 256 && splits == 1 && pl.tok_tiles >= 2;
    } else {
      // weight-major (swap-AB): 128 weight rows x BN tokens per tile, split K
      // so about two CTAs per SM stream at once and all fit in one wave
      pl.bn = tc::pick_bn(M);
      pl.tok_tiles = ceil_div(M, pl.bn);
      pl.row_tiles = feature_tiles(tc::BM);
      // (the stream-K kernel measured slower here than whole-tile CTAs: its
      // extra shared-tile reductions cost more than the wave balance gains)
      const int tiles = pl.row_tiles * pl.tok_tiles;
      const int slots = kNumSMs * tc::ctas_per_sm(pl.bn);
      if (tiles < slots) splits = std::max(1, std::min(kb_total, slots / tiles));
    }
    splits = std::max(1, std::min(splits, 32));
    pl.kb_per_split = ceil_div(kb_total, splits);
    pl.splits = ceil_div(kb_total, pl.kb_per_split);
    const int tiles = pl.row_tiles * pl.tok_tiles;
    pl.partial_floats =
        pl.splits > 1 ? static_cast<size_t>(tiles) * pl.splits * pl.bn * tc::BM : 0;
    pl.counters = pl.splits > 1 ? tiles : 0;
    return pl;
  }
  for (int s = 0; s < job.nseg; ++s) {
    const int mats = job.seg[s].op == EPI_SWIGLU ? 2 : 1;
    n_cols += mats * job.seg[s].rows;
    pl.row_tiles += mats * ceil_div(job.seg[s].rows, simt::TR);
  }
  pl.bn = simt::TT;
  pl.tok_tiles = ceil_div(M, pl.bn);
  const int kb_total = ceil_div(job.K, simt::TK);
  const int tiles = pl.row_tiles * pl.tok_tiles;
  const int target = kNumSMs * 4;
  int splits = tiles < target ? std::min(kb_total, ceil_div(target, tiles)) : 1;
  splits = std::max(1, std::min(splits, 32));
  pl.kb_per_split = ceil_div(kb_total, splits);
  pl.splits = ceil_div(kb_total, pl.kb_per_split);
  pl.partial_floats = static_cast<size_t>(pl.splits) * M * n_cols;
  pl.counters = 0;
  return pl;
}

static cudaError_t launch_gemm_simt(const GemmJob& job, const GemmPlan& pl, float* partial,
                                    uint32_t* status, cudaStream_t st) {
  if (job.rss != nullptr) return cudaErrorInvalidValue;   // bf16 paths only
  simt::Params p{};
  simt::FinishParams f{};
  int tiles = 0, col = 0, n = 0;
  for (int s = 0; s < job.nseg; ++s) {
    const GemmOut& o = job.seg[s];
    const int mats = o.op == EPI_SWIGLU ? 2 : 1;
    f.seg[s] = {o.op, o.rows, col, o.rope, o.use_dst, o.op == EPI_SWIGLU ? col + o.rows : 0,
                o.out_stride, o.out};
    for (int m = 0; m < mats; ++m) {
      p.w[n] = m == 0 ? o.w0 : o.w1;
      p.seg_tile_begin[n] = tiles;
      p.seg_rows[n] = o.rows;
      p.seg_col0[n] = col;
      tiles += ceil_div(o.rows, simt::TR);
      col += o.rows;
      ++n;
    }
  }
  p.seg_tile_begin[n] = tiles;
  p.nseg = n;
  p.x = job.x;
  p.M = static_cast<int>(job.M);
  p.K = job.K;
  p.k_per_split = pl.kb_per_split * simt::TK;
  p.n_cols = col;
  p.partial = partial;
  p.status = status;
  cudaError_t e = launch_k(simt::gemm_kernel<false>, dim3(tiles, pl.tok_tiles, pl.splits),
                           dim3(256), 0, st, p);
  if (e != cudaSuccess) return e;
  f.nseg = job.nseg;
  f.out_cols = 0;
  for (int s = 0; s < job.nseg; ++s) f.out_cols += job.seg[s].rows;
  f.M = job.M;
  f.n_cols = col;
  f.splits = pl.splits;
  f.partial = partial;
  f.pos = job.pos;
  f.dst = job.dst;
  f.head_dim = job.head_dim;
  fill_inv_freq(job.theta, std::max(job.head_dim, 2), f.inv_freq);
  const int64_t total = job.M * f.out_cols;
  const int grid = static_cast<int>(std::min<int64_t>((total + 255) / 256, kNumSMs * 16));
  return launch_k(simt::finish_kernel, dim3(grid), dim3(256), 0, st, f);
}

cudaError_t launch_gemm(const GemmJob& job, const GemmPlan& pl, float* partial,
                        uint32_t* counters, uint32_t* status, cudaStream_t st) {
  if (job.M <= 0) return cudaSuccess;
  if (job.dtype != DFLASH_BF16) return launch_gemm_simt(job, pl, partial, status, st);
  tc::Params p{};
  int tiles = 0, maps = 0;
  for (int s = 0; s < job.nseg; ++s) {
    const GemmOut& o = job.seg[s];
    tc::Seg& S = p.seg[s];
    S.tile_begin = tiles;
    S.map = maps;
    S.rows = o.rows;
    S.pair = o.op == EPI_SWIGLU;
    S.op = o.op;
    S.rope = o.rope;
    S.use_dst = o.use_dst;
    S.out_stride = o.out_stride;
    S.out = o.out;
    // rows of one weight box: the tile's feature count (half of it per
    // matrix for a SwiGLU pair)
    const int per_tile = pl.tok_major ? pl.bn : tc::BM;
    if (pl.two) {
      // each CTA of a pair stages 128 rows: half a tile, or one SwiGLU half
      if (!encode_tmap_bf16_2d(&p.tm[maps++], o.w0, job.K, o.rows, tc::BK, 128) ||
          (S.pair && !encode_tmap_bf16_2d(&p.tm[maps++], o.w1, job.K, o.rows, tc::BK, 128)))
        return cudaErrorInvalidValue;
      tiles += S.pair ? ceil_div(o.rows, 128) : ceil_div(o.rows, 256);
    } else if (S.pair) {
      if (!encode_tmap_bf16_2d(&p.tm[maps++], o.w0, job.K, o.rows, tc::BK, per_tile / 2) ||
          !encode_tmap_bf16_2d(&p.tm[maps++], o.w1, job.K, o.rows, tc::BK, per_tile / 2))
        return cudaErrorInvalidValue;
      tiles += ceil_div(o.rows, per_tile / 2);
    } else {
      if (!encode_tmap_bf16_2d(&p.tm[maps++], o.w0, job.K, o.rows, tc::BK, per_tile))
        return cudaErrorInvalidValue;
      tiles += ceil_div(o.rows, per_tile);
    }
    if (maps > 4) return cudaErrorInvalidValue;
  }
  if (!encode_tmap_bf16_2d(&p.tm_x, job.x, job.K, job.M, tc::BK,
                           pl.tok_major ? tc::BM : pl.bn))
    return cudaErrorInvalidValue;
  p.nseg = job.nseg;
  p.M = static_cast<int>(job.M);
  p.kb_total = ceil_div(job.K, tc::BK);
  p.kb_per_split = pl.kb_per_split;
  p.splits = pl.splits;
  p.row_tiles = tiles;
  p.partial = partial;
  p.counters = counters;
  p.pos = job.pos;
  p.dst = job.dst;
  p.head_dim = job.head_dim > 0 ? job.head_dim : 128;
  p.rope_tab = job.rope_tab;
  p.rss = job.rss;
  p.rss_parts = job.rss_parts;
  p.rss_inv = job.rss_inv;
  p.rss_eps = job.rss_eps;
  p.rope_len = job.rope_len;
  fill_inv_freq(job.theta, p.head_dim, p.inv_freq);
  p.status = status;
  if (pl.stream_k) {
    tc::SkGeom geo{};
    geo.units = static_cast<int64_t>(tiles) * pl.tok_tiles * p.kb_total;
    geo.grid = pl.sk_grid;
    geo.max_slots = pl.sk_slots;
    return tc::dispatch_sk<false>(pl.bn, p, geo, st);
  }
  dim3 grid(tiles, pl.tok_tiles, pl.splits);
  if (pl.tok_major) {
    p.tok_fast = tc::tok_fast(pl.tok_tiles, tiles);
    if (pl.two) {
      const int tt = (pl.tok_tiles + 1) & ~1;   // whole pairs; a spare tile is all padding
      if (tc::use_persistent(tiles * (tt / 2)))
        return tc::launch_tokp<false>(p, tiles * (tt / 2), st);
      return tc::launch_tok2<false>(p, dim3(static_cast<unsigned>(tiles) * tt), st);
    }
    if (p.tok_fast) grid = dim3(pl.tok_tiles, tiles, pl.splits);
    return tc::dispatch_tok<false>(pl.bn, p, grid, st);
  }
  return tc::dispatch<false>(pl.bn, p, grid, st);
}

GemmPlan plan_lmhead(int dtype, int V, int64_t M, int K) {
  GemmPlan pl{};
  if (dtype != DFLASH_BF16 || M >= tc::kTokMajorMin) return pl;
  pl.bn = tc::pick_bn(M);
  pl.tok_tiles = ceil_div(M, pl.bn);
  pl.row_tiles = ceil_div(V, tc::BM);
  const int tiles = pl.row_tiles * pl.tok_tiles;
  const tc::SkGeom g = tc::sk_geometry(tiles, ceil_div(K, tc::BK));
  pl.stream_k = 1;
  pl.sk_grid = g.grid;
  pl.sk_slots = g.max_slots;
  pl.splits = 1;
  pl.partial_floats = g.max_slots > 1 ? static_cast<size_t>(tiles) * g.max_slots * pl.bn * tc::BM
                                      : 0;
  pl.counters = g.max_slots > 1 ? tiles : 0;
  return pl;
}

int lmhead_tiles(int dtype, int V, int64_t M) {
  if (dtype == DFLASH_BF16 && M >= tc::kTokMajorMin) return ceil_div(V, 256);
  if (dtype == DFLASH_BF16) return ceil_div(V, tc::BM);
  return ceil_div(V, simt::TR);
}

cudaError_t launch_lmhead_argmax(int dtype, const void* W, int V, const void* X, int64_t M,
                                 int K, unsigned long long* keys, uint32_t* status,
                                 cudaStream_t st, float* partial, uint32_t* counters,
                                 float2* lse) {
  if (M <= 0) return cudaSuccess;
  if (dtype == DFLASH_BF16 && M >= tc::kTokMajorMin) {
    tc::Params p{};
    constexpr int BW = 256;
    const int tt = ceil_div(M, tc::BM);
    const bool two = tt >= 2;   // CTA pairs over consecutive token tiles
    if (!encode_tmap_bf16_2d(&p.tm[0], W, K, V, tc::BK, two ? BW / 2 : BW))
      return cudaErrorInvalidValue;
    if (!encode_tmap_bf16_2d(&p.tm_x, X, K, M, tc::BK, tc::BM)) return cudaErrorInvalidValue;
    p.seg[0].rows = V;
    p.nseg = 1;
    p.M = static_cast<int>(M);
    p.kb_total = ceil_div(K, tc::BK);
    p.kb_per_split = p.kb_total;
    p.splits = 1;
    p.row_tiles = ceil_div(V, BW);
    p.keys = keys;
    p.lse = lse;
    p.status = status;
    p.tok_fast = tc::tok_fast(tt, p.row_tiles);
    if (two) {
      const int te = (tt + 1) & ~1;
      if (tc::use_persistent(p.row_tiles * (te / 2)))
        return tc::launch_tokp<true>(p, p.row_tiles * (te / 2), st);
      return tc::launch_tok2<true>(p, dim3(static_cast<unsigned>(p.row_tiles) * te), st);
    }
    const dim3 grid = p.tok_fast ? dim3(tt, p.row_tiles, 1) : dim3(p.row_tiles, tt, 1);
    return tc::dispatch_tok<true>(BW, p, grid, st);
  }
  if (dtype == DFLASH_BF16 && partial != nullptr) {
    tc::Params p{};
    if (!encode_tmap_bf16_2d(&p.tm[0], W, K, V, tc::BK, tc::BM)) return cudaErrorInvalidValue;
    const int bn = tc::pick_bn(M);
    if (!encode_tmap_bf16_2d(&p.tm_x, X, K, M, tc::BK, bn)) return cudaErrorInvalidValue;
    p.seg[0].rows = V;
    p.nseg = 1;
    p.M = static_cast<int>(M);
    p.kb_total = ceil_div(K, tc::BK);
    p.kb_per_split = p.kb_total;
    p.splits = 1;
    p.row_tiles = ceil_div(V, tc::BM);
    p.partial = partial;
    p.counters = counters;
    p.keys = keys;
    p.lse = lse;
    p.status = status;
    const tc::SkGeom geo = tc::sk_geometry(p.row_tiles * ceil_div(M, bn), p.kb_total);
    return tc::dispatch_sk<true>(bn, p, geo, st);
  }
  if (dtype == DFLASH_BF16) {
    tc::Params p{};
    if (!encode_tmap_bf16_2d(&p.tm[0], W, K, V, tc::BK, tc::BM)) return cudaErrorInvalidValue;
    const int bn = tc::pick_bn(M);
    if (!encode_tmap_bf16_2d(&p.tm_x, X, K, M, tc::BK, bn)) return cudaErrorInvalidValue;
    p.seg[0].tile_begin = 0;
    p.seg[0].map = 0;
    p.seg[0].rows = V;
    p.nseg = 1;
    p.M = static_cast<int>(M);
    p.kb_total = ceil_div(K, tc::BK);
    p.kb_per_split = p.kb_total;
    p.splits = 1;
    p.row_tiles = ceil_div(V, tc::BM);
    p.keys = keys;
    p.lse = lse;
    p.status = status;
    dim3 grid(ceil_div(V, tc::BM), ceil_div(M, bn), 1);
    return tc::dispatch<true>(bn, p, grid, st);
  }
  simt::Params p{};
  p.w[0] = W;
  p.seg_tile_begin[0] = 0;
  p.seg_tile_begin[1] = ceil_div(V, simt::TR);
  p.seg_rows[0] = V;
  p.nseg = 1;
  p.x = X;
  p.M = static_cast<int>(M);
  p.K = K;
  p.k_per_split = K;
  p.keys = keys;
  p.lse = lse;
  p.status = status;
  return launch_k(simt::gemm_kernel<true>, dim3(ceil_div(V, simt::TR), ceil_div(M, simt::TT), 1),
                  dim3(256), 0, st, p);
}

}  // namespace dfl
