// Block attention with KV injection (DFLARE summary, section 2.2): the B
// block queries of every head attend, without a mask, to the keys of
// [request context ; this block], GQA group G = Hq / Hkv.
//
// Split-KV (flash-decoding): the grid is (block x kv head, split, query-row
// chunk).  A split streams its slice of the request's packed context K/V
// (split 0 also takes the B block keys) and keeps an fp32 online softmax
// (running max m, sum l, unnormalised output o) per query row.  In the bf16
// path the splits of one (block, kv head, row chunk) form a thread-block
// cluster: each split leaves its partials in its own shared memory and, after
// a cluster barrier, every CTA merges a slice of the rows by reading all the
// splits' partials over distributed shared memory, so partials never reach
// global memory and no second kernel runs.  The fp32 path writes partials
// and a combine kernel merges them.  Both merge the splits in a fixed order.
#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dfl {

struct AttnParams {
  CUtensorMap tm_k;          // bf16 context cache [rows][Hkv][d] (3-D TMA map)
  CUtensorMap tm_v;
  uint32_t* status;
  const void* q;
  const void* kb;
  const void* vb;
  const void* kc;
  const void* vc;
  const int64_t* ctx_off;
  const int32_t* ctx_len;    // nullable: rows of request r = ctx_len[r]
  const int32_t* block_req;
  int B, Hq, Hkv, G;
  int splits, chunk, rows_per_cta;
  float scale;
  float* part_o;   // [nb*B*Hq][splits][d]
  float* part_ml;  // [nb*B*Hq][splits][2]
  void* out;       // [nb*B*Hq][d] (bf16 cluster / single-split paths)
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
  pdl_wait();
  const int b = blockIdx.x / p.Hkv, g = blockIdx.x % p.Hkv;
  const int split = blockIdx.y;
  const int r = p.block_req[b];
  const int64_t c_begin = p.ctx_off[r];
  int64_t L = p.ctx_len ? static_cast<int64_t>(p.ctx_len[r]) : p.ctx_off[r + 1] - c_begin;
  if (!DFL_BOUNDS(L >= 0 && L <= p.ctx_off[r + 1] - c_begin, p.status, 86)) L = 0;
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
  if (tid == 0) pdl_launch();

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

// ---------------------------------------------------------------------------
// bf16 tensor-core variant: 4 warps x 16 query rows, 64-key tiles in a
// double-buffered shared-memory ring (full tiles by TMA, the ragged tail and
// the block keys by cp.async; 16-byte chunks XOR-swizzled per row so
// ldmatrix is conflict-free), S = Q K^T and O += P V on mma.sync m16n8k16
// with fp32 accumulation, P kept in registers, online softmax in the exp2
// domain.
// ---------------------------------------------------------------------------
constexpr int kMmaRows = 64;
constexpr int kMmaKeys = 64;

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = smem_u32(dst);
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                          uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t& r0, uint32_t& r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];"
               : "=r"(r0), "=r"(r1) : "r"(addr));
}
// a register-only instruction: not volatile, so the compiler may interleave
// independent MMAs with the fragment loads
__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float dsmem_ld(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float4 dsmem_ld4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr) : "memory");
  return v;
}

// Context K/V tiles of 64 keys stream through TMA (cp.async.bulk.tensor on a
// 3-D map [rows][Hkv][d] of the packed cache, one 64-dim box per 128-byte
// swizzled sub-tile) into a 2-stage mbarrier ring; every full 64-key tile of
// a split comes this way.  The split's ragged tail tile (fewer than 64
// context keys) and, for split 0, the B block keys are gathered with
// cp.async, in the same swizzled layout, into ring stages that no TMA will
// write again, so the TMA never reads past the request's last row.  Sub-tile s of a 64-key tile is
// 64 keys x 64 dims (8 KB); 16-byte chunk c of key k sits at chunk
// c ^ (k & 7) of its 128-byte row (the TMA 128-byte swizzle), which keeps
// the ldmatrix reads conflict-free.
//
// Splits: the CS CTAs of one (block, kv head, row chunk) divide THIS
// request's context into CS near-equal 64-key-aligned slices, so ragged
// requests spread their keys over all CTAs of their cluster.
//
// CS = 0: partials to global memory for the combine kernel.  CS = 1: one
// split, normalised in registers.  CS >= 2: the grid's y extent is CS and
// each cluster of CS CTAs (one per split) merges through shared memory.
constexpr int kAttnStages = 2;
constexpr uint64_t kMaxCacheRows = 1ull << 28;   // row extent of the K/V tensor maps

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
        "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// byte offset of 16-byte chunk `ch` of key `kk` in a swizzled 64-key tile
__device__ __forceinline__ uint32_t tile_off(int kk, int ch) {
  return static_cast<uint32_t>((ch >> 3) * 8192 + kk * 128 + (((ch & 7) ^ (kk & 7)) << 4));
}

template <int D, int CS>
__global__ void __launch_bounds__(128, 3) attn_mma_kernel(const __grid_constant__ AttnParams p) {
  constexpr int CH = D / 8;                 // 16-byte chunks per key row
  constexpr int NT = kMmaKeys / 8;          // n-tiles of S per key tile
  constexpr int KS = D / 16;                // k-steps of Q K^T
  constexpr int DT = D / 8;                 // n-tiles of O
  constexpr int TILE = kMmaKeys * D * 2;    // bytes of one K (or V) tile
  constexpr int SUB = D / 64;               // 64-dim TMA boxes per tile
  extern __shared__ __align__(1024) uint8_t smraw_[];
  uint8_t* smraw = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smraw_) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smraw;                                // [stage][K tile | V tile]
  __shared__ __align__(8) uint64_t full[kAttnStages];
  __shared__ volatile int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < kAttnStages; ++i) mbar_init(&full[i], 1);
    abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&p.tm_k);
    tma_prefetch_desc(&p.tm_v);
  }
  __syncthreads();
  pdl_wait();
  if (tid == 0) pdl_launch();
  const int b = blockIdx.x / p.Hkv, g = blockIdx.x % p.Hkv;
  const int split = blockIdx.y;
  const int nsplit = CS >= 1 ? CS : p.splits;
  const int r = p.block_req[b];
  const int64_t c_begin = p.ctx_off[r];
  int64_t L = p.ctx_len ? static_cast<int64_t>(p.ctx_len[r]) : p.ctx_off[r + 1] - c_begin;
  if (!DFL_BOUNDS(L >= 0 && L <= p.ctx_off[r + 1] - c_begin, p.status, 85)) L = 0;
  const int64_t chunk = ((L + nsplit - 1) / nsplit + kMmaKeys - 1) / kMmaKeys * kMmaKeys;
  const int64_t k_lo = static_cast<int64_t>(split) * chunk;
  const int n_ctx = static_cast<int>(std::max<int64_t>(0, std::min<int64_t>(L, k_lo + chunk) - k_lo));
  const int n_full = n_ctx / kMmaKeys;                 // TMA tiles
  const int n_tail = n_ctx - n_full * kMmaKeys;        // keys of the gathered tail tile
  const int n_blk = split == 0 ? p.B : 0;
  const int nrows_all = p.B * p.G;
  const int gq = lane >> 2, tq = lane & 3;
  const int rbase = blockIdx.z * kMmaRows + warp * 16;
  const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(p.q);
  const __nv_bfloat16* KC = static_cast<const __nv_bfloat16*>(p.kc);
  const __nv_bfloat16* VC = static_cast<const __nv_bfloat16*>(p.vc);
  const __nv_bfloat16* KB = static_cast<const __nv_bfloat16*>(p.kb);
  const __nv_bfloat16* VB = static_cast<const __nv_bfloat16*>(p.vb);
  const int row0 = static_cast<int>(c_begin + k_lo);

  auto issue = [&](int t) {   // TMA of full tile t into stage t % kAttnStages
    const int st = t % kAttnStages;
    uint8_t* dst = ring + st * 2 * TILE;
    mbar_arrive_expect_tx(&full[st], 2 * TILE);
#pragma unroll
    for (int sb = 0; sb < SUB; ++sb) {
      tma_load_3d(dst + sb * 8192, &p.tm_k, &full[st], sb * 64, g, row0 + t * kMmaKeys);
      tma_load_3d(dst + TILE + sb * 8192, &p.tm_v, &full[st], sb * 64, g, row0 + t * kMmaKeys);
    }
  };
  // gather n keys (the ragged context tail, or the block rows) into ring
  // stage `st` once no TMA is pending on it: the tail goes to the stage that
  // tile n_full would use (free after tile n_full - 2), the block keys to the
  // other one (free after tile n_full - 1)
  auto gather = [&](bool block_keys, int n, int st) {
    uint8_t* man = ring + st * 2 * TILE;
    for (int c = tid; c < kMmaKeys * CH; c += 128) {
      const int kk = c / CH, ch = c % CH;
      const bool valid = kk < n;
      const __nv_bfloat16* sk = KB;   // any valid address when nothing is read
      const __nv_bfloat16* sv = VB;
      size_t off = 0;
      if (valid && !block_keys) {
        sk = KC;
        sv = VC;
        off = (static_cast<size_t>(row0 + n_full * kMmaKeys + kk) * p.Hkv + g) * D + ch * 8;
      } else if (valid) {
        off = ((static_cast<size_t>(b) * p.B + kk) * p.Hkv + g) * D + ch * 8;
      }
      cp_async16(man + tile_off(kk, ch), sk + off, valid);
      cp_async16(man + TILE + tile_off(kk, ch), sv + off, valid);
    }
    cp_async_commit();
  };

  const int st_tail = n_full & 1, st_blk = (n_full + 1) & 1;
  if (tid == 0)
    for (int t = 0; t < n_full && t < kAttnStages; ++t) issue(t);
  if (n_tail > 0 && n_full <= 1) gather(false, n_tail, st_tail);
  if (n_blk > 0 && n_full == 0) gather(true, n_blk, st_blk);

  // Q fragments of this warp's 16 rows (rows past B*G read as zero)
  uint32_t qf[KS][4];
  {
    const __nv_bfloat16* qrow[2] = {nullptr, nullptr};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rr = rbase + gq + 8 * h;
      if (rr < nrows_all) {
        const int s = rr / p.G, j = rr % p.G;
        qrow[h] = Q + ((static_cast<size_t>(b) * p.B + s) * p.Hq + g * p.G + j) * D;
      }
    }
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int col = ks * 16 + 2 * tq;
        qf[ks][h] = qrow[h] ? *reinterpret_cast<const uint32_t*>(qrow[h] + col) : 0u;
        qf[ks][h + 2] = qrow[h] ? *reinterpret_cast<const uint32_t*>(qrow[h] + col + 8) : 0u;
      }
    }
  }

  constexpr float kLog2e = 1.4426950408889634f;
  const float sl2 = p.scale * kLog2e;
  float o[DT][4];
#pragma unroll
  for (int i = 0; i < DT; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  // one 64-key tile (K at kbase, V at vbase, swizzled), keys < nvalid count
  auto process = [&](uint32_t kbase, uint32_t vbase, int nvalid) {
    float sc[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    // k-step outer, key tile inner: consecutive MMAs accumulate into
    // different tiles
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int kk = nt * 8 + (lane & 7);
        const int ch = ks * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1;
        ldsm_x2(kbase + tile_off(kk, ch), b0, b1);
        mma_bf16(sc[nt], qf[ks], b0, b1);
      }
    }
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = nt * 8 + 2 * tq + e < nvalid;
        sc[nt][e] = ok ? sc[nt][e] * sl2 : -INFINITY;
        sc[nt][e + 2] = ok ? sc[nt][e + 2] * sl2 : -INFINITY;
        mx0 = fmaxf(mx0, sc[nt][e]);
        mx1 = fmaxf(mx1, sc[nt][e + 2]);
      }
    }
#pragma unroll
    for (int off = 1; off < 4; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float c0 = exp2f(m0 - mn0), c1 = exp2f(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    l0 *= c0;
    l1 *= c1;
#pragma unroll
    for (int i = 0; i < DT; ++i) {
      o[i][0] *= c0; o[i][1] *= c0;
      o[i][2] *= c1; o[i][3] *= c1;
    }
    uint32_t pf[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float p0 = exp2f(sc[nt][0] - mn0), p1 = exp2f(sc[nt][1] - mn0);
      const float p2 = exp2f(sc[nt][2] - mn1), p3 = exp2f(sc[nt][3] - mn1);
      l0 += p0 + p1;
      l1 += p2 + p3;
      pf[nt][0] = pack_bf16(p0, p1);
      pf[nt][1] = pack_bf16(p2, p3);
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < kMmaKeys / 16; ++kk) {
      const uint32_t a[4] = {pf[2 * kk][0], pf[2 * kk][1], pf[2 * kk + 1][0], pf[2 * kk + 1][1]};
#pragma unroll
      for (int dt = 0; dt < DT; dt += 2) {
        const int mi = lane >> 3;
        const int key = kk * 16 + (mi & 1) * 8 + (lane & 7);
        const int ch = dt + (mi >> 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbase + tile_off(key, ch), b0, b1, b2, b3);
        mma_bf16(o[dt], a, b0, b1);
        mma_bf16(o[dt + 1], a, b2, b3);
      }
    }
  };

  // full context tiles through the TMA ring; one block barrier per tile
  int t = 0;
  for (; t < n_full; ++t) {
    const int st = t % kAttnStages;
    // every thread waits (bounded); a warp computes only if all its lanes saw
    // the tile, and every warp reaches the barrier below either way
    const bool ok = mbar_wait(&full[st], static_cast<uint32_t>((t / kAttnStages) & 1),
                              p.status, 71);
    if (!ok) abort_flag = 1;
    if (__all_sync(0xffffffffu, ok)) {
      const uint32_t base = smem_u32(ring + st * 2 * TILE);
      process(base, base + TILE, kMmaKeys);
    }
    __syncthreads();   // every warp is done with the stage before it is refilled
    if (abort_flag) break;
    if (tid == 0 && t + kAttnStages < n_full) issue(t + kAttnStages);
    // the stages freed for good take the gathered tiles
    if (t == n_full - 2 && n_tail > 0) gather(false, n_tail, st_tail);
    if (t == n_full - 1 && n_blk > 0) gather(true, n_blk, st_blk);
  }
  if (abort_flag) {
    // let TMA copies still in flight land before the CTA's shared memory goes away
    if (tid == 0)
      for (int q = t; q < n_full && q <= t + 1; ++q)   // tiles t, t + 1 may be in flight
        mbar_wait(&full[q % kAttnStages], static_cast<uint32_t>((q / kAttnStages) & 1),
                  p.status, 72);
    cp_async_wait<0>();
    __syncthreads();
  } else {
    // the gathered tail tile, then (split 0) the block keys
    if (n_tail > 0) {
      if (n_blk > 0) cp_async_wait<1>();   // the block keys may still be landing
      else cp_async_wait<0>();
      __syncthreads();
      process(smem_u32(ring + st_tail * 2 * TILE), smem_u32(ring + st_tail * 2 * TILE + TILE),
              n_tail);
    }
    if (n_blk > 0) {
      cp_async_wait<0>();
      __syncthreads();
      process(smem_u32(ring + st_blk * 2 * TILE), smem_u32(ring + st_blk * 2 * TILE + TILE),
              n_blk);
    }
    __syncthreads();
  }
  // partial results: unnormalised O, running max (natural-log units), sum
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  constexpr float kLn2 = 0.6931471805599453f;
  auto out_row = [&](int rr) -> size_t {   // output row of query row rr
    const int s = rr / p.G, j = rr % p.G;
    return (static_cast<size_t>(b) * p.B + s) * p.Hq + g * p.G + j;
  };
  if constexpr (CS == 0) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rr = rbase + gq + 8 * h;
      if (rr >= nrows_all) continue;
      const size_t pr = out_row(rr);
      float* po = p.part_o + (pr * p.splits + split) * D;
#pragma unroll
      for (int dt = 0; dt < DT; ++dt)
        *reinterpret_cast<float2*>(po + dt * 8 + 2 * tq) =
            make_float2(o[dt][2 * h], o[dt][2 * h + 1]);
      if (tq == 0) {
        const float mm = h ? m1 : m0;
        p.part_ml[(pr * p.splits + split) * 2 + 0] = mm == -INFINITY ? -INFINITY : mm * kLn2;
        p.part_ml[(pr * p.splits + split) * 2 + 1] = h ? l1 : l0;
      }
    }
  } else if constexpr (CS == 1) {
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rr = rbase + gq + 8 * h;
      if (rr >= nrows_all) continue;
      const float inv = 1.f / (h ? l1 : l0);
      __nv_bfloat16* orow = out + out_row(rr) * D;
#pragma unroll
      for (int dt = 0; dt < DT; ++dt)
        *reinterpret_cast<__nv_bfloat162*>(orow + dt * 8 + 2 * tq) =
            __floats2bfloat162_rn(o[dt][2 * h] * inv, o[dt][2 * h + 1] * inv);
    }
  } else {
    // this split's partials into its own shared memory (the K/V ring is free:
    // the loop ended on a block barrier)
    constexpr int OS = D + 4;                 // padded row stride (16-byte aligned)
    constexpr int RPR = kMmaRows / CS;        // rows merged by each CTA
    float* so = reinterpret_cast<float*>(smraw);            // [64][OS]
    float* sml = so + kMmaRows * OS;                         // [64][2]
    __shared__ float w_s[RPR][CS];
    __shared__ float den_s[RPR];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int row = warp * 16 + gq + 8 * h;
#pragma unroll
      for (int dt = 0; dt < DT; ++dt)
        *reinterpret_cast<float2*>(so + row * OS + dt * 8 + 2 * tq) =
            make_float2(o[dt][2 * h], o[dt][2 * h + 1]);
      if (tq == 0) {
        const float mm = h ? m1 : m0;
        sml[row * 2 + 0] = mm == -INFINITY ? -INFINITY : mm * kLn2;
        sml[row * 2 + 1] = h ? l1 : l0;
      }
    }
    cluster_sync_all();   // every split's partials are now visible cluster-wide
    const uint32_t rank = cluster_rank();
    const uint32_t so_u = smem_u32(so), sml_u = smem_u32(sml);
    if (tid < RPR) {
      const int row = static_cast<int>(rank) * RPR + tid;
      float ms[CS], ls[CS];
#pragma unroll
      for (int sp = 0; sp < CS; ++sp) {
        const uint32_t a = dsmem_addr(sml_u + row * 8, sp);
        ms[sp] = dsmem_ld(a);
        ls[sp] = dsmem_ld(a + 4);
      }
      float M = -INFINITY;
#pragma unroll
      for (int sp = 0; sp < CS; ++sp)
        if (ls[sp] > 0.f) M = fmaxf(M, ms[sp]);
      float den = 0.f;
#pragma unroll
      for (int sp = 0; sp < CS; ++sp) {
        const float w = ls[sp] > 0.f ? __expf(ms[sp] - M) : 0.f;
        den = fmaf(ls[sp], w, den);
        w_s[tid][sp] = w;
      }
      den_s[tid] = den;
    }
    __syncthreads();
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out);
    constexpr int C4 = D / 4;
    for (int e = tid; e < RPR * C4; e += 128) {
      const int r = e / C4, c4 = e % C4;
      const int row = static_cast<int>(rank) * RPR + r;
      const int rr = blockIdx.z * kMmaRows + row;
      if (rr >= nrows_all) continue;
      float4 v[CS];
#pragma unroll
      for (int sp = 0; sp < CS; ++sp)
        v[sp] = dsmem_ld4(dsmem_addr(so_u + (row * OS + c4 * 4) * 4, sp));
      float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int sp = 0; sp < CS; ++sp) {
        const float w = w_s[r][sp];
        num.x = fmaf(v[sp].x, w, num.x);
        num.y = fmaf(v[sp].y, w, num.y);
        num.z = fmaf(v[sp].z, w, num.z);
        num.w = fmaf(v[sp].w, w, num.w);
      }
      const float den = den_s[r];
      __nv_bfloat162 lo = __floats2bfloat162_rn(num.x / den, num.y / den);
      __nv_bfloat162 hi = __floats2bfloat162_rn(num.z / den, num.w / den);
      uint2 pk;
      pk.x = *reinterpret_cast<uint32_t*>(&lo);
      pk.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(out + out_row(rr) * D + c4 * 4) = pk;
    }
    cluster_sync_all();   // peers may still be reading this CTA's partials
  }
}

// out[pr][dd] = sum_s o_s e^{m_s - M} / sum_s l_s e^{m_s - M}, splits in a
// fixed order; one thread per output element.
template <typename T>
__global__ void __launch_bounds__(256) attn_combine_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_ml,
                                                           int64_t n_rows, int splits, int D,
                                                           T* __restrict__ out) {
  pdl_wait();
  if (threadIdx.x == 0) pdl_launch();
  const int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (idx >= n_rows * D) return;
  const int64_t pr = idx / D;
  const int dd = static_cast<int>(idx - pr * D);
  const float* ml = part_ml + pr * splits * 2;
  const float* po = part_o + pr * splits * D + dd;
  float M = -INFINITY;
  for (int s = 0; s < splits; ++s)
    if (ml[2 * s + 1] > 0.f) M = fmaxf(M, ml[2 * s]);
  float num = 0.f, den = 0.f;
#pragma unroll 8
  for (int s = 0; s < splits; ++s) {
    const float ls = ml[2 * s + 1];
    const float w = ls > 0.f ? __expf(ml[2 * s] - M) : 0.f;
    den = fmaf(ls, w, den);
    num = fmaf(po[s * D], w, num);
  }
  out[idx] = from_f<T>(num / den);
}

// Dynamic shared memory of the bf16 kernel: the TMA ring (which also takes
// the gathered tiles) and 1 KB of slack for the 1024-byte alignment of the
// swizzled tiles.
static size_t attn_smem_bytes(int d) {
  return static_cast<size_t>(kAttnStages * 2) * kMmaKeys * d * 2 + 1024;
}

// Opt every attention kernel into large dynamic shared memory once (on the
// first call, which must come before any stream capture), allow the
// 16-CTA clusters, and record the largest cluster the device can schedule.
static int g_max_cluster = 8;

template <int D>
static void attn_kernels(const void** ks) {
  ks[0] = reinterpret_cast<const void*>(attn_mma_kernel<D, 0>);
  ks[1] = reinterpret_cast<const void*>(attn_mma_kernel<D, 1>);
  ks[2] = reinterpret_cast<const void*>(attn_mma_kernel<D, 2>);
  ks[3] = reinterpret_cast<const void*>(attn_mma_kernel<D, 4>);
  ks[4] = reinterpret_cast<const void*>(attn_mma_kernel<D, 8>);
  ks[5] = reinterpret_cast<const void*>(attn_mma_kernel<D, 16>);
  ks[6] = reinterpret_cast<const void*>(attn_simt_kernel<float, D>);
}

static cudaError_t allow_smem() {
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    const int bytes = 200 * 1024;
    const void* ks[14];
    attn_kernels<64>(ks);
    attn_kernels<128>(ks + 7);
    for (const void* k : ks) {
      cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (e != cudaSuccess && err == cudaSuccess) err = e;
    }
    // 16-CTA clusters are opt-in; keep them only if one can be resident
    bool ok16 = true;
    for (const void* k : {ks[5], ks[12]})
      ok16 = ok16 && cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                         cudaSuccess;
    if (ok16) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(1, 16, 1);
      cfg.blockDim = dim3(128);
      cfg.dynamicSmemBytes = attn_smem_bytes(128);
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 1;
      attr[0].val.clusterDim.y = 16;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      ok16 = cudaOccupancyMaxActiveClusters(&n, attn_mma_kernel<128, 16>, &cfg) == cudaSuccess &&
             n > 0;
    }
    cudaGetLastError();   // a refused probe leaves no error behind
    g_max_cluster = ok16 ? 16 : 8;
  });
  return err;
}

AttnPlan plan_attn(int dtype, int nb, int B, int Hq, int Hkv, int d, int64_t max_ctx_len) {
  (void)d;
  AttnPlan p{};
  p.rows_per_cta = dtype == DFLASH_BF16 ? kMmaRows : kAttnWarps * kAttnRowsPerWarp;
  const int G = Hq / Hkv;
  p.row_chunks = (B * G + p.rows_per_cta - 1) / p.rows_per_cta;
  const int64_t base = static_cast<int64_t>(nb) * Hkv * p.row_chunks;
  const int64_t want = (2 * kNumSMs + base - 1) / base;
  if (dtype == DFLASH_BF16) {
    // one cluster of 2^k splits (up to 16) per (block, kv head, row chunk);
    // at least 128 context keys per split
    p.cluster = 1;
    if (max_ctx_len <= 0) {
      p.splits = 1;
      p.chunk = 64;
      return p;
    }
    // Each request divides its own context into n splits.  Every CTA pays a
    // fixed cost (Q fragments, ring fill, the cluster merge), so n doubles
    // only while the grid stays within ~2.5 waves of resident CTAs (three
    // per SM) and each split of the longest context keeps at least four
    // 64-key tiles.
    const int64_t slots = 3 * static_cast<int64_t>(kNumSMs);
    int64_t n = 1;
    while (n < 16 && base * (2 * n) * 2 <= 5 * slots && max_ctx_len / (2 * n) >= 4 * kMmaKeys)
      n *= 2;
    while (p.cluster < n) p.cluster *= 2;
    int64_t chunk = (max_ctx_len + p.cluster - 1) / p.cluster;
    p.chunk = static_cast<int>((chunk + 63) / 64 * 64);
    p.splits = p.cluster;
    return p;
  }
  p.cluster = 0;
  if (max_ctx_len <= 0) {
    p.splits = 1;
    p.chunk = 64;
    return p;
  }
  // at least 256 context keys per split: the fp32 partials of a split
  // then stay below the K/V bytes it streams
  const int64_t min_chunk = 256;
  const int64_t max_splits = std::min<int64_t>(64, (max_ctx_len + min_chunk - 1) / min_chunk);
  int64_t splits = std::max<int64_t>(1, std::min(want, max_splits));
  int64_t chunk = (max_ctx_len + splits - 1) / splits;
  chunk = (chunk + 63) / 64 * 64;
  p.chunk = static_cast<int>(chunk);
  p.splits = static_cast<int>((max_ctx_len + chunk - 1) / chunk);
  return p;
}

// Partials in global memory are only needed by the fp32 path and by the
// bf16 fallback when a 16-CTA cluster cannot be scheduled.
size_t attn_ws_bytes(const AttnPlan& p, int nb, int B, int Hq, int d) {
  const size_t rows = static_cast<size_t>(nb) * B * Hq;
  return rows * p.splits * (d + 2) * sizeof(float);
}

template <int D, int CS>
static cudaError_t launch_cluster(const AttnParams& p, dim3 grid, size_t smem, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = CS;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  count_launch();
  return cudaLaunchKernelEx(&cfg, attn_mma_kernel<D, CS>, p);
}

template <int D>
static cudaError_t launch_bf16(const AttnParams& p, int cs, dim3 grid, size_t smem,
                               cudaStream_t st) {
  switch (cs) {
    case 1: return launch_k(attn_mma_kernel<D, 1>, grid, dim3(128), smem, st, p);
    case 2: return launch_cluster<D, 2>(p, grid, smem, st);
    case 4: return launch_cluster<D, 4>(p, grid, smem, st);
    case 8: return launch_cluster<D, 8>(p, grid, smem, st);
    case 16: return launch_cluster<D, 16>(p, grid, smem, st);
    default: return launch_k(attn_mma_kernel<D, 0>, grid, dim3(128), smem, st, p);
  }
}

cudaError_t launch_attn(int dtype, const AttnPlan& plan, int nb, int B, int Hq, int Hkv, int d,
                        const void* q, const void* kb, const void* vb, const void* kc,
                        const void* vc, const int64_t* ctx_off, const int32_t* block_req,
                        void* out, float* ws, uint32_t* status, cudaStream_t st,
                        const int32_t* ctx_len) {
  if (nb <= 0) return cudaSuccess;
  AttnParams p{};
  p.q = q; p.kb = kb; p.vb = vb; p.kc = kc; p.vc = vc;
  p.ctx_off = ctx_off;
  p.ctx_len = ctx_len;
  p.block_req = block_req;
  p.B = B; p.Hq = Hq; p.Hkv = Hkv; p.G = Hq / Hkv;
  p.splits = plan.splits;
  p.chunk = plan.chunk;
  p.rows_per_cta = plan.rows_per_cta;
  p.scale = 1.0f / sqrtf(static_cast<float>(d));
  p.out = out;
  p.status = status;
  const int64_t n_rows = static_cast<int64_t>(nb) * B * Hq;
  p.part_o = ws;
  p.part_ml = ws + static_cast<size_t>(n_rows) * plan.splits * d;
  dim3 grid(nb * Hkv, plan.splits, plan.row_chunks);
  cudaError_t e = allow_smem();
  if (e != cudaSuccess) return e;
  int cs = 0;   // 0: partials through global memory + combine kernel
  if (dtype == DFLASH_BF16) {
    cs = plan.cluster <= g_max_cluster ? plan.cluster : 0;
    // context K/V as 3-D tensors [rows][Hkv][d]; only rows of the requests'
    // contexts are ever loaded, so the row extent is an upper bound
    // (kMaxCacheRows, far above any cache this path is sized for)
    const void* kbase = kc ? kc : kb;
    const void* vbase = vc ? vc : vb;
    if (!encode_tmap_bf16_3d(&p.tm_k, kbase, d, Hkv, kMaxCacheRows, 64, 1, kMmaKeys) ||
        !encode_tmap_bf16_3d(&p.tm_v, vbase, d, Hkv, kMaxCacheRows, 64, 1, kMmaKeys))
      return cudaErrorInvalidValue;
    const size_t smem = attn_smem_bytes(d);
    e = d == 64 ? launch_bf16<64>(p, cs, grid, smem, st) : launch_bf16<128>(p, cs, grid, smem, st);
    if (e != cudaSuccess || cs != 0) return e;
  } else {
    const size_t smem = (static_cast<size_t>(plan.rows_per_cta) * d +
                         kAttnKeyTile * (d + 1) + kAttnKeyTile * d) * sizeof(float);
    e = d == 64 ? launch_k(attn_simt_kernel<float, 64>, grid, dim3(kAttnWarps * 32), smem, st, p)
                : launch_k(attn_simt_kernel<float, 128>, grid, dim3(kAttnWarps * 32), smem, st,
                           p);
    if (e != cudaSuccess) return e;
  }
  const int64_t total = n_rows * d;
  const dim3 cgrid(static_cast<unsigned>((total + 255) / 256));
  if (dtype == DFLASH_BF16)
    return launch_k(attn_combine_kernel<__nv_bfloat16>, cgrid, dim3(256), 0, st, p.part_o,
                    p.part_ml, n_rows, plan.splits, d, static_cast<__nv_bfloat16*>(out));
  return launch_k(attn_combine_kernel<float>, cgrid, dim3(256), 0, st, p.part_o, p.part_ml,
                  n_rows, plan.splits, d, static_cast<float*>(out));
}

}  // namespace dfl
