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
//   warps 0-3     : epilogue (TMEM -> registers -> global), one TMEM lane
//                   (= one weight row) per thread
//
// Split-K writes fp32 partial sums that a fixed-order finish kernel reduces
// (deterministic).  The LM-head variant keeps a per-CTA running (max, index)
// and merges it with one 64-bit atomicMax per token, so logits never reach
// global memory.  fp32 models run on a SIMT FFMA kernel with the same
// partial layout (tensor-core tf32 would miss a 1e-4 tolerance).
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace dfl {

// ===========================================================================
// tcgen05 kernel
// ===========================================================================
namespace tc {

constexpr int BM = 128;          // weight rows per tile (UMMA M)
constexpr int BK = 64;           // bf16 per k-block: one 128-byte swizzle row
constexpr int UK = 16;           // K per tcgen05.mma (kind::f16)
constexpr int A_BYTES = BM * BK * 2;

struct Params {
  CUtensorMap tm_w0, tm_w1, tm_w2;  // weights of up to three segments
  CUtensorMap tm_x;                 // activations [M][K]
  int seg_tile_begin[kMaxSegs + 1]; // row-tile ranges of the segments
  int seg_rows[kMaxSegs];
  int seg_col0[kMaxSegs];
  int nseg;
  int M;
  int kb_total;
  int kb_per_split;
  int n_cols;
  float* partial;                   // [splits][M][n_cols]
  unsigned long long* keys;         // argmax mode: [M]
  uint32_t* status;
};

template <int BN, int STAGES, bool ARGMAX>
__global__ void __launch_bounds__(128, 1) gemm_kernel(const __grid_constant__ Params p) {
  constexpr int B_BYTES = BN * BK * 2;
  constexpr int STAGE = A_BYTES + B_BYTES;
  constexpr uint32_t TMEM_COLS = BN < 32 ? 32 : BN;
  constexpr uint32_t IDESC = idesc_bf16(BM, BN);
  static_assert(STAGE % 1024 == 0, "stages must stay 1024-byte aligned");

  extern __shared__ uint8_t dsmem[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full_bar[STAGES];
  __shared__ __align__(8) uint64_t empty_bar[STAGES];
  __shared__ __align__(8) uint64_t acc_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_flag;
  __shared__ unsigned long long red[ARGMAX ? 4 : 1][ARGMAX ? BN : 1];

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Which weight segment this row tile belongs to.
  const int tile = blockIdx.x;
  int seg = 0;
  while (seg + 1 < p.nseg && tile >= p.seg_tile_begin[seg + 1]) ++seg;
  const int row0 = (tile - p.seg_tile_begin[seg]) * BM;
  const int seg_rows = p.seg_rows[seg];
  const int tok0 = blockIdx.y * BN;
  const int kb0 = blockIdx.z * p.kb_per_split;
  const int kb1 = min(p.kb_total, kb0 + p.kb_per_split);
  const int nkb = kb1 - kb0;
  const CUtensorMap* tmw = seg == 0 ? &p.tm_w0 : (seg == 1 ? &p.tm_w1 : &p.tm_w2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(&acc_bar, 1);
    abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(tmw);
    tma_prefetch_desc(&p.tm_x);
  }
  if (warp == 2) tmem_alloc(&tmem_slot, TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    int issued = 0;
    for (int i = 0; i < nkb; ++i) {
      const int s = i % STAGES;
      if (i >= STAGES) {
        if (!mbar_wait(&empty_bar[s], ((i / STAGES) & 1) ^ 1, p.status, 11)) {
          abort_flag = 1;
          break;
        }
      }
      if (abort_flag) break;
      uint8_t* sa = smem + s * STAGE;
      mbar_arrive_expect_tx(&full_bar[s], STAGE);
      tma_load_2d(sa, tmw, &full_bar[s], (kb0 + i) * BK, row0);
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
  const bool live = ok && !abort_flag;
  const int row = row0 + warp * 32 + lane;
  const uint32_t lane_addr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  if (live) {
#pragma unroll 1
    for (int c = 0; c < BN; c += 16) {
      float v[16];
      tmem_ld16(lane_addr + c, v);
      if constexpr (!ARGMAX) {
        if (row < seg_rows) {
          float* dst = p.partial + (static_cast<size_t>(blockIdx.z) * p.M) * p.n_cols +
                       p.seg_col0[seg] + row;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = tok0 + c + j;
            if (t < p.M) dst[static_cast<size_t>(t) * p.n_cols] = v[j];
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          unsigned long long key = 0ull;
          if (row < seg_rows && tok0 + c + j < p.M) {
            if (!isfinite(v[j])) report(p.status, DFLASH_ENUMERIC, 15);
            key = argmax_key(v[j], static_cast<uint32_t>(row));
          }
          key = warp_max_u64(key);
          if (lane == 0) red[warp][c + j] = key;
        }
      }
    }
  }
  if constexpr (ARGMAX) {
    __syncthreads();
    if (live) {
      for (int j = threadIdx.x; j < BN; j += blockDim.x) {
        unsigned long long k = red[0][j];
#pragma unroll
        for (int w = 1; w < 4; ++w) k = red[w][j] > k ? red[w][j] : k;
        const int t = tok0 + j;
        if (t < p.M && k != 0ull) atomicMax(p.keys + t, k);
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
  gemm_kernel<BN, STAGES, ARGMAX><<<grid, 128, SMEM, st>>>(p);
  count_launch();
  return cudaGetLastError();
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
// SIMT kernel (fp32 models): 64 weight rows x 32 tokens per CTA
// ===========================================================================
namespace simt {

constexpr int TR = 64, TT = 32, TK = 32;

struct Params {
  const void* w[kMaxSegs];
  int seg_tile_begin[kMaxSegs + 1];
  int seg_rows[kMaxSegs];
  int seg_col0[kMaxSegs];
  int nseg;
  const void* x;
  int M, K;
  int k_per_split;
  int n_cols;
  float* partial;
  unsigned long long* keys;
  uint32_t* status;
};

template <typename T, bool ARGMAX>
__global__ void __launch_bounds__(256) gemm_kernel(const Params p) {
  __shared__ float ws[TK][TR + 1];
  __shared__ float xs[TK][TT + 1];
  __shared__ unsigned long long red[16][TT];
  const int tile = blockIdx.x;
  int seg = 0;
  while (seg + 1 < p.nseg && tile >= p.seg_tile_begin[seg + 1]) ++seg;
  const int row0 = (tile - p.seg_tile_begin[seg]) * TR;
  const int rows = p.seg_rows[seg];
  const T* W = static_cast<const T*>(p.w[seg]);
  const T* X = static_cast<const T*>(p.x);
  const int tok0 = blockIdx.y * TT;
  const int k0 = blockIdx.z * p.k_per_split;
  const int k1 = min(p.K, k0 + p.k_per_split);
  const int tid = threadIdx.x;
  const int ty = tid >> 4, tx = tid & 15;   // rows ty + 16i, tokens tx + 16j
  float acc[4][2] = {};
  for (int kk = k0; kk < k1; kk += TK) {
    for (int e = tid; e < TR * TK; e += 256) {
      const int r = e / TK, k = e % TK;
      const int gr = row0 + r, gk = kk + k;
      ws[k][r] = (gr < rows && gk < k1) ? to_f(W[static_cast<size_t>(gr) * p.K + gk]) : 0.f;
    }
    for (int e = tid; e < TT * TK; e += 256) {
      const int t = e / TK, k = e % TK;
      const int gt = tok0 + t, gk = kk + k;
      xs[k][t] = (gt < p.M && gk < k1) ? to_f(X[static_cast<size_t>(gt) * p.K + gk]) : 0.f;
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
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = row0 + ty + 16 * i, t = tok0 + tx + 16 * j;
        if (r < rows && t < p.M) {
          if (!isfinite(acc[i][j])) report(p.status, DFLASH_ENUMERIC, 16);
          const unsigned long long k = argmax_key(acc[i][j], static_cast<uint32_t>(r));
          best = k > best ? k : best;
        }
      }
      red[ty][tx + 16 * j] = best;
    }
    __syncthreads();
    if (tid < TT) {
      unsigned long long best = 0ull;
      for (int y = 0; y < 16; ++y) best = red[y][tid] > best ? red[y][tid] : best;
      if (tok0 + tid < p.M && best) atomicMax(p.keys + tok0 + tid, best);
    }
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

int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

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

GemmPlan plan_gemm(int dtype, const int* seg_rows, int nseg, int64_t M, int K) {
  GemmPlan pl{};
  pl.n_cols = 0;
  int row_tiles = 0;
  const int tr = dtype == DFLASH_BF16 ? tc::BM : simt::TR;
  for (int s = 0; s < nseg; ++s) {
    pl.n_cols += seg_rows[s];
    row_tiles += ceil_div(seg_rows[s], tr);
  }
  int kb_total, target;
  if (dtype == DFLASH_BF16) {
    pl.bn = tc::pick_bn(M);
    kb_total = ceil_div(K, tc::BK);
    target = kNumSMs * tc::ctas_per_sm(pl.bn);
  } else {
    pl.bn = simt::TT;
    kb_total = ceil_div(K, simt::TK);
    target = kNumSMs * 4;
  }
  const int tiles = row_tiles * ceil_div(M, pl.bn);
  int splits = 1;
  if (tiles < target) splits = std::min(kb_total, ceil_div(target, tiles));
  splits = std::max(1, std::min(splits, 32));
  pl.kb_per_split = ceil_div(kb_total, splits);
  pl.splits = ceil_div(kb_total, pl.kb_per_split);
  return pl;
}

cudaError_t launch_gemm_partial(int dtype, const GemmSeg* segs, int nseg, const void* X,
                                int64_t M, int K, const GemmPlan& pl, float* partial,
                                uint32_t* status, cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  if (dtype == DFLASH_BF16) {
    tc::Params p{};
    CUtensorMap* maps[3] = {&p.tm_w0, &p.tm_w1, &p.tm_w2};
    int tiles = 0;
    for (int s = 0; s < nseg; ++s) {
      if (!encode_tmap_bf16_2d(maps[s], segs[s].w, K, segs[s].rows, tc::BK, tc::BM))
        return cudaErrorInvalidValue;
      p.seg_tile_begin[s] = tiles;
      p.seg_rows[s] = segs[s].rows;
      p.seg_col0[s] = s == 0 ? 0 : p.seg_col0[s - 1] + segs[s - 1].rows;
      tiles += ceil_div(segs[s].rows, tc::BM);
    }
    p.seg_tile_begin[nseg] = tiles;
    if (!encode_tmap_bf16_2d(&p.tm_x, X, K, M, tc::BK, pl.bn)) return cudaErrorInvalidValue;
    p.nseg = nseg;
    p.M = static_cast<int>(M);
    p.kb_total = ceil_div(K, tc::BK);
    p.kb_per_split = pl.kb_per_split;
    p.n_cols = pl.n_cols;
    p.partial = partial;
    p.status = status;
    dim3 grid(tiles, ceil_div(M, pl.bn), pl.splits);
    return tc::dispatch<false>(pl.bn, p, grid, st);
  }
  simt::Params p{};
  int tiles = 0;
  for (int s = 0; s < nseg; ++s) {
    p.w[s] = segs[s].w;
    p.seg_tile_begin[s] = tiles;
    p.seg_rows[s] = segs[s].rows;
    p.seg_col0[s] = s == 0 ? 0 : p.seg_col0[s - 1] + segs[s - 1].rows;
    tiles += ceil_div(segs[s].rows, simt::TR);
  }
  p.seg_tile_begin[nseg] = tiles;
  p.nseg = nseg;
  p.x = X;
  p.M = static_cast<int>(M);
  p.K = K;
  p.k_per_split = pl.kb_per_split * simt::TK;
  p.n_cols = pl.n_cols;
  p.partial = partial;
  p.status = status;
  dim3 grid(tiles, ceil_div(M, simt::TT), pl.splits);
  simt::gemm_kernel<float, false><<<grid, 256, 0, st>>>(p);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_lmhead_argmax(int dtype, const void* W, int V, const void* X, int64_t M,
                                 int K, unsigned long long* keys, uint32_t* status,
                                 cudaStream_t st) {
  if (M <= 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(keys, 0, sizeof(unsigned long long) * M, st);
  if (e != cudaSuccess) return e;
  if (dtype == DFLASH_BF16) {
    tc::Params p{};
    if (!encode_tmap_bf16_2d(&p.tm_w0, W, K, V, tc::BK, tc::BM)) return cudaErrorInvalidValue;
    const int bn = tc::pick_bn(M);
    if (!encode_tmap_bf16_2d(&p.tm_x, X, K, M, tc::BK, bn)) return cudaErrorInvalidValue;
    p.seg_tile_begin[0] = 0;
    p.seg_tile_begin[1] = ceil_div(V, tc::BM);
    p.seg_rows[0] = V;
    p.nseg = 1;
    p.M = static_cast<int>(M);
    p.kb_total = ceil_div(K, tc::BK);
    p.kb_per_split = p.kb_total;
    p.keys = keys;
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
  p.status = status;
  dim3 grid(ceil_div(V, simt::TR), ceil_div(M, simt::TT), 1);
  simt::gemm_kernel<float, true><<<grid, 256, 0, st>>>(p);
  count_launch();
  return cudaGetLastError();
}

// ===========================================================================
// finish: fixed-order split reduction + epilogue op
// ===========================================================================
template <typename T>
__global__ void __launch_bounds__(256) finish_kernel(const EpiParams p) {
  // output columns of all active segments, concatenated
  int out_cols = 0;
  for (int s = 0; s < p.nseg; ++s)
    if (p.seg[s].op != EPI_NONE) out_cols += p.seg[s].rows;
  const int64_t total = p.M * out_cols;
  const size_t split_stride = static_cast<size_t>(p.M) * p.n_cols;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t m = idx / out_cols;
    int c = static_cast<int>(idx % out_cols);
    int s = 0;
    while (p.seg[s].op == EPI_NONE || c >= p.seg[s].rows) {
      if (p.seg[s].op != EPI_NONE) c -= p.seg[s].rows;
      ++s;
    }
    const EpiSeg& sg = p.seg[s];
    const float* src = p.partial + static_cast<size_t>(m) * p.n_cols + sg.col0;
    float v = 0.f;
    for (int k = 0; k < p.splits; ++k) v += src[k * split_stride + c];
    if (sg.op == EPI_RESID) {
      float* h = static_cast<float*>(sg.out) + m * sg.out_stride + c;
      *h = *h + v;
      continue;
    }
    if (sg.op == EPI_SWIGLU) {
      const float* up = p.partial + static_cast<size_t>(m) * p.n_cols + p.seg[s + 1].col0;
      float u = 0.f;
      for (int k = 0; k < p.splits; ++k) u += up[k * split_stride + c];
      const float a = v / (1.f + __expf(-v)) * u;
      static_cast<T*>(sg.out)[m * sg.out_stride + c] = from_f<T>(a);
      continue;
    }
    // EPI_STORE
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
    const int64_t orow = sg.use_dst ? p.dst_row[m] : m;
    static_cast<T*>(sg.out)[orow * sg.out_stride + c] = from_f<T>(v);
  }
}

cudaError_t launch_gemm_finish(const EpiParams& p, cudaStream_t st) {
  int out_cols = 0;
  for (int s = 0; s < p.nseg; ++s)
    if (p.seg[s].op != EPI_NONE) out_cols += p.seg[s].rows;
  const int64_t total = p.M * out_cols;
  if (total <= 0) return cudaSuccess;
  const int64_t want = (total + 255) / 256;
  const int grid = static_cast<int>(std::min<int64_t>(want, kNumSMs * 16));
  if (p.out_bf16)
    finish_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(p);
  else
    finish_kernel<float><<<grid, 256, 0, st>>>(p);
  count_launch();
  return cudaGetLastError();
}

}  // namespace dfl
