// Block pooling (step 1), block scoring (step 2) and top-k block selection
// (step 3) of dynamic block-sparse attention.
//
// Pooling estimates each block's activation by the mean of its rows (the
// "DeepSeek NSA" article, section 2.1, decides activation per 32x32 block with
// a light estimate; the zblog.xzdbk.com/559 post, section
// 硬件友好的稀疏计算实现, decides per 64x64 block). Scores and the ranking stay
// in fp32 ("DeepSeek NSA", section 2.2). Selection keeps the forced local
// window and sink blocks plus the top-k remaining causal blocks (zblog post,
// section 基于Top-k选择的局部-全局混合), ties going to the lower block index.
//
// All three steps are memory-bound (pooling reads every Q and K element
// once) or small (scores: Hq * nb^2 / 2 dot products of length d), so they run
// on the CUDA cores with 16-byte vector loads.
#include "dsa_internal.cuh"
#include "select_row.cuh"

namespace dsa {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kSelWarps = 8;  // rows per CTA in the score/select kernels
constexpr int kSelThreads = kSelWarps * 32;

__device__ __forceinline__ uint4 load_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void add_bf16x2(float& a, float& b, uint32_t w) {
  a += __uint_as_float(w << 16);
  b += __uint_as_float(w & 0xffff0000u);
}

// ---------------------------------------------------------------------------
// Step 1: pooled[blk, :] = (1/BS) * sum of the BS rows of block blk.
// One CTA per block. Thread (rr, c) sums rows rr, rr+RPP, ... of 16-byte
// column chunk c in fp32, in that order; the RPP partial rows are then added
// in row order. Q blocks come first in the grid, then K blocks.
// ---------------------------------------------------------------------------
template <int D, int BS>
__device__ __forceinline__ void pool_block(const __nv_bfloat16* __restrict__ src, float* __restrict__ dst) {
  constexpr int CH = D / 8;
  constexpr int RPP = kPoolThreads / CH;
  constexpr int ROWS = BS / RPP;
  static_assert(BS % RPP == 0 && ROWS >= 1, "block/dim combination");
  __shared__ float part[RPP][D + 4];
  const int c = threadIdx.x % CH;
  const int rr = threadIdx.x / CH;
  uint4 v[ROWS];
#pragma unroll
  for (int r = 0; r < ROWS; ++r) v[r] = load_stream16(src + (size_t)(rr + r * RPP) * D + c * 8);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int r = 0; r < ROWS; ++r) {
    add_bf16x2(acc[0], acc[1], v[r].x);
    add_bf16x2(acc[2], acc[3], v[r].y);
    add_bf16x2(acc[4], acc[5], v[r].z);
    add_bf16x2(acc[6], acc[7], v[r].w);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rr][c * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float sum = 0.f;
#pragma unroll 8
    for (int r = 0; r < RPP; ++r) sum += part[r][threadIdx.x];
    dst[threadIdx.x] = sum * (1.0f / BS);
  }
}

template <int D, int BS>
__global__ void __launch_bounds__(kPoolThreads)
pool_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
            float* __restrict__ qp, float* __restrict__ kp, long long n_qblocks) {
  long long blk = blockIdx.x;
  if (blk < n_qblocks) {
    pool_block<D, BS>(q + blk * (long long)(BS * D), qp + blk * D);
  } else {
    blk -= n_qblocks;
    pool_block<D, BS>(k + blk * (long long)(BS * D), kp + blk * D);
  }
}

// Key blocks j0 .. j0+nj-1 of every (batch, KV head) of a cache of nb blocks.
template <int D, int BS>
__global__ void __launch_bounds__(kPoolThreads)
pool_range_kernel(const __nv_bfloat16* __restrict__ k, float* __restrict__ kp, int nb, int j0, int nj) {
  const long long bg = blockIdx.x / nj;
  const long long blk = bg * nb + j0 + blockIdx.x % nj;
  pool_block<D, BS>(k + blk * (long long)(BS * D), kp + blk * D);
}

// ---------------------------------------------------------------------------
// Step 2 (+3 when FUSED): one CTA scores kRowTile pooled query rows against the
// pooled key rows 0..jmax of their KV head, as a tiled fp32 GEMM, then selects
// each row from the scores held in shared memory (or writes them out).
// Rows are heads [h0, h0+HB) of one KV group times query blocks [i0, i0+RB),
// HB * RB <= kRowTile. A score is the fp32 sum of two fused multiply-add
// chains, over the even and over the odd d in increasing order; both the fused
// and the split path run this kernel, so they agree bit for bit.
// ---------------------------------------------------------------------------
constexpr int kRowTile = 32;   // query rows per CTA
constexpr int kColTile = 128;  // key blocks per column pass
constexpr int kDTile = 32;     // head-dim slice per pass over the key tile
template <int D>
struct QStride {
  static constexpr int value = D + 4;
};
constexpr int kKStride = kDTile + 4;

struct RowTile {
  int b, kvh, h0, i0;
};

__device__ __forceinline__ RowTile row_tile(const Shape& s, int HB, int RB) {
  const int n_hc = (s.group + HB - 1) / HB;
  const int n_ic = (s.nb + RB - 1) / RB;
  int x = blockIdx.x;
  // largest query blocks first: they have the most candidates
  const int ic = n_ic - 1 - (x % n_ic);
  x /= n_ic;
  const int hc = x % n_hc;
  x /= n_hc;
  const int kvh = x % s.Hkv;
  const int b = x / s.Hkv;
  RowTile t;
  t.b = b;
  t.kvh = kvh;
  t.h0 = kvh * s.group + hc * HB;
  t.i0 = ic * RB;
  return t;
}

// Shared memory: qs [kRowTile][D+4] and ks [kColTile][kDTile+4] during the
// GEMM, reused as the selection histograms [kSelWarps][256] afterwards; then
// sc [kRowTile][nb].
template <int D>
size_t score_smem_bytes(int nb) {
  const size_t gemm = (size_t)(kRowTile * QStride<D>::value + kColTile * kKStride) * sizeof(float);
  static_assert((size_t)(kRowTile * QStride<D>::value + kColTile * kKStride) >= (size_t)kSelWarps * kHistWords,
                "the histograms fit in the GEMM buffers");
  return gemm + (size_t)kRowTile * nb * sizeof(float);
}

// Blocks per lane of a selection row: ceil(nb / 32) rounded up to 8, 16 or 32.
inline int select_tmax(int nb) { return nb <= 256 ? 8 : nb <= 512 ? 16 : 32; }

template <int D, bool FUSED, int TMAX>
__global__ void __launch_bounds__(kSelThreads)
score_kernel(Shape s, KBudget kb, int HB, int RB, const float* __restrict__ qp,
             const float* __restrict__ kp, float* __restrict__ scores, int32_t* __restrict__ idx,
             int32_t* __restrict__ cnt, WsHeader* hdr) {
  extern __shared__ float sm_f[];
  constexpr int QS = QStride<D>::value;
  float* const qs = sm_f;                                   // [kRowTile][QS]
  float* const ks = sm_f + kRowTile * QS;                   // [kColTile][kKStride]
  const size_t lead = (size_t)kRowTile * QS + kColTile * kKStride;
  uint32_t* const sk = reinterpret_cast<uint32_t*>(sm_f);  // [kSelWarps][256], after the GEMM
  float* const sc = sm_f + lead;                            // [kRowTile][nb]
  const RowTile tile = row_tile(s, HB, RB);
  const int h_end = min(tile.h0 + HB, (tile.kvh + 1) * s.group);
  const int i_end = min(tile.i0 + RB, s.nb);
  const int tid = threadIdx.x;

  // tile row r -> (h, i); rows outside the problem hold zeros and are never read back
  for (int e = tid; e < kRowTile * (D / 4); e += kSelThreads) {
    const int r = e / (D / 4), c4 = e % (D / 4);
    const int h = tile.h0 + r / RB, i = tile.i0 + r % RB;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r < HB * RB && h < h_end && i < i_end)
      v = *reinterpret_cast<const float4*>(qp + (((size_t)tile.b * s.Hq + h) * s.nb + i) * D + 4 * c4);
    *reinterpret_cast<float4*>(qs + r * QS + 4 * c4) = v;
  }

  // thread (rg, cg) owns rows rg + 8u (u < 4) and columns cg + 32v (v < 4) of
  // each column pass; the strides keep the shared loads free of bank conflicts
  const int rg = tid % 8, cg = tid / 8;
  const int jmax = i_end - 1;
  const float* const kbase = kp + ((size_t)tile.b * s.Hkv + tile.kvh) * s.nb * D;
  // the key tile streams through shared memory one (column pass, d slice) at a
  // time; the next slice is fetched into registers while this one is used
  constexpr int kSlices = D / kDTile;
  constexpr int kLoads = kColTile * (kDTile / 4) / kSelThreads;  // float4 per thread per slice
  const int n_pass = jmax / kColTile + 1;
  float4 nxt[kLoads];
  auto fetch = [&](int pass, int slice) {
#pragma unroll
    for (int u = 0; u < kLoads; ++u) {
      const int e = tid + u * kSelThreads;
      const int col = e / (kDTile / 4), d4 = e % (kDTile / 4);
      const int j = pass * kColTile + col;
      nxt[u] = j <= jmax ? __ldg(reinterpret_cast<const float4*>(kbase + (size_t)j * D + slice * kDTile) + d4)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  fetch(0, 0);
  for (int pass = 0; pass < n_pass; ++pass) {
    const int jc = pass * kColTile;
    float2 acc[4][4];  // partial sums over even and odd d
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = make_float2(0.f, 0.f);
    for (int sl = 0; sl < kSlices; ++sl) {
      __syncthreads();  // the previous slice has been consumed (and qs is complete)
#pragma unroll
      for (int u = 0; u < kLoads; ++u) {
        const int e = tid + u * kSelThreads;
        const int col = e / (kDTile / 4), d4 = e % (kDTile / 4);
        *reinterpret_cast<float4*>(ks + col * kKStride + 4 * d4) = nxt[u];
      }
      __syncthreads();
      if (sl + 1 < kSlices) fetch(pass, sl + 1);
      else if (pass + 1 < n_pass) fetch(pass + 1, 0);
      const int dc = sl * kDTile;
#pragma unroll 2
      for (int d4 = 0; d4 < kDTile / 4; ++d4) {
        float4 qv[4], kv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) qv[u] = *reinterpret_cast<const float4*>(qs + (rg + 8 * u) * QS + dc + 4 * d4);
#pragma unroll
        for (int v = 0; v < 4; ++v) kv[v] = *reinterpret_cast<const float4*>(ks + (cg + 32 * v) * kKStride + 4 * d4);
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            acc[u][v] = __ffma2_rn(make_float2(qv[u].x, qv[u].y), make_float2(kv[v].x, kv[v].y), acc[u][v]);
            acc[u][v] = __ffma2_rn(make_float2(qv[u].z, qv[u].w), make_float2(kv[v].z, kv[v].w), acc[u][v]);
          }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = rg + 8 * u;
      const int i = tile.i0 + r % RB;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int j = jc + cg + 32 * v;
        if (j <= jmax) sc[r * s.nb + j] = (j <= i) ? __fadd_rn(acc[u][v].x, acc[u][v].y) : -INFINITY;
      }
    }
  }
  __syncthreads();  // all scores written; qs/ks are free for the selection scratch

  const int warp = tid / 32, lane = tid % 32;
  if (FUSED && s.group_select) {
    // one list per query block of the tile: the tile holds every head of the
    // KV group (rows u * RB + ii); their scores are added in head order into
    // the first head's row, and the list goes to all of them
    for (int ii = warp; ii < RB; ii += kSelWarps) {
      const int i = tile.i0 + ii;
      if (i >= i_end) continue;
      float* const row0 = sc + ii * s.nb;
      for (int j = lane; j <= i; j += 32) {
        float a = row0[j];
        for (int u = 1; u < HB; ++u) a = __fadd_rn(a, sc[(u * RB + ii) * s.nb + j]);
        row0[j] = a;
      }
      __syncwarp();
      const size_t row = ((size_t)tile.b * s.Hq + tile.h0) * s.nb + i;
      select_row<TMAX>(row0, sk + warp * kHistWords, i, kb.k[0], s.lw, s.ns, s.W, s.tau, s.c2,
                       idx + row * s.W, cnt + row, HB, (size_t)s.nb * s.W, (size_t)s.nb, hdr, lane);
    }
    return;
  }
  for (int r = warp; r < kRowTile; r += kSelWarps) {
    const int h = tile.h0 + r / RB, i = tile.i0 + r % RB;
    if (r >= HB * RB || h >= h_end || i >= i_end) continue;
    const size_t row = ((size_t)tile.b * s.Hq + h) * s.nb + i;
    if (FUSED) {
      const int k = s.per_head ? kb.k[h] : kb.k[0];
      select_row<TMAX>(sc + r * s.nb, sk + warp * kHistWords, i, k, s.lw, s.ns, s.W, s.tau, s.c2,
                       idx + row * s.W, cnt + row, 1, 0, 0, hdr, lane);
    } else {
      float* dst = scores + row * s.nb;
      for (int j = lane; j < s.nb; j += 32) dst[j] = (j <= i) ? sc[r * s.nb + j] : -INFINITY;
    }
  }
}

// Selection on caller scores: one warp per row (b, h, i), or with the
// group-shared rule per (b, KV head, i) from the group's scores added in head
// order (the same fp32 additions as the fused kernel).
template <int TMAX>
__global__ void __launch_bounds__(kSelThreads)
select_kernel(Shape s, KBudget kb, const float* __restrict__ scores, int32_t* __restrict__ idx,
              int32_t* __restrict__ cnt, WsHeader* hdr, long long n_rows) {
  extern __shared__ float sm_f[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long row = (long long)blockIdx.x * kSelWarps + warp;
  if (row >= n_rows) return;
  const int i = (int)(row % s.nb);
  float* sc = sm_f + warp * s.nb;
  uint32_t* sk = reinterpret_cast<uint32_t*>(sm_f + kSelWarps * s.nb) + warp * kHistWords;
  if (s.group_select) {
    const long long bk = row / s.nb;  // b * Hkv + KV head
    const size_t head0 = (size_t)bk * s.group;  // b * Hq + first query head of the group
    for (int j = lane; j <= i; j += 32) {
      float a = scores[(head0 * s.nb + i) * s.nb + j];
      for (int u = 1; u < s.group; ++u) a = __fadd_rn(a, scores[((head0 + u) * s.nb + i) * s.nb + j]);
      sc[j] = a;
    }
    __syncwarp();
    const size_t out = head0 * s.nb + i;
    select_row<TMAX>(sc, sk, i, kb.k[0], s.lw, s.ns, s.W, s.tau, s.c2, idx + out * s.W, cnt + out,
                     s.group, (size_t)s.nb * s.W, (size_t)s.nb, hdr, lane);
    return;
  }
  const int h = (int)((row / s.nb) % s.Hq);
  const float* src = scores + (size_t)row * s.nb;
  for (int j = lane; j <= i; j += 32) sc[j] = src[j];
  __syncwarp();
  const int k = s.per_head ? kb.k[h] : kb.k[0];
  select_row<TMAX>(sc, sk, i, k, s.lw, s.ns, s.W, s.tau, s.c2, idx + (size_t)row * s.W, cnt + row, 1, 0,
                   0, hdr, lane);
}

void row_tiling(const Shape& s, int& HB, int& RB) {
  HB = s.group < kRowTile ? s.group : kRowTile;
  RB = kRowTile / HB;
  if (RB < 1) RB = 1;
}

int score_grid(const Shape& s, int HB, int RB) {
  const int n_hc = (s.group + HB - 1) / HB;
  const int n_ic = (s.nb + RB - 1) / RB;
  return s.B * s.Hkv * n_hc * n_ic;
}

template <int D, bool FUSED>
cudaError_t launch_score_d(const Shape& s, const KBudget& kb, const float* qp, const float* kp,
                           float* scores, int32_t* idx, int32_t* cnt, WsHeader* hdr, cudaStream_t st) {
  int HB, RB;
  row_tiling(s, HB, RB);
  const size_t smem = score_smem_bytes<D>(s.nb);
  const int grid = score_grid(s, HB, RB);
  auto f = select_tmax(s.nb) == 8 ? score_kernel<D, FUSED, 8>
           : select_tmax(s.nb) == 16 ? score_kernel<D, FUSED, 16> : score_kernel<D, FUSED, 32>;
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  f<<<grid, kSelThreads, smem, st>>>(s, kb, HB, RB, qp, kp, scores, idx, cnt, hdr);
  return cudaGetLastError();
}

template <bool FUSED>
cudaError_t launch_score_impl(const Shape& s, const KBudget& kb, const float* qp, const float* kp,
                              float* scores, int32_t* idx, int32_t* cnt, WsHeader* hdr,
                              cudaStream_t st) {
  if (s.d == 64) return launch_score_d<64, FUSED>(s, kb, qp, kp, scores, idx, cnt, hdr, st);
  return launch_score_d<128, FUSED>(s, kb, qp, kp, scores, idx, cnt, hdr, st);
}

}  // namespace

cudaError_t launch_pool(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k, float* qp,
                        float* kp, cudaStream_t st) {
  const long long nq = (long long)s.B * s.Hq * s.nb;
  const long long nk = (long long)s.B * s.Hkv * s.nb;
  const long long grid = nq + nk;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
#define DSA_POOL_CASE(D_, BS_)                                                        \
  if (s.d == D_ && s.bs == BS_) {                                                     \
    pool_kernel<D_, BS_><<<(unsigned)grid, kPoolThreads, 0, st>>>(q, k, qp, kp, nq);  \
    return cudaGetLastError();                                                        \
  }
  DSA_POOL_CASE(64, 32)
  DSA_POOL_CASE(64, 64)
  DSA_POOL_CASE(64, 128)
  DSA_POOL_CASE(128, 32)
  DSA_POOL_CASE(128, 64)
  DSA_POOL_CASE(128, 128)
#undef DSA_POOL_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_pool_range(const Shape& s, const __nv_bfloat16* k, float* kp, int j0, int j1,
                              cudaStream_t st) {
  const int nj = j1 - j0;
  const long long grid = (long long)s.B * s.Hkv * nj;
  if (nj <= 0) return cudaSuccess;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
#define DSA_POOL_CASE(D_, BS_)                                                                 \
  if (s.d == D_ && s.bs == BS_) {                                                              \
    pool_range_kernel<D_, BS_><<<(unsigned)grid, kPoolThreads, 0, st>>>(k, kp, s.nb, j0, nj);   \
    return cudaGetLastError();                                                                 \
  }
  DSA_POOL_CASE(64, 32)
  DSA_POOL_CASE(64, 64)
  DSA_POOL_CASE(64, 128)
  DSA_POOL_CASE(128, 32)
  DSA_POOL_CASE(128, 64)
  DSA_POOL_CASE(128, 128)
#undef DSA_POOL_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_scores(const Shape& s, const float* qp, const float* kp, float* scores,
                          cudaStream_t st) {
  KBudget kb{};
  return launch_score_impl<false>(s, kb, qp, kp, scores, nullptr, nullptr, nullptr, st);
}

cudaError_t launch_score_select(const Shape& s, const KBudget& kb, const float* qp, const float* kp,
                                int32_t* idx, int32_t* cnt, WsHeader* hdr, cudaStream_t st) {
  return launch_score_impl<true>(s, kb, qp, kp, nullptr, idx, cnt, hdr, st);
}

cudaError_t launch_select(const Shape& s, const KBudget& kb, const float* scores, int32_t* idx,
                          int32_t* cnt, WsHeader* hdr, cudaStream_t st) {
  const long long n_rows = (long long)s.B * (s.group_select ? s.Hkv : s.Hq) * s.nb;
  const long long grid = (n_rows + kSelWarps - 1) / kSelWarps;
  const size_t smem = (size_t)kSelWarps * (s.nb + kHistWords) * sizeof(float);
  auto f = select_tmax(s.nb) == 8 ? select_kernel<8> : select_tmax(s.nb) == 16 ? select_kernel<16> : select_kernel<32>;
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  f<<<(unsigned)grid, kSelThreads, smem, st>>>(s, kb, scores, idx, cnt, hdr, n_rows);
  return cudaGetLastError();
}

}  // namespace dsa
