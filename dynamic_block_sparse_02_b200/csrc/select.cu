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

namespace dsa {
namespace {

constexpr int kPoolThreads = 256;
constexpr int kSelWarps = 8;  // rows per CTA in the score/select kernels
constexpr int kSelThreads = kSelWarps * 32;
constexpr unsigned kFull = 0xffffffffu;

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
__global__ void __launch_bounds__(kPoolThreads)
pool_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
            float* __restrict__ qp, float* __restrict__ kp, long long n_qblocks) {
  constexpr int CH = D / 8;
  constexpr int RPP = kPoolThreads / CH;
  constexpr int ROWS = BS / RPP;
  static_assert(BS % RPP == 0 && ROWS >= 1, "block/dim combination");
  __shared__ float part[RPP][D + 4];

  long long blk = blockIdx.x;
  const __nv_bfloat16* src;
  float* dst;
  if (blk < n_qblocks) {
    src = q + blk * (long long)(BS * D);
    dst = qp + blk * D;
  } else {
    blk -= n_qblocks;
    src = k + blk * (long long)(BS * D);
    dst = kp + blk * D;
  }
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
    float s = 0.f;
#pragma unroll 8
    for (int r = 0; r < RPP; ++r) s += part[r][threadIdx.x];
    dst[threadIdx.x] = s * (1.0f / BS);
  }
}

// ---------------------------------------------------------------------------
// Step 2: the block score of one pooled query row and one pooled key row.
// Four fp32 partial sums over d (d = 4t+0 .. 4t+3), fused multiply-adds in
// increasing t, combined as (x + y) + (z + w). Every kernel that produces a
// score calls this function, so the split and the fused paths agree bit for
// bit.
// ---------------------------------------------------------------------------
template <int D, int R>
__device__ __forceinline__ void score_rows(const float* __restrict__ qs /*smem [R][D]*/,
                                           const float* __restrict__ kp_row, float (&out)[R]) {
  float4 a[R];
#pragma unroll
  for (int r = 0; r < R; ++r) a[r] = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4* k4 = reinterpret_cast<const float4*>(kp_row);
#pragma unroll 4
  for (int t = 0; t < D / 4; ++t) {
    const float4 kv = __ldg(k4 + t);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const float4 qv = reinterpret_cast<const float4*>(qs + r * D)[t];
      a[r].x = __fmaf_rn(qv.x, kv.x, a[r].x);
      a[r].y = __fmaf_rn(qv.y, kv.y, a[r].y);
      a[r].z = __fmaf_rn(qv.z, kv.z, a[r].z);
      a[r].w = __fmaf_rn(qv.w, kv.w, a[r].w);
    }
  }
#pragma unroll
  for (int r = 0; r < R; ++r) out[r] = __fadd_rn(__fadd_rn(a[r].x, a[r].y), __fadd_rn(a[r].z, a[r].w));
}

// Map a score to an unsigned key whose order is the fp32 order (-0 == +0).
// Every finite score maps to a key >= 0x00800000, so 0 can mark "not a
// candidate".
__device__ __forceinline__ uint32_t ordered_key(float f) {
  if (f == 0.f) f = 0.f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------------------
// Step 3: selection of one row (b, h, i) by one warp.
// s: the row's scores s[0..i] (shared memory); skey: per-warp scratch of at
// least i+1 words. Writes idx_row[0..W) (kept blocks ascending, then -1) and
// *cnt_out.
//
// Candidates are the causal blocks outside the forced set; lane l owns blocks
// l, l+32, l+64, ... The k best (larger fp32 score first, lower block index on
// ties) are found in three steps:
//  1. a lower bound L on the k-th best key: with r = ceil(k/32), every lane's
//     r-th largest key is >= the minimum of those over the warp, so at least
//     32r >= k keys are >= L (L = 0, no bound, when some lane has fewer than
//     r candidates or r > 4);
//  2. the candidates with key >= L ("survivors") are compacted into skey;
//  3. a most-significant-bit-first radix select over the survivors, starting
//     at the highest bit in which they differ, finds the threshold prefix;
//     equal keys left at the end are taken in increasing block index.
// ---------------------------------------------------------------------------
__device__ __forceinline__ bool is_forced(int j, int win_lo, int ns) { return j >= win_lo || j < ns; }

__device__ void select_row(const float* s, uint32_t* skey, int i, int k, int lw, int ns, int W,
                           int32_t* __restrict__ idx_row, int32_t* __restrict__ cnt_out,
                           WsHeader* hdr, int lane) {
  const int n = i + 1;
  const int win_lo = lw > 0 ? max(0, i - lw + 1) : n;  // window = [win_lo, i]
  const int nforced = (n - win_lo) + min(ns, win_lo);
  const int ncand = n - nforced;
  const int keff = min(k, ncand);
  const int T = (n + 31) >> 5;
  const uint32_t lt = (1u << lane) - 1u;

  uint32_t surv = 0;          // bit t: block lane + 32t is a survivor
  uint32_t prefix = 0, pmask = 0;
  int need = keff;
  if (keff > 0 && keff < ncand) {
    // 1. lower bound from each lane's r-th largest key
    const int r = (keff + 31) >> 5;
    uint32_t L = 0;
    if (r <= 4) {
      uint32_t t0 = 0, t1 = 0, t2 = 0, t3 = 0;  // this lane's largest keys, descending
      for (int t = 0; t < T; ++t) {
        const int j = t * 32 + lane;
        if (j < n && !is_forced(j, win_lo, ns)) {
          uint32_t v = ordered_key(s[j]), u;
          u = max(t0, v); v = min(t0, v); t0 = u;
          u = max(t1, v); v = min(t1, v); t1 = u;
          u = max(t2, v); v = min(t2, v); t2 = u;
          t3 = max(t3, v);
        }
      }
      const uint32_t mine = r == 1 ? t0 : r == 2 ? t1 : r == 3 ? t2 : t3;
      L = __reduce_min_sync(kFull, mine);
    }
    // 2. compact the survivors' keys
    int m = 0;
    for (int t = 0; t < T; ++t) {
      const int j = t * 32 + lane;
      uint32_t key = 0;
      if (j < n && !is_forced(j, win_lo, ns)) key = ordered_key(s[j]);
      const bool sv = key != 0u && key >= L;
      const uint32_t bm = __ballot_sync(kFull, sv);
      if (sv) skey[m + __popc(bm & lt)] = key;
      surv |= (uint32_t)sv << t;
      m += __popc(bm);
    }
    __syncwarp();
    // 3. radix select over the survivors from their highest differing bit
    const uint32_t k0 = skey[0];
    uint32_t diff = 0;
    for (int u = lane; u < m; u += 32) diff |= skey[u] ^ k0;
    diff = __reduce_or_sync(kFull, diff);
    if (diff == 0u) {
      pmask = 0xffffffffu;  // all survivors equal: lowest indices win
      prefix = k0;
    } else {
      const int hb = 31 - __clz(diff);
      pmask = hb == 31 ? 0u : ~((2u << hb) - 1u);
      prefix = k0 & pmask;
      int msurv = m;
      for (int bit = hb; bit >= 0 && msurv != need; --bit) {
        const uint32_t bb = 1u << bit;
        int c = 0;
        for (int u = lane; u < m; u += 32) {
          const uint32_t key = skey[u];
          c += ((key & pmask) == prefix) & ((key & bb) != 0u);
        }
        c = __reduce_add_sync(kFull, c);
        if (c >= need) {
          prefix |= bb;
          msurv = c;
        } else {
          need -= c;
          msurv -= c;
        }
        pmask |= bb;
      }
    }
  } else if (keff > 0) {
    // every candidate is kept
    for (int t = 0; t < T; ++t) {
      const int j = t * 32 + lane;
      surv |= (uint32_t)(j < n && !is_forced(j, win_lo, ns)) << t;
    }
    need = ncand;  // pmask = prefix = 0: every survivor matches
  }

  // emit forced blocks and picks in ascending block order
  int base = 0, rank_base = 0;
  for (int t = 0; t < T; ++t) {
    const int j = t * 32 + lane;
    const bool forced = j < n && is_forced(j, win_lo, ns);
    const bool sv = (surv >> t) & 1u;
    const uint32_t key = sv ? ordered_key(s[j]) : 0u;
    const bool above = sv && ((key & pmask) > prefix);
    const bool match = sv && ((key & pmask) == prefix);
    const uint32_t mm = __ballot_sync(kFull, match);
    const int rk = rank_base + __popc(mm & lt);
    rank_base += __popc(mm);
    const bool sel = forced || above || (match && rk < need);
    const uint32_t sm = __ballot_sync(kFull, sel);
    const int pos = base + __popc(sm & lt);
    if (sel) {
      if (pos < W) idx_row[pos] = j;
      else raise_error(hdr, DSA_ERR_DEVICE_BOUNDS, kKernSelect, i, pos);
    }
    base += __popc(sm);
  }
  for (int p = base + lane; p < W; p += 32) idx_row[p] = -1;
  if (lane == 0) *cnt_out = min(base, W);
  __syncwarp();
}

// Rows handled by one CTA of the score kernels: heads [h0, h0+HB) of one KV
// group (all share pooled K) times query blocks [i0, i0+RB), HB*RB <= 8.
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

// Scores of the CTA's rows against key blocks 0..jmax into shared memory;
// then either the fused selection (FUSED) or a plain copy to `scores`.
template <int D, bool FUSED>
__global__ void __launch_bounds__(kSelThreads)
score_kernel(Shape s, KBudget kb, int HB, int RB, const float* __restrict__ qp,
             const float* __restrict__ kp, float* __restrict__ scores, int32_t* __restrict__ idx,
             int32_t* __restrict__ cnt, WsHeader* hdr) {
  extern __shared__ float sm_f[];
  float* qs = sm_f;                       // [8][D]
  float* sc = sm_f + kSelWarps * D;       // [8][nb]
  uint32_t* sk = reinterpret_cast<uint32_t*>(sc + kSelWarps * s.nb);  // [8][nb] (FUSED only)
  const RowTile tile = row_tile(s, HB, RB);
  const int h_end = min(tile.h0 + HB, (tile.kvh + 1) * s.group);
  const int i_end = min(tile.i0 + RB, s.nb);

  // slot r -> (h, i); inactive slots hold zeros and are never read back
  for (int e = threadIdx.x; e < kSelWarps * D; e += kSelThreads) {
    const int r = e / D, c = e % D;
    const int h = tile.h0 + r / RB, i = tile.i0 + r % RB;
    float v = 0.f;
    if (r < HB * RB && h < h_end && i < i_end)
      v = qp[(((size_t)tile.b * s.Hq + h) * s.nb + i) * D + c];
    qs[e] = v;
  }
  __syncthreads();

  const int jmax = i_end - 1;
  const float* kbase = kp + ((size_t)tile.b * s.Hkv + tile.kvh) * s.nb * D;
  for (int j = threadIdx.x; j <= jmax; j += kSelThreads) {
    float o[kSelWarps];
    score_rows<D, kSelWarps>(qs, kbase + (size_t)j * D, o);
#pragma unroll
    for (int r = 0; r < kSelWarps; ++r) {
      const int i = tile.i0 + r % RB;
      sc[r * s.nb + j] = (j <= i) ? o[r] : -INFINITY;
    }
  }
  __syncthreads();

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int r = warp;
  const int h = tile.h0 + r / RB, i = tile.i0 + r % RB;
  if (r >= HB * RB || h >= h_end || i >= i_end) return;
  const size_t row = ((size_t)tile.b * s.Hq + h) * s.nb + i;
  if (FUSED) {
    const int k = s.per_head ? kb.k[h] : kb.k[0];
    select_row(sc + r * s.nb, sk + r * s.nb, i, k, s.lw, s.ns, s.W, idx + row * s.W, cnt + row, hdr,
               lane);
  } else {
    float* dst = scores + row * s.nb;
    for (int j = lane; j < s.nb; j += 32) dst[j] = (j <= i) ? sc[r * s.nb + j] : -INFINITY;
  }
}

// Selection on caller scores: one warp per row (b, h, i).
__global__ void __launch_bounds__(kSelThreads)
select_kernel(Shape s, KBudget kb, const float* __restrict__ scores, int32_t* __restrict__ idx,
              int32_t* __restrict__ cnt, WsHeader* hdr, long long n_rows) {
  extern __shared__ float sm_f[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const long long row = (long long)blockIdx.x * kSelWarps + warp;
  if (row >= n_rows) return;
  const int i = (int)(row % s.nb);
  const int h = (int)((row / s.nb) % s.Hq);
  float* sc = sm_f + warp * s.nb;
  uint32_t* sk = reinterpret_cast<uint32_t*>(sm_f + kSelWarps * s.nb) + warp * s.nb;
  const float* src = scores + (size_t)row * s.nb;
  for (int j = lane; j <= i; j += 32) sc[j] = src[j];
  __syncwarp();
  const int k = s.per_head ? kb.k[h] : kb.k[0];
  select_row(sc, sk, i, k, s.lw, s.ns, s.W, idx + (size_t)row * s.W, cnt + row, hdr, lane);
}

void row_tiling(const Shape& s, int& HB, int& RB) {
  HB = s.group < kSelWarps ? s.group : kSelWarps;
  RB = kSelWarps / HB;
  if (RB < 1) RB = 1;
}

int score_grid(const Shape& s, int HB, int RB) {
  const int n_hc = (s.group + HB - 1) / HB;
  const int n_ic = (s.nb + RB - 1) / RB;
  return s.B * s.Hkv * n_hc * n_ic;
}

template <bool FUSED>
cudaError_t launch_score_impl(const Shape& s, const KBudget& kb, const float* qp, const float* kp,
                              float* scores, int32_t* idx, int32_t* cnt, WsHeader* hdr,
                              cudaStream_t st) {
  int HB, RB;
  row_tiling(s, HB, RB);
  const size_t smem = (size_t)kSelWarps * (s.d + (FUSED ? 2 : 1) * s.nb) * sizeof(float);
  const int grid = score_grid(s, HB, RB);
  if (s.d == 64) {
    auto f = score_kernel<64, FUSED>;
    cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    f<<<grid, kSelThreads, smem, st>>>(s, kb, HB, RB, qp, kp, scores, idx, cnt, hdr);
  } else {
    auto f = score_kernel<128, FUSED>;
    cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    f<<<grid, kSelThreads, smem, st>>>(s, kb, HB, RB, qp, kp, scores, idx, cnt, hdr);
  }
  return cudaGetLastError();
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
  const long long n_rows = (long long)s.B * s.Hq * s.nb;
  const long long grid = (n_rows + kSelWarps - 1) / kSelWarps;
  const size_t smem = (size_t)kSelWarps * 2 * s.nb * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  select_kernel<<<(unsigned)grid, kSelThreads, smem, st>>>(s, kb, scores, idx, cnt, hdr, n_rows);
  return cudaGetLastError();
}

}  // namespace dsa
