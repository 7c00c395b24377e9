// Block-sparse causal attention forward (step 4) on the warp-level tensor-core
// path (mma.sync m16n8k16, bf16 in, fp32 accumulate).
//
// This is the legacy-path kernel: one CTA per work item (b, query head h,
// query block i), one warp per 16 query rows, K/V tiles of the kept blocks
// double-buffered in shared memory with cp.async. It computes, for each row,
// an online softmax over the kept key blocks in ascending order
// ("稀疏注意力 vs Flash Attention v2", section 1: scores, sparsity pattern,
// softmax with 1/sqrt(d_k), product with V; FlashAttention-style tiling and
// incremental softmax as described there), with the causal mask inside the
// diagonal block and query head h reading KV head h / (Hq/Hkv).
#include "dsa_internal.cuh"
#include "mma_sync.cuh"

namespace dsa {
namespace {

template <int BS, int D>
struct MmaCfg {
  static constexpr int kWarps = BS / 16;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kTile = BS * D;  // elements of one tile
  static constexpr size_t kSmem = (size_t)kTile * 2 * 5 + (size_t)kMaxBlocks * 4;
};

struct AttnArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* idx;
  const int32_t* cnt;
  __nv_bfloat16* out;
  float* lse;
  WsHeader* hdr;
  int B, Hq, Hkv, N, nb, W, group;
  float scale_log2;  // softmax scale * log2(e)
};

template <int BS, int D>
__device__ __forceinline__ void load_tile(__nv_bfloat16* dst, const __nv_bfloat16* src, int tid) {
  constexpr int CH = D / 8;
  constexpr int T = MmaCfg<BS, D>::kThreads;
#pragma unroll 4
  for (int e = tid; e < BS * CH; e += T) {
    const int r = e / CH, c = e % CH;
    cp_async16(smem_u32(dst + swz<D>(r, c)), src + (size_t)r * D + c * 8);
  }
}

template <int BS, int D>
__global__ void __launch_bounds__(MmaCfg<BS, D>::kThreads)
attn_mma_kernel(AttnArgs a) {
  using Cfg = MmaCfg<BS, D>;
  constexpr int NT_S = BS / 8;  // n-tiles of S per warp (keys)
  constexpr int NT_O = D / 8;   // n-tiles of O per warp (head dim)
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sK = sQ + Cfg::kTile;      // [2][BS][D]
  __nv_bfloat16* sV = sK + 2 * Cfg::kTile;  // [2][BS][D]
  int* sList = reinterpret_cast<int*>(sV + 2 * Cfg::kTile);
  __shared__ int sCount;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  // KV-head-major order (CTAs resident together share one KV head's K/V in
  // L2); inside a KV head the longest rows (last query blocks) come first.
  const int per_kv = a.group * a.nb;
  const int bk = blockIdx.x / per_kv;
  const int rem = blockIdx.x - bk * per_kv;
  const int b = bk / a.Hkv;
  const int kvh = bk - b * a.Hkv;
  const int i = a.nb - 1 - rem / a.group;
  const int h = kvh * a.group + rem % a.group;
  const int bh = b * a.Hq + h;
  const size_t row_id = (size_t)bh * a.nb + i;

  // Kept list -> shared memory, dropping out-of-range and out-of-order
  // entries (flagged): an entry must exceed the one before it.
  if (tid == 0) {
    int n = a.cnt[row_id];
    if (n < 0 || n > a.W) {
      raise_error(a.hdr, DSA_ERR_DEVICE_BOUNDS, kKernAttnMma, (int)row_id, n);
      n = n < 0 ? 0 : a.W;
    }
    const int32_t* lst = a.idx + row_id * a.W;
    int m = 0, prev = -1;
    for (int t = 0; t < n; ++t) {
      const int j = lst[t];
      const bool ok = j >= 0 && j <= i && (t == 0 || j > prev);
      prev = j;
      if (!ok) {
        raise_error(a.hdr, DSA_ERR_DEVICE_BOUNDS, kKernAttnMma, (int)row_id, j);
        continue;
      }
      sList[m++] = j;
    }
    sCount = m;
  }
  __syncthreads();
  const int n_kept = sCount;

  const __nv_bfloat16* gQ = a.q + ((size_t)bh * a.N + (size_t)i * BS) * D;
  const __nv_bfloat16* gK = a.k + ((size_t)(b * a.Hkv + kvh) * a.N) * D;
  const __nv_bfloat16* gV = a.v + ((size_t)(b * a.Hkv + kvh) * a.N) * D;

  load_tile<BS, D>(sQ, gQ, tid);
  if (n_kept > 0) {
    const int j0 = sList[0];
    load_tile<BS, D>(sK, gK + (size_t)j0 * BS * D, tid);
    load_tile<BS, D>(sV, gV + (size_t)j0 * BS * D, tid);
  }
  cp_async_commit();

  float o[NT_O][4];
#pragma unroll
  for (int t = 0; t < NT_O; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  uint32_t qf[D / 16][4];

  const int g = lane / 4, cq = lane % 4;
  const int row0 = warp * 16 + g;  // local query rows row0 and row0 + 8

  for (int n = 0; n < n_kept; ++n) {
    const int j = sList[n];
    if (n + 1 < n_kept) {
      const int jn = sList[n + 1];
      const int nb_ = (n + 1) & 1;
      load_tile<BS, D>(sK + nb_ * Cfg::kTile, gK + (size_t)jn * BS * D, tid);
      load_tile<BS, D>(sV + nb_ * Cfg::kTile, gV + (size_t)jn * BS * D, tid);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (n == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int m = lane / 8;
        const int r = warp * 16 + (m % 2) * 8 + (lane % 8);
        ldsm_x4(qf[kk], smem_u32(sQ + swz<D>(r, kk * 2 + m / 2)));
      }
    }
    const __nv_bfloat16* cK = sK + (n & 1) * Cfg::kTile;
    const __nv_bfloat16* cV = sV + (n & 1) * Cfg::kTile;

    // S = Q K^T for this warp's 16 rows x BS keys
    float s[NT_S][4];
#pragma unroll
    for (int t = 0; t < NT_S; ++t) s[t][0] = s[t][1] = s[t][2] = s[t][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
      for (int np = 0; np < BS / 16; ++np) {
        uint32_t kb[4];
        const int m = lane / 8;
        const int key = np * 16 + (m / 2) * 8 + (lane % 8);
        ldsm_x4(kb, smem_u32(cK + swz<D>(key, kk * 2 + (m % 2))));
        mma_bf16(s[2 * np], qf[kk], kb[0], kb[1]);
        mma_bf16(s[2 * np + 1], qf[kk], kb[2], kb[3]);
      }
    }

    // scale into the log2 domain, causal mask on the diagonal block, row max
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int t = 0; t < NT_S; ++t) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float x = s[t][e] * a.scale_log2;
        if (j == i) {
          const int col = t * 8 + 2 * cq + (e & 1);
          const int row = row0 + (e >> 1) * 8;
          if (col > row) x = -INFINITY;
        }
        s[t][e] = x;
      }
      mx0 = fmaxf(mx0, fmaxf(s[t][0], s[t][1]));
      mx1 = fmaxf(mx1, fmaxf(s[t][2], s[t][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float mu0 = mn0 == -INFINITY ? 0.f : mn0;  // all-masked row so far
    const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
    const float al0 = ex2(m0 - mu0), al1 = ex2(m1 - mu1);
    m0 = mn0;
    m1 = mn1;
    // P in bf16 (the MMA's input); row sums are taken over the same bf16 values
    float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
    for (int t = 0; t < NT_S; ++t) {
      s[t][0] = bf16_round(ex2(s[t][0] - mu0));
      s[t][1] = bf16_round(ex2(s[t][1] - mu0));
      s[t][2] = bf16_round(ex2(s[t][2] - mu1));
      s[t][3] = bf16_round(ex2(s[t][3] - mu1));
      ps0 += s[t][0] + s[t][1];
      ps1 += s[t][2] + s[t][3];
    }
    l0 = l0 * al0 + ps0;
    l1 = l1 * al1 + ps1;
#pragma unroll
    for (int t = 0; t < NT_O; ++t) {
      o[t][0] *= al0;
      o[t][1] *= al0;
      o[t][2] *= al1;
      o[t][3] *= al1;
    }

    // O += P V
#pragma unroll
    for (int kk = 0; kk < BS / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t vb[4];
        const int m = lane / 8;
        const int key = kk * 16 + (m % 2) * 8 + (lane % 8);
        ldsm_x4_t(vb, smem_u32(cV + swz<D>(key, dp * 2 + m / 2)));
        mma_bf16(o[2 * dp], pa, vb[0], vb[1]);
        mma_bf16(o[2 * dp + 1], pa, vb[2], vb[3]);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  // epilogue: normalise, round to bf16, write O and the log-sum-exp
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f;
  const float inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
  const size_t q_row0 = (size_t)bh * a.N + (size_t)i * BS + row0;
  __nv_bfloat16* o0 = a.out + q_row0 * D;
  __nv_bfloat16* o1 = o0 + 8 * D;
#pragma unroll
  for (int t = 0; t < NT_O; ++t) {
    *reinterpret_cast<uint32_t*>(o0 + t * 8 + 2 * cq) = pack_bf16(o[t][0] * inv0, o[t][1] * inv0);
    *reinterpret_cast<uint32_t*>(o1 + t * 8 + 2 * cq) = pack_bf16(o[t][2] * inv1, o[t][3] * inv1);
  }
  if (a.lse != nullptr && cq == 0) {
    a.lse[q_row0] = (l0 > 0.f) ? (m0 * kLn2 + logf(l0)) : -INFINITY;
    a.lse[q_row0 + 8] = (l1 > 0.f) ? (m1 * kLn2 + logf(l1)) : -INFINITY;
  }
}

template <int BS, int D>
cudaError_t launch_impl(const Shape& s, const AttnArgs& a, cudaStream_t st) {
  using Cfg = MmaCfg<BS, D>;
  auto f = attn_mma_kernel<BS, D>;
  cudaError_t e =
      cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::kSmem);
  if (e != cudaSuccess) return e;
  const long long grid = (long long)s.B * s.Hq * s.nb;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  f<<<(unsigned)grid, Cfg::kThreads, Cfg::kSmem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_mma(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                            const __nv_bfloat16* v, const int32_t* idx, const int32_t* cnt,
                            __nv_bfloat16* out, float* lse, WsHeader* hdr, cudaStream_t st) {
  AttnArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.idx = idx;
  a.cnt = cnt;
  a.out = out;
  a.lse = lse;
  a.hdr = hdr;
  a.B = s.B;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.N = s.N;
  a.nb = s.nb;
  a.W = s.W;
  a.group = s.group;
  a.scale_log2 = s.scale * kLog2e;
  if (s.bs == 32 && s.d == 64) return launch_impl<32, 64>(s, a, st);
  if (s.bs == 64 && s.d == 64) return launch_impl<64, 64>(s, a, st);
  if (s.bs == 128 && s.d == 64) return launch_impl<128, 64>(s, a, st);
  if (s.bs == 32 && s.d == 128) return launch_impl<32, 128>(s, a, st);
  if (s.bs == 64 && s.d == 128) return launch_impl<64, 128>(s, a, st);
  if (s.bs == 128 && s.d == 128) return launch_impl<128, 128>(s, a, st);
  return cudaErrorInvalidValue;
}

}  // namespace dsa
