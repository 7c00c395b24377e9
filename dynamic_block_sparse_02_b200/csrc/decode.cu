// Decode step: one new query token per (batch, query head) against a KV cache.
//
// The zblog.xzdbk.com/559 post (section 动态开销与计算收益的权衡, point 2) keeps
// the sparse index with the KV cache so that inference reuses it; here the
// cache keeps the pooled key blocks (dsa_pool_keys) and every decode call
// scores the token against them, selects, and attends:
//   i      = (length - 1) / block, the token's query block;
//   s_j    = q . Kp[j] for the complete blocks j < i (pooled cache), and
//            q . mean(present keys of block i) for j = i (pooled here);
//   select = the prefill rules on that one row (top-k, group-shared top-k,
//            threshold), by the same warp selection as the prefill kernels;
//   out    = softmax(q K^T * scale) V over the present keys of the kept blocks.
//
// One CTA of 8 warps per (batch, query head). The keys are few (kept blocks
// times block size) and the product has one query row, so the attention runs
// on the CUDA cores: the warps take the kept blocks in turn, a lane owns one key
// of a 32-key chunk for the dot product and D/32 head-dim elements of the
// output, and the warps' online-softmax states are merged at the end.
#include "dsa_internal.cuh"
#include "select_row.cuh"

namespace dsa {
namespace {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr float kLog2eDec = 1.4426950408889634f;
constexpr float kLn2Dec = 0.6931471805599453f;

struct DecodeArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* kp;
  __nv_bfloat16* out;
  float* lse;
  int32_t* idx;
  int32_t* cnt;
  WsHeader* hdr;
  int length;
};

__device__ __forceinline__ void bf16x8_to_f32(uint4 w, float (&f)[8]) {
  f[0] = __uint_as_float(w.x << 16);
  f[1] = __uint_as_float(w.x & 0xffff0000u);
  f[2] = __uint_as_float(w.y << 16);
  f[3] = __uint_as_float(w.y & 0xffff0000u);
  f[4] = __uint_as_float(w.z << 16);
  f[5] = __uint_as_float(w.z & 0xffff0000u);
  f[6] = __uint_as_float(w.w << 16);
  f[7] = __uint_as_float(w.w & 0xffff0000u);
}

// Shared memory (dynamic), every region starting on a 16-byte boundary (the
// selection clears its histogram with 16-byte stores): qs [G][D] query rows
// (G = group size in the group-shared rule, else 1), kmean [D], sc [nb],
// hist [kDecWarps][256], list [nb], wm/wl [kDecWarps], wo [kDecWarps][D], cnt.
__host__ __device__ constexpr int align4(int n) { return (n + 3) & ~3; }

struct DecodeSmem {
  int qs, kmean, sc, hist, list, wm, wl, wo, cnt, total;  // offsets in 4-byte words
};

__host__ __device__ inline DecodeSmem decode_smem(int G, int D, int nb) {
  DecodeSmem m;
  m.qs = 0;
  m.kmean = align4(m.qs + G * D);
  m.sc = align4(m.kmean + D);
  m.hist = align4(m.sc + nb);
  m.list = align4(m.hist + kDecWarps * kHistWords);
  m.wm = align4(m.list + nb);
  m.wl = align4(m.wm + kDecWarps);
  m.wo = align4(m.wl + kDecWarps);
  m.cnt = align4(m.wo + kDecWarps * D);
  m.total = align4(m.cnt + 1);
  return m;
}
template <int D, int TMAX>
__global__ void __launch_bounds__(kDecThreads)
decode_kernel(Shape s, KBudget kb, DecodeArgs a) {
  extern __shared__ __align__(16) float sm[];
  const int G = s.group_select ? s.group : 1;
  const DecodeSmem lay = decode_smem(G, D, s.nb);
  float* const qs = sm + lay.qs;                                           // [G][D]
  float* const kmean = sm + lay.kmean;                                     // [D]
  float* const sc = sm + lay.sc;                                           // [nb]
  uint32_t* const hist = reinterpret_cast<uint32_t*>(sm + lay.hist);       // [kDecWarps][256]
  int32_t* const list = reinterpret_cast<int32_t*>(sm + lay.list);         // [nb]
  float* const wm = sm + lay.wm;                                           // [kDecWarps]
  float* const wl = sm + lay.wl;                                           // [kDecWarps]
  float* const wo = sm + lay.wo;                                           // [kDecWarps][D]
  int32_t* const scnt = reinterpret_cast<int32_t*>(sm + lay.cnt);

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int b = blockIdx.x / s.Hq, h = blockIdx.x % s.Hq;
  const int kvh = h / s.group;
  const int L = a.length;
  const int i = (L - 1) / s.bs;
  const size_t kv_base = ((size_t)b * s.Hkv + kvh) * s.N;  // row index of key 0 of this KV head

  // query rows: this head, or every head of its group (group-shared rule)
  const int h0 = s.group_select ? kvh * s.group : h;
  for (int e = tid; e < G * D; e += kDecThreads) {
    const int u = e / D, c = e % D;
    qs[e] = __bfloat162float(a.q[((size_t)b * s.Hq + h0 + u) * D + c]);
  }
  // the token's own block: mean of its present keys (rows in order, fp32)
  const int r0 = i * s.bs, nrow = L - r0;
  if (tid < D) {
    float acc = 0.f;
    for (int r = 0; r < nrow; ++r) acc += __bfloat162float(a.k[(kv_base + r0 + r) * D + tid]);
    kmean[tid] = acc / (float)nrow;
  }
  __syncthreads();

  // block scores j <= i: four fp32 partial sums over d, combined pairwise; in
  // the group rule the heads' scores are added in head order
  const float* const kp_head = a.kp + ((size_t)b * s.Hkv + kvh) * s.nb * D;
  for (int j = tid; j <= i; j += kDecThreads) {
    const float* kr = j < i ? kp_head + (size_t)j * D : kmean;
    float tot = 0.f;
    for (int u = 0; u < G; ++u) {
      const float* qr = qs + u * D;
      float x0 = 0.f, x1 = 0.f, x2 = 0.f, x3 = 0.f;
#pragma unroll 8
      for (int d4 = 0; d4 < D / 4; ++d4) {
        const float4 kv = *reinterpret_cast<const float4*>(kr + 4 * d4);
        const float4 qv = *reinterpret_cast<const float4*>(qr + 4 * d4);
        x0 = __fmaf_rn(qv.x, kv.x, x0);
        x1 = __fmaf_rn(qv.y, kv.y, x1);
        x2 = __fmaf_rn(qv.z, kv.z, x2);
        x3 = __fmaf_rn(qv.w, kv.w, x3);
      }
      const float one = __fadd_rn(__fadd_rn(x0, x1), __fadd_rn(x2, x3));
      tot = u == 0 ? one : __fadd_rn(tot, one);
    }
    sc[j] = tot;
  }
  __syncthreads();

  // selection of the row by warp 0, into shared memory
  if (warp == 0) {
    const int k = s.per_head ? kb.k[h] : kb.k[0];
    select_row<TMAX>(sc, hist, i, k, s.lw, s.ns, s.W, s.tau, s.c2, list, scnt, 1, 0, 0, a.hdr, lane);
  }
  __syncthreads();
  const int n = *scnt;
  if (a.idx != nullptr) {
    const size_t row = (size_t)b * s.Hq + h;
    for (int e = tid; e < s.W; e += kDecThreads) a.idx[row * s.W + e] = e < n ? list[e] : -1;
    if (tid == 0) a.cnt[row] = n;
  }

  // attention over the kept blocks: warp w takes list entries w, w + 8, ...
  constexpr int DPL = D / 32;  // output elements per lane: d = lane * DPL ..
  const float* const q = s.group_select ? qs + (h - h0) * D : qs;
  const float c2 = s.scale * kLog2eDec;
  float m = -INFINITY, l = 0.f;
  float o[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) o[e] = 0.f;
  for (int e = warp; e < n; e += kDecWarps) {
    const int blk = list[e];
    const int t_end = min((blk + 1) * s.bs, L);
    for (int t0 = blk * s.bs; t0 < t_end; t0 += 32) {
      const int t = t0 + lane;
      const bool live = t < t_end;
      float x = -INFINITY;
      if (live) {
        const uint4* kr = reinterpret_cast<const uint4*>(a.k + (kv_base + t) * D);
        float acc = 0.f;
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
          float f[8];
          bf16x8_to_f32(kr[c], f);
#pragma unroll
          for (int u = 0; u < 8; ++u) acc = __fmaf_rn(q[c * 8 + u], f[u], acc);
        }
        x = acc * c2;
      }
      float mc = x;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mc = fmaxf(mc, __shfl_xor_sync(kFullMask, mc, off));
      const float mn = fmaxf(m, mc);
      const float alpha = exp2f(m - mn);  // 0 when m is -inf
      l *= alpha;
#pragma unroll
      for (int e2 = 0; e2 < DPL; ++e2) o[e2] *= alpha;
      m = mn;
      const float p = live ? exp2f(x - mn) : 0.f;
      l += p;
      const int nk = min(32, t_end - t0);
      for (int u = 0; u < nk; ++u) {
        const float pu = __shfl_sync(kFullMask, p, u);
        const __nv_bfloat16* vr = a.v + (kv_base + t0 + u) * D + lane * DPL;
#pragma unroll
        for (int e2 = 0; e2 < DPL; ++e2) o[e2] = __fmaf_rn(pu, __bfloat162float(vr[e2]), o[e2]);
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) l += __shfl_xor_sync(kFullMask, l, off);
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = l;
  }
#pragma unroll
  for (int e2 = 0; e2 < DPL; ++e2) wo[warp * D + lane * DPL + e2] = o[e2];
  __syncthreads();

  // merge the warps' states
  if (tid < D) {
    float M = -INFINITY;
    for (int w = 0; w < kDecWarps; ++w) M = fmaxf(M, wm[w]);
    float lt = 0.f, ot = 0.f;
    if (M > -INFINITY) {
      for (int w = 0; w < kDecWarps; ++w) {
        const float f = exp2f(wm[w] - M);
        lt += f * wl[w];
        ot += f * wo[w * D + tid];
      }
    }
    const size_t row = (size_t)b * s.Hq + h;
    a.out[row * D + tid] = __float2bfloat16_rn(lt > 0.f ? ot / lt : 0.f);
    if (a.lse != nullptr && tid == 0) a.lse[row] = lt > 0.f ? M * kLn2Dec + logf(lt) : -INFINITY;
  }
}

template <int D, int TMAX>
cudaError_t launch_decode_d(const Shape& s, const KBudget& kb, const DecodeArgs& a, cudaStream_t st) {
  const int G = s.group_select ? s.group : 1;
  const size_t smem = sizeof(float) * (size_t)decode_smem(G, D, s.nb).total;
  auto f = decode_kernel<D, TMAX>;
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long grid = (long long)s.B * s.Hq;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  f<<<(unsigned)grid, kDecThreads, smem, st>>>(s, kb, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const Shape& s, const KBudget& kb, const __nv_bfloat16* q,
                          const __nv_bfloat16* k, const __nv_bfloat16* v, const float* kp,
                          int length, __nv_bfloat16* out, float* lse, int32_t* idx, int32_t* cnt,
                          WsHeader* hdr, cudaStream_t st) {
  DecodeArgs a{q, k, v, kp, out, lse, idx, cnt, hdr, length};
  const int tmax = s.nb <= 256 ? 8 : s.nb <= 512 ? 16 : 32;
  if (s.d == 64) {
    if (tmax == 8) return launch_decode_d<64, 8>(s, kb, a, st);
    if (tmax == 16) return launch_decode_d<64, 16>(s, kb, a, st);
    return launch_decode_d<64, 32>(s, kb, a, st);
  }
  if (tmax == 8) return launch_decode_d<128, 8>(s, kb, a, st);
  if (tmax == 16) return launch_decode_d<128, 16>(s, kb, a, st);
  return launch_decode_d<128, 32>(s, kb, a, st);
}

}  // namespace dsa
