// Backward of the block-sparse causal attention: dQ, dK, dV over the kept
// blocks, with the kept lists held fixed (the selection is a discrete choice
// and passes no gradient). The DeepSeek NSA article (section 2.2) trains with
// the sparse pattern but gives no backward rule; this is the exact gradient of
// O = softmax(Q K^T * scale) V over the kept, causally visible keys:
//   P = exp(S * scale - lse)             (lse from the forward),
//   dP = dO V^T,  D_r = dO_r . O_r,  dS = P * (dP - D),
//   dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO,
// with dK and dV of KV head g summed over its query heads (GQA sharing).
//
// Warp-level tensor-core path (mma.sync m16n8k16, bf16 operands, fp32
// accumulators), four steps and no atomics on the gradients:
//  1. bwd_prep_kernel: D_r = dO_r . O_r and lse in base 2 per query row;
//  2. bwd_colbits_kernel: the transpose of the kept lists as one bitmap per
//     key block (b, g, j): bit (u * nb + i) is set when query head g*G + u
//     keeps j in query block i;
//  3. bwd_dq_kernel: one CTA per query block (b, h, i), its kept blocks in
//     ascending order; recomputes S and P, forms dS and accumulates dQ;
//  4. bwd_dkv_kernel: one CTA per key block (b, g, j), the (head, query
//     block) pairs of its bitmap in bit order; recomputes S^T and P^T, forms
//     dS^T and accumulates dK and dV.
// Every sum runs in a fixed order, so the results are deterministic.
#include "dsa_internal.cuh"
#include "mma_sync.cuh"

namespace dsa {
namespace {

struct BwdArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* o;
  const __nv_bfloat16* dout;
  const float* lse;
  const int32_t* idx;
  const int32_t* cnt;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  float* drow;       // [B, Hq, N] D_r = dO_r . O_r
  float* lse2;       // [B, Hq, N] lse * log2(e) (+inf for a row with no visible key)
  uint32_t* colbits; // [B, Hkv, nb, cw] transposed kept lists
  WsHeader* hdr;
  int B, Hq, Hkv, N, nb, W, group, cw;
  float scale, c2;  // scale, scale * log2(e)
};

template <int BS, int D>
struct BwdCfg {
  static constexpr int kWarps = BS / 16;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kTile = BS * D;                 // elements of one tile
  static constexpr int KT = BS < 64 ? BS : 64;         // key sub-tile of the dQ kernel
  static constexpr int QT = 32;                        // query sub-tile of the dK/dV kernel
  static constexpr int kPairChunk = 2048;              // pairs listed at a time (dK/dV kernel)
  // dQ: Q, dO, 2 x (K, V); list; lse2 and D of the block's rows
  static constexpr size_t kSmemDq = (size_t)kTile * 2 * 6 + (size_t)kMaxBlocks * 4 + 2 * BS * 4;
  // dK/dV: K, V, 2 x (Q, dO); 2 x (lse2, D); pair list
  static constexpr size_t kSmemDkv = (size_t)kTile * 2 * 6 + 4 * BS * 4 + kPairChunk * 4;
};

template <int BS, int D, int T>
__device__ __forceinline__ void load_tile_t(__nv_bfloat16* dst, const __nv_bfloat16* src, int tid) {
  constexpr int CH = D / 8;
#pragma unroll 4
  for (int e = tid; e < BS * CH; e += T) {
    const int r = e / CH, c = e % CH;
    cp_async16(smem_u32(dst + swz<D>(r, c)), src + (size_t)r * D + c * 8);
  }
}

template <int BS, int T>
__device__ __forceinline__ void load_vec(float* dst, const float* src, int tid) {
  for (int e = tid; e < BS / 4; e += T) cp_async16(smem_u32(dst + 4 * e), src + 4 * e);
}

// ---------------------------------------------------------------------------
// 1. D_r and base-2 lse per query row: one warp per row.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(BwdArgs a) {
  constexpr int VPL = D / 32;
  const size_t row = (size_t)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const size_t rows = (size_t)a.B * a.Hq * a.N;
  if (row >= rows) return;
  const __nv_bfloat16* o = a.o + row * D + lane * VPL;
  const __nv_bfloat16* g = a.dout + row * D + lane * VPL;
  float x = 0.f;
#pragma unroll
  for (int e = 0; e < VPL; ++e) x = __fmaf_rn(__bfloat162float(o[e]), __bfloat162float(g[e]), x);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  if (lane == 0) {
    a.drow[row] = x;
    const float l = a.lse[row];
    a.lse2[row] = l == -INFINITY ? INFINITY : l * kLog2e;
  }
}

// ---------------------------------------------------------------------------
// 2. Transposed kept lists: one thread per (row, list entry).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_colbits_kernel(BwdArgs a) {
  const size_t e = (size_t)blockIdx.x * 256 + threadIdx.x;
  const size_t total = (size_t)a.B * a.Hq * a.nb * a.W;
  if (e >= total) return;
  const size_t row = e / a.W;
  const int t = (int)(e % a.W);
  const int i = (int)(row % a.nb);
  const int h = (int)((row / a.nb) % a.Hq);
  const int b = (int)(row / ((size_t)a.nb * a.Hq));
  int n = a.cnt[row];
  if (n < 0 || n > a.W) {
    if (t == 0) raise_error(a.hdr, DSA_ERR_DEVICE_BOUNDS, kKernAttnBwd, (int)row, n);
    n = n < 0 ? 0 : a.W;
  }
  if (t >= n) return;
  const int j = a.idx[row * a.W + t];
  // the same entries as the dQ passes use: in range and above the one before
  if (j < 0 || j > i || (t > 0 && j <= a.idx[row * a.W + t - 1])) {
    raise_error(a.hdr, DSA_ERR_DEVICE_BOUNDS, kKernAttnBwd, (int)row, j);
    return;
  }
  const int kvh = h / a.group, u = h % a.group;
  const int bit = u * a.nb + i;
  atomicOr(a.colbits + (((size_t)b * a.Hkv + kvh) * a.nb + j) * a.cw + bit / 32, 1u << (bit % 32));
}

// ---------------------------------------------------------------------------
// 3. dQ: one CTA per query block (b, h, i); warp w owns query rows 16w..16w+15.
// ---------------------------------------------------------------------------
template <int BS, int D>
__global__ void __launch_bounds__(BwdCfg<BS, D>::kThreads) bwd_dq_kernel(BwdArgs a) {
  using Cfg = BwdCfg<BS, D>;
  constexpr int T = Cfg::kThreads;
  constexpr int KT = Cfg::KT;
  constexpr int NT_S = KT / 8;  // n-tiles of a key sub-tile
  constexpr int NT_O = D / 8;   // n-tiles of dQ (head dim)
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sdO = sQ + Cfg::kTile;
  __nv_bfloat16* sK = sdO + Cfg::kTile;     // [2][BS][D]
  __nv_bfloat16* sV = sK + 2 * Cfg::kTile;  // [2][BS][D]
  int* sList = reinterpret_cast<int*>(sV + 2 * Cfg::kTile);
  float* sL2 = reinterpret_cast<float*>(sList + kMaxBlocks);  // [BS]
  float* sDr = sL2 + BS;                                      // [BS]
  __shared__ int sCount;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  // KV-head-major order (CTAs resident together share one KV head in L2);
  // inside a KV head the longest rows (last query blocks) come first
  const int per_kv = a.group * a.nb;
  const int bk = blockIdx.x / per_kv;
  const int rem = blockIdx.x - bk * per_kv;
  const int b = bk / a.Hkv, kvh = bk - b * a.Hkv;
  const int i = a.nb - 1 - rem / a.group;
  const int h = kvh * a.group + rem % a.group;
  const int bh = b * a.Hq + h;
  const size_t row_id = (size_t)bh * a.nb + i;

  // kept list -> shared memory, 32 entries per step by warp 0, dropping
  // out-of-range and out-of-order entries (flagged)
  if (warp == 0) {
    int n = a.cnt[row_id];
    if (n < 0 || n > a.W) {
      if (lane == 0) raise_error(a.hdr, DSA_ERR_DEVICE_BOUNDS, kKernAttnBwd, (int)row_id, n);
      n = n < 0 ? 0 : a.W;
    }
    const int32_t* lst = a.idx + row_id * a.W;
    int m = 0;
    for (int t0 = 0; t0 < n; t0 += 32) {
      const int t = t0 + lane;
      const int j = t < n ? lst[t] : 0;
      const bool bad = t < n && !list_entry_ok(lst, t, j, i, true);
      if (bad) raise_error(a.hdr, DSA_ERR_DEVICE_BOUNDS, kKernAttnBwd, (int)row_id, j);
      const uint32_t keep = __ballot_sync(0xffffffffu, t < n && !bad);
      if ((keep >> lane) & 1u) sList[m + __popc(keep & ((1u << lane) - 1u))] = j;
      m += __popc(keep);
    }
    if (lane == 0) sCount = m;
  }
  __syncthreads();
  const int n_kept = sCount;

  const size_t q_row0 = (size_t)bh * a.N + (size_t)i * BS;
  const __nv_bfloat16* gK = a.k + ((size_t)(b * a.Hkv + kvh) * a.N) * D;
  const __nv_bfloat16* gV = a.v + ((size_t)(b * a.Hkv + kvh) * a.N) * D;
  load_tile_t<BS, D, T>(sQ, a.q + q_row0 * D, tid);
  load_tile_t<BS, D, T>(sdO, a.dout + q_row0 * D, tid);
  load_vec<BS, T>(sL2, a.lse2 + q_row0, tid);
  load_vec<BS, T>(sDr, a.drow + q_row0, tid);
  if (n_kept > 0) {
    const int j0 = sList[0];
    load_tile_t<BS, D, T>(sK, gK + (size_t)j0 * BS * D, tid);
    load_tile_t<BS, D, T>(sV, gV + (size_t)j0 * BS * D, tid);
  }
  cp_async_commit();

  float dq[NT_O][4];
#pragma unroll
  for (int t = 0; t < NT_O; ++t) dq[t][0] = dq[t][1] = dq[t][2] = dq[t][3] = 0.f;
  uint32_t qf[D / 16][4];
  const int g = lane / 4, cq = lane % 4;
  const int row0 = warp * 16 + g;  // local query rows row0 and row0 + 8
  float l2_0 = 0.f, l2_1 = 0.f, dr0 = 0.f, dr1 = 0.f;
  const int mq = lane / 8;

  for (int n = 0; n < n_kept; ++n) {
    const int j = sList[n];
    if (n + 1 < n_kept) {
      const int jn = sList[n + 1];
      const int nbuf = (n + 1) & 1;
      load_tile_t<BS, D, T>(sK + nbuf * Cfg::kTile, gK + (size_t)jn * BS * D, tid);
      load_tile_t<BS, D, T>(sV + nbuf * Cfg::kTile, gV + (size_t)jn * BS * D, tid);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (n == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int r = warp * 16 + (mq % 2) * 8 + (lane % 8);
        ldsm_x4(qf[kk], smem_u32(sQ + swz<D>(r, kk * 2 + mq / 2)));
      }
      l2_0 = sL2[row0];
      l2_1 = sL2[row0 + 8];
      dr0 = sDr[row0];
      dr1 = sDr[row0 + 8];
    }
    const __nv_bfloat16* cK = sK + (n & 1) * Cfg::kTile;
    const __nv_bfloat16* cV = sV + (n & 1) * Cfg::kTile;

#pragma unroll 1
    for (int kt = 0; kt < BS / KT; ++kt) {
      // S = Q K^T and dP = dO V^T for this warp's 16 rows x KT keys
      float s[NT_S][4], dp[NT_S][4];
#pragma unroll
      for (int t = 0; t < NT_S; ++t) {
        s[t][0] = s[t][1] = s[t][2] = s[t][3] = 0.f;
        dp[t][0] = dp[t][1] = dp[t][2] = dp[t][3] = 0.f;
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t df[4];
        {
          const int r = warp * 16 + (mq % 2) * 8 + (lane % 8);
          ldsm_x4(df, smem_u32(sdO + swz<D>(r, kk * 2 + mq / 2)));
        }
#pragma unroll
        for (int np = 0; np < KT / 16; ++np) {
          const int key = kt * KT + np * 16 + (mq / 2) * 8 + (lane % 8);
          uint32_t kb[4], vb[4];
          ldsm_x4(kb, smem_u32(cK + swz<D>(key, kk * 2 + (mq % 2))));
          ldsm_x4(vb, smem_u32(cV + swz<D>(key, kk * 2 + (mq % 2))));
          mma_bf16(s[2 * np], qf[kk], kb[0], kb[1]);
          mma_bf16(s[2 * np + 1], qf[kk], kb[2], kb[3]);
          mma_bf16(dp[2 * np], df, vb[0], vb[1]);
          mma_bf16(dp[2 * np + 1], df, vb[2], vb[3]);
        }
      }
      // P = 2^(S c2 - lse2) with the causal mask on the diagonal block;
      // dS = P (dP - D), rounded to bf16 for the product with K
#pragma unroll
      for (int t = 0; t < NT_S; ++t) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = kt * KT + t * 8 + 2 * cq + (e & 1);
          const int row = row0 + (e >> 1) * 8;
          const bool masked = (j == i) && (col > row);
          const float p = masked ? 0.f : ex2(s[t][e] * a.c2 - ((e >> 1) ? l2_1 : l2_0));
          s[t][e] = p * (dp[t][e] - ((e >> 1) ? dr1 : dr0));
        }
      }
      // dQ += dS K
#pragma unroll
      for (int kk = 0; kk < KT / 16; ++kk) {
        uint32_t pa[4];
        pa[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
        pa[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
        pa[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
        pa[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
        for (int dpi = 0; dpi < D / 16; ++dpi) {
          uint32_t kb[4];
          const int key = kt * KT + kk * 16 + (mq % 2) * 8 + (lane % 8);
          ldsm_x4_t(kb, smem_u32(cK + swz<D>(key, dpi * 2 + mq / 2)));
          mma_bf16(dq[2 * dpi], pa, kb[0], kb[1]);
          mma_bf16(dq[2 * dpi + 1], pa, kb[2], kb[3]);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  __nv_bfloat16* d0 = a.dq + (q_row0 + row0) * D;
  __nv_bfloat16* d1 = d0 + 8 * D;
#pragma unroll
  for (int t = 0; t < NT_O; ++t) {
    *reinterpret_cast<uint32_t*>(d0 + t * 8 + 2 * cq) = pack_bf16(dq[t][0] * a.scale, dq[t][1] * a.scale);
    *reinterpret_cast<uint32_t*>(d1 + t * 8 + 2 * cq) = pack_bf16(dq[t][2] * a.scale, dq[t][3] * a.scale);
  }
}

// ---------------------------------------------------------------------------
// 4. dK, dV: one CTA per key block (b, g, j); warp w owns key rows 16w..16w+15.
// ---------------------------------------------------------------------------
template <int BS, int D>
__global__ void __launch_bounds__(BwdCfg<BS, D>::kThreads) bwd_dkv_kernel(BwdArgs a) {
  using Cfg = BwdCfg<BS, D>;
  constexpr int T = Cfg::kThreads;
  constexpr int QT = Cfg::QT;
  constexpr int NT_S = QT / 8;  // n-tiles of a query sub-tile
  constexpr int NT_O = D / 8;   // n-tiles of dK, dV (head dim)
  extern __shared__ __align__(128) uint8_t smem_raw[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* sV = sK + Cfg::kTile;
  __nv_bfloat16* sQ = sV + Cfg::kTile;       // [2][BS][D]
  __nv_bfloat16* sdO = sQ + 2 * Cfg::kTile;  // [2][BS][D]
  float* sL2 = reinterpret_cast<float*>(sdO + 2 * Cfg::kTile);  // [2][BS]
  float* sDr = sL2 + 2 * BS;                                    // [2][BS]
  int* sPair = reinterpret_cast<int*>(sDr + 2 * BS);            // [kPairChunk]
  __shared__ int sNp;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  // key block j = 0 (the densest columns: every row keeps its sinks) first
  const int BH = a.B * a.Hkv;
  const int j = blockIdx.x / BH;
  const int bk = blockIdx.x - j * BH;
  const int b = bk / a.Hkv, kvh = bk - b * a.Hkv;
  const size_t k_row0 = ((size_t)(b * a.Hkv + kvh) * a.N) + (size_t)j * BS;
  const uint32_t* bits = a.colbits + ((size_t)bk * a.nb + j) * a.cw;

  load_tile_t<BS, D, T>(sK, a.k + k_row0 * D, tid);
  load_tile_t<BS, D, T>(sV, a.v + k_row0 * D, tid);
  cp_async_commit();

  float dk[NT_O][4], dv[NT_O][4];
#pragma unroll
  for (int t = 0; t < NT_O; ++t) {
    dk[t][0] = dk[t][1] = dk[t][2] = dk[t][3] = 0.f;
    dv[t][0] = dv[t][1] = dv[t][2] = dv[t][3] = 0.f;
  }
  const int g = lane / 4, cq = lane % 4;
  const int kr0 = warp * 16 + g;  // local key rows kr0 and kr0 + 8
  const int mq = lane / 8;

  auto load_pair = [&](int pair, int buf) {
    const int u = pair / a.nb, i = pair - u * a.nb;
    const size_t q_row0 = ((size_t)b * a.Hq + kvh * a.group + u) * a.N + (size_t)i * BS;
    load_tile_t<BS, D, T>(sQ + buf * Cfg::kTile, a.q + q_row0 * D, tid);
    load_tile_t<BS, D, T>(sdO + buf * Cfg::kTile, a.dout + q_row0 * D, tid);
    load_vec<BS, T>(sL2 + buf * BS, a.lse2 + q_row0, tid);
    load_vec<BS, T>(sDr + buf * BS, a.drow + q_row0, tid);
  };

  // the pairs of this key block, listed kPairChunk bit positions at a time
  for (int w0 = 0; w0 < a.cw; w0 += Cfg::kPairChunk / 32) {
    const int wn = min(Cfg::kPairChunk / 32, a.cw - w0);
    __syncthreads();  // the previous chunk's list is no longer read
    if (warp == 0) {
      int base = 0;
      for (int wb = 0; wb < wn; wb += 32) {
        const uint32_t word = wb + lane < wn ? bits[w0 + wb + lane] : 0u;
        int cntw = __popc(word), incl = cntw;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += y;
        }
        int pos = base + incl - cntw;
        uint32_t wv = word;
        while (wv != 0u) {
          const int bt = __ffs(wv) - 1;
          wv &= wv - 1u;
          sPair[pos++] = (w0 + wb + lane) * 32 + bt;
        }
        base += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) sNp = base;
    }
    __syncthreads();
    const int np_ = sNp;
    if (np_ > 0) load_pair(sPair[0], 0);
    cp_async_commit();
    for (int p = 0; p < np_; ++p) {
      const int pair = sPair[p];
      const int i = pair % a.nb;
      if (p + 1 < np_) load_pair(sPair[p + 1], (p + 1) & 1);
      cp_async_commit();
      cp_async_wait<1>();
      __syncthreads();
      const __nv_bfloat16* cQ = sQ + (p & 1) * Cfg::kTile;
      const __nv_bfloat16* cdO = sdO + (p & 1) * Cfg::kTile;
      const float* cL2 = sL2 + (p & 1) * BS;
      const float* cDr = sDr + (p & 1) * BS;
#pragma unroll 1
      for (int qt = 0; qt < BS / QT; ++qt) {
        // S^T = K Q^T and dP^T = V dO^T for this warp's 16 keys x QT queries
        float st[NT_S][4], dpt[NT_S][4];
#pragma unroll
        for (int t = 0; t < NT_S; ++t) {
          st[t][0] = st[t][1] = st[t][2] = st[t][3] = 0.f;
          dpt[t][0] = dpt[t][1] = dpt[t][2] = dpt[t][3] = 0.f;
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          uint32_t kf[4], vf[4];
          const int r = warp * 16 + (mq % 2) * 8 + (lane % 8);
          ldsm_x4(kf, smem_u32(sK + swz<D>(r, kk * 2 + mq / 2)));
          ldsm_x4(vf, smem_u32(sV + swz<D>(r, kk * 2 + mq / 2)));
#pragma unroll
          for (int np = 0; np < QT / 16; ++np) {
            const int qr = qt * QT + np * 16 + (mq / 2) * 8 + (lane % 8);
            uint32_t qb[4], ob[4];
            ldsm_x4(qb, smem_u32(cQ + swz<D>(qr, kk * 2 + (mq % 2))));
            ldsm_x4(ob, smem_u32(cdO + swz<D>(qr, kk * 2 + (mq % 2))));
            mma_bf16(st[2 * np], kf, qb[0], qb[1]);
            mma_bf16(st[2 * np + 1], kf, qb[2], qb[3]);
            mma_bf16(dpt[2 * np], vf, ob[0], ob[1]);
            mma_bf16(dpt[2 * np + 1], vf, ob[2], ob[3]);
          }
        }
        // P^T and dS^T; a query sees a key of the diagonal block only when
        // the key is not after it
#pragma unroll
        for (int t = 0; t < NT_S; ++t) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int qc = qt * QT + t * 8 + 2 * cq + e;
            const float l2q = cL2[qc], drq = cDr[qc];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int kr = kr0 + hh * 8;
              const bool masked = (i == j) && (qc < kr);
              const float p = masked ? 0.f : ex2(st[t][2 * hh + e] * a.c2 - l2q);
              st[t][2 * hh + e] = p;
              dpt[t][2 * hh + e] = p * (dpt[t][2 * hh + e] - drq);
            }
          }
        }
        // dV += P^T dO and dK += dS^T Q
#pragma unroll
        for (int kk = 0; kk < QT / 16; ++kk) {
          uint32_t pa[4], sa[4];
          pa[0] = pack_bf16(st[2 * kk][0], st[2 * kk][1]);
          pa[1] = pack_bf16(st[2 * kk][2], st[2 * kk][3]);
          pa[2] = pack_bf16(st[2 * kk + 1][0], st[2 * kk + 1][1]);
          pa[3] = pack_bf16(st[2 * kk + 1][2], st[2 * kk + 1][3]);
          sa[0] = pack_bf16(dpt[2 * kk][0], dpt[2 * kk][1]);
          sa[1] = pack_bf16(dpt[2 * kk][2], dpt[2 * kk][3]);
          sa[2] = pack_bf16(dpt[2 * kk + 1][0], dpt[2 * kk + 1][1]);
          sa[3] = pack_bf16(dpt[2 * kk + 1][2], dpt[2 * kk + 1][3]);
#pragma unroll
          for (int dpi = 0; dpi < D / 16; ++dpi) {
            const int qr = qt * QT + kk * 16 + (mq % 2) * 8 + (lane % 8);
            uint32_t ob[4], qb[4];
            ldsm_x4_t(ob, smem_u32(cdO + swz<D>(qr, dpi * 2 + mq / 2)));
            ldsm_x4_t(qb, smem_u32(cQ + swz<D>(qr, dpi * 2 + mq / 2)));
            mma_bf16(dv[2 * dpi], pa, ob[0], ob[1]);
            mma_bf16(dv[2 * dpi + 1], pa, ob[2], ob[3]);
            mma_bf16(dk[2 * dpi], sa, qb[0], qb[1]);
            mma_bf16(dk[2 * dpi + 1], sa, qb[2], qb[3]);
          }
        }
      }
      __syncthreads();
    }
    cp_async_wait<0>();
  }
  cp_async_wait<0>();

  __nv_bfloat16* k0 = a.dk + (k_row0 + kr0) * D;
  __nv_bfloat16* v0 = a.dv + (k_row0 + kr0) * D;
#pragma unroll
  for (int t = 0; t < NT_O; ++t) {
    *reinterpret_cast<uint32_t*>(k0 + t * 8 + 2 * cq) = pack_bf16(dk[t][0] * a.scale, dk[t][1] * a.scale);
    *reinterpret_cast<uint32_t*>(k0 + 8 * D + t * 8 + 2 * cq) =
        pack_bf16(dk[t][2] * a.scale, dk[t][3] * a.scale);
    *reinterpret_cast<uint32_t*>(v0 + t * 8 + 2 * cq) = pack_bf16(dv[t][0], dv[t][1]);
    *reinterpret_cast<uint32_t*>(v0 + 8 * D + t * 8 + 2 * cq) = pack_bf16(dv[t][2], dv[t][3]);
  }
}

template <int BS, int D>
cudaError_t launch_bwd_impl(const BwdArgs& a, const Shape& s, const BwdTcArgs* tc, cudaStream_t st) {
  using Cfg = BwdCfg<BS, D>;
  cudaError_t e;
  {
    const size_t rows = (size_t)a.B * a.Hq * a.N;
    const size_t grid = (rows + 7) / 8;
    if (grid > 0x7fffffffULL) return cudaErrorInvalidConfiguration;
    bwd_prep_kernel<D><<<(unsigned)grid, 256, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    e = cudaMemsetAsync(a.colbits, 0, sizeof(uint32_t) * (size_t)a.B * a.Hkv * a.nb * a.cw, st);
    if (e != cudaSuccess) return e;
    const size_t total = (size_t)a.B * a.Hq * a.nb * a.W;
    const size_t grid = (total + 255) / 256;
    if (grid > 0x7fffffffULL) return cudaErrorInvalidConfiguration;
    if (grid > 0) {
      bwd_colbits_kernel<<<(unsigned)grid, 256, 0, st>>>(a);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  // the tensor-core passes (attn_bwd_tc.cu) take over from here
  if (tc != nullptr) return launch_attn_bwd_tc(s, *tc, st);
  {
    auto f = bwd_dq_kernel<BS, D>;
    e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::kSmemDq);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)a.B * a.Hq * a.nb;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    f<<<(unsigned)grid, Cfg::kThreads, Cfg::kSmemDq, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    auto f = bwd_dkv_kernel<BS, D>;
    e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cfg::kSmemDkv);
    if (e != cudaSuccess) return e;
    const long long grid = (long long)a.B * a.Hkv * a.nb;
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    f<<<(unsigned)grid, Cfg::kThreads, Cfg::kSmemDkv, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_attn_bwd(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                            const __nv_bfloat16* v, const __nv_bfloat16* o, const float* lse,
                            const __nv_bfloat16* dout, const int32_t* idx, const int32_t* cnt,
                            __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv, void* ws,
                            bool use_tc, cudaStream_t st) {
  const BwdWs lw = bwd_ws_layout(s);
  char* base = static_cast<char*>(ws);
  BwdArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.dout = dout;
  a.lse = lse;
  a.idx = idx;
  a.cnt = cnt;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.drow = reinterpret_cast<float*>(base + lw.drow);
  a.lse2 = reinterpret_cast<float*>(base + lw.lse2);
  a.colbits = reinterpret_cast<uint32_t*>(base + lw.colbits);
  a.hdr = static_cast<WsHeader*>(ws);
  a.B = s.B;
  a.Hq = s.Hq;
  a.Hkv = s.Hkv;
  a.N = s.N;
  a.nb = s.nb;
  a.W = s.W;
  a.group = s.group;
  a.cw = lw.cw;
  a.scale = s.scale;
  a.c2 = s.scale * kLog2e;
  BwdTcArgs t;
  const BwdTcArgs* tc = nullptr;
  if (use_tc) {
    t.q = q;
    t.k = k;
    t.v = v;
    t.dout = dout;
    t.idx = idx;
    t.cnt = cnt;
    t.drow = a.drow;
    t.lse2 = a.lse2;
    t.colbits = a.colbits;
    t.pairs = reinterpret_cast<int32_t*>(base + lw.pairs);
    t.npairs = reinterpret_cast<int32_t*>(base + lw.npairs);
    t.dq = dq;
    t.dk = dk;
    t.dv = dv;
    t.hdr = a.hdr;
    t.B = s.B;
    t.Hq = s.Hq;
    t.Hkv = s.Hkv;
    t.N = s.N;
    t.nb = s.nb;
    t.W = s.W;
    t.group = s.group;
    t.cw = lw.cw;
    t.scale = s.scale;
    t.c2 = a.c2;
    tc = &t;
  }
  if (s.bs == 32 && s.d == 64) return launch_bwd_impl<32, 64>(a, s, tc, st);
  if (s.bs == 64 && s.d == 64) return launch_bwd_impl<64, 64>(a, s, tc, st);
  if (s.bs == 128 && s.d == 64) return launch_bwd_impl<128, 64>(a, s, tc, st);
  if (s.bs == 32 && s.d == 128) return launch_bwd_impl<32, 128>(a, s, tc, st);
  if (s.bs == 64 && s.d == 128) return launch_bwd_impl<64, 128>(a, s, tc, st);
  if (s.bs == 128 && s.d == 128) return launch_bwd_impl<128, 128>(a, s, tc, st);
  return cudaErrorInvalidValue;
}

}  // namespace dsa
