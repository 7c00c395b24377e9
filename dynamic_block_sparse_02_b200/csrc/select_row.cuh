// Step 3 of the path: selection of one row (b, h, i) by one warp, shared by
// the prefill selection kernels and the decode kernel.
#pragma once

#include "dsa_internal.cuh"

namespace dsa {
namespace {

constexpr unsigned kFullMask = 0xffffffffu;
constexpr int kHistWords = 256;  // per-warp radix histogram of the selection

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
// s: the row's scores s[0..i] (shared memory); hist: 256 words of per-warp
// scratch. Writes the list to n_out output rows u = 0..n_out-1:
// idx_row[u * idx_stride + 0..W) (kept blocks ascending, then -1) and
// cnt_out[u * cnt_stride]. TMAX >= ceil((i+1)/32) bounds the blocks per lane.
//
// Candidates are the causal blocks outside the forced set; lane l owns blocks
// l, l+32, l+64, ..., whose order-preserving keys it keeps in registers. The k
// best (larger fp32 score first, lower block index on ties) are found as:
//  1. a lower bound L on the k-th best key: with r = ceil(k/32), every lane's
//     r-th largest key is >= the minimum of those over the warp, so at least
//     32r >= k keys are >= L (no bound when r > 4); keys >= L survive;
//  2. a most-significant-digit-first radix select over the survivors, from the
//     highest bit in which L and the largest key differ (the survivors agree on
//     every bit above it), 8 bits per pass: a histogram of the
//     current digit among survivors that match the prefix found so far picks
//     the digit holding the k-th best; it stops once every matching survivor
//     is needed;
//  3. survivors above the prefix are kept, and of those matching it the
//     lowest block indices, as many as still needed.
// ---------------------------------------------------------------------------
template <int TMAX>
__device__ void select_row(const float* s, uint32_t* hist, int i, int k, int lw, int ns, int W,
                           float tau, float c2, int32_t* __restrict__ idx_row,
                           int32_t* __restrict__ cnt_out, int n_out, size_t idx_stride,
                           size_t cnt_stride, WsHeader* hdr, int lane) {
  const int n = i + 1;
  const int win_lo = lw > 0 ? max(0, i - lw + 1) : n;  // window = [win_lo, i]
  const int nforced = (n - win_lo) + min(ns, win_lo);
  const int ncand = n - nforced;
  const int T = (n + 31) >> 5;
  const uint32_t lt = (1u << lane) - 1u;

  // Threshold rule (tau > 0): the budget shrinks to the candidates whose block
  // probability 2^(c2 (s_j - m)) / Z over the causal blocks reaches tau. The
  // passing candidates are the highest-scoring ones, so the top-k machinery
  // below then keeps exactly them (or the best k when more pass).
  if (tau > 0.f) {
    float m = -INFINITY;
#pragma unroll
    for (int t = 0; t < TMAX; ++t) {
      if (t >= T) break;
      const int j = t * 32 + lane;
      if (j < n) m = fmaxf(m, s[j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, off));
    float z = 0.f;
#pragma unroll
    for (int t = 0; t < TMAX; ++t) {
      if (t >= T) break;
      const int j = t * 32 + lane;
      if (j < n) z += exp2f(c2 * (s[j] - m));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(kFullMask, z, off);
    const float bar = tau * z;
    int passing = 0;
#pragma unroll
    for (int t = 0; t < TMAX; ++t) {
      if (t >= T) break;
      const int j = t * 32 + lane;
      const bool pass = j >= ns && j < win_lo && exp2f(c2 * (s[j] - m)) >= bar;
      passing += __popc(__ballot_sync(kFullMask, pass));
    }
    k = min(k, passing);
  }
  const int keff = min(k, ncand);

  // candidates are ns <= j < win_lo (the forced blocks are j < ns and j >= win_lo)
  uint32_t key[TMAX];  // 0: not a candidate (every finite score has a key >= 0x00800000)
#pragma unroll
  for (int t = 0; t < TMAX; ++t) {
    key[t] = 0u;
    if (t >= T) break;
    const int j = t * 32 + lane;
    if (j >= ns && j < win_lo) key[t] = ordered_key(s[j]);
  }

  uint32_t L = 1u;               // survivors: key >= L
  uint32_t prefix = 0, pmask = 0;
  int need = keff;               // still to take among survivors matching the prefix
  if (keff == 0) {
    L = 0xffffffffu;             // nothing survives (0xffffffff is not a finite key)
    need = 0;
  } else if (keff < ncand) {
    // 1. lower bound from each lane's r-th largest key; the largest key overall
    const int r = (keff + 31) >> 5;
    uint32_t kmax;
    if (r <= 2) {
      uint32_t t0 = 0, t1 = 0;  // this lane's two largest keys, descending
#pragma unroll
      for (int t = 0; t < TMAX; ++t) {
        if (t >= T) break;
        const uint32_t v = key[t];
        t1 = max(t1, min(t0, v));
        t0 = max(t0, v);
      }
      L = max(__reduce_min_sync(kFullMask, r == 1 ? t0 : t1), 1u);
      kmax = __reduce_max_sync(kFullMask, t0);
    } else if (r <= 4) {
      uint32_t t0 = 0, t1 = 0, t2 = 0, t3 = 0;  // this lane's largest keys, descending
#pragma unroll
      for (int t = 0; t < TMAX; ++t) {
        if (t >= T) break;
        uint32_t v = key[t], u;
        u = max(t0, v); v = min(t0, v); t0 = u;
        u = max(t1, v); v = min(t1, v); t1 = u;
        u = max(t2, v); v = min(t2, v); t2 = u;
        t3 = max(t3, v);
      }
      L = max(__reduce_min_sync(kFullMask, r == 3 ? t2 : t3), 1u);
      kmax = __reduce_max_sync(kFullMask, t0);
    } else {
      uint32_t m = 0;
#pragma unroll
      for (int t = 0; t < TMAX; ++t) {
        if (t >= T) break;
        m = max(m, key[t]);
      }
      kmax = __reduce_max_sync(kFullMask, m);
    }
    // 2. radix select; every survivor lies in [L, kmax], so the survivors agree
    // on all bits above the highest bit in which L and kmax differ
    const uint32_t diff = kmax ^ L;
    if (diff == 0u) {
      pmask = 0xffffffffu;  // all survivors equal: lowest indices win
      prefix = kmax;
    } else {
      int top = 31 - __clz(diff);
      pmask = top == 31 ? 0u : ~((2u << top) - 1u);
      prefix = kmax & pmask;
      while (top >= 0) {
        const int lo = max(top - 7, 0);
        const uint32_t dmask = (2u << (top - lo)) - 1u;
        reinterpret_cast<uint4*>(hist)[2 * lane] = make_uint4(0u, 0u, 0u, 0u);
        reinterpret_cast<uint4*>(hist)[2 * lane + 1] = make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();
#pragma unroll
        for (int t = 0; t < TMAX; ++t) {
          if (t >= T) break;
          if (key[t] >= L && (key[t] & pmask) == prefix) atomicAdd(&hist[(key[t] >> lo) & dmask], 1u);
        }
        __syncwarp();
        // bins 8*lane .. 8*lane+7; counts above a bin come from higher lanes
        const uint4 h0 = reinterpret_cast<const uint4*>(hist)[2 * lane];
        const uint4 h1 = reinterpret_cast<const uint4*>(hist)[2 * lane + 1];
        const uint32_t c[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
        const int tl = (int)(((c[0] + c[1]) + (c[2] + c[3])) + ((c[4] + c[5]) + (c[6] + c[7])));
        int incl = tl;  // sum over lanes >= this one
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_down_sync(kFullMask, incl, off);
          if (lane + off < 32) incl += y;
        }
        const int excl = incl - tl;
        const uint32_t owner = __ballot_sync(kFullMask, excl < need && need <= incl);
        const int ol = owner ? __ffs(owner) - 1 : 0;
        int dg = 0, above = excl, cnt_dg = 0;
        if (lane == ol) {
#pragma unroll
          for (int b = 7; b >= 0; --b) {
            if (above + (int)c[b] >= need) {
              dg = 8 * lane + b;
              cnt_dg = (int)c[b];
              break;
            }
            above += (int)c[b];
          }
        }
        dg = __shfl_sync(kFullMask, dg, ol);
        above = __shfl_sync(kFullMask, above, ol);
        cnt_dg = __shfl_sync(kFullMask, cnt_dg, ol);
        need -= above;
        prefix |= (uint32_t)dg << lo;
        pmask |= dmask << lo;
        if (cnt_dg == need) break;  // every survivor matching the prefix is taken
        top = lo - 1;
        __syncwarp();
      }
    }
  } else {
    need = ncand;  // every candidate is kept: L = 1, pmask = prefix = 0
  }

  // 3. emit forced blocks and picks in ascending block order
  int base = 0, rank_base = 0;
#pragma unroll
  for (int t = 0; t < TMAX; ++t) {
    if (t >= T) break;
    const int j = t * 32 + lane;
    const bool forced = j < n && (j < ns || j >= win_lo);
    const bool sv = key[t] >= L;  // L >= 1, so non-candidates (key 0) never survive
    const bool above = sv && ((key[t] & pmask) > prefix);
    const bool match = sv && ((key[t] & pmask) == prefix);
    const uint32_t mm = __ballot_sync(kFullMask, match);
    const int rk = rank_base + __popc(mm & lt);
    rank_base += __popc(mm);
    const bool sel = forced || above || (match && rk < need);
    const uint32_t sm = __ballot_sync(kFullMask, sel);
    const int pos = base + __popc(sm & lt);
    if (sel) {
      if (pos < W) {
        for (int u = 0; u < n_out; ++u) idx_row[u * idx_stride + pos] = j;
      } else {
        raise_error(hdr, DSA_ERR_DEVICE_BOUNDS, kKernSelect, i, pos);
      }
    }
    base += __popc(sm);
  }
  for (int u = 0; u < n_out; ++u) {
    for (int p = base + lane; p < W; p += 32) idx_row[u * idx_stride + p] = -1;
    if (lane == 0) cnt_out[u * cnt_stride] = min(base, W);
  }
  __syncwarp();
}

}  // namespace
}  // namespace dsa
