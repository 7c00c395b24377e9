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
// Two kernels. decode_score_kernel spreads the block scores over many CTAs
// (a warp per pooled row, lanes across the head dimension, one partial dot
// per query head of the KV head, butterfly sums). decode_attn_kernel runs one
// CTA per (batch, KV head, chunk of <= 8 query heads, split): every CTA of a
// chunk selects the chunk's rows from the stored scores (the same lists in
// every split), forms the union of the kept blocks with a bitmask of the heads
// that keep each, and takes every S-th block of that union. A block's present
// keys and values are contiguous rows of the cache: one bulk copy each (TMA,
// completing on the stage's mbarrier) fills a stage of a multi-stage ring in
// shared memory, so the loads of later blocks run under the arithmetic of
// earlier ones and each block crosses HBM once for all heads of the chunk. Attention is on the CUDA cores (one query
// row per head): warps are tied to heads; a lane owns one key of a 32-key
// chunk for q.k (head-dim chunks read in a lane-rotated order, free of bank
// conflicts) and d/32 output elements for P.V, with an online softmax per warp.
// Each CTA leaves its heads' partial states (m, l, o) in the workspace; the
// last CTA of the chunk to arrive (arrival counter) merges the splits in split
// order and writes out and lse.
#include "dsa_internal.cuh"
#include "select_row.cuh"

namespace dsa {
namespace {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kMaxSelGroup = 32;  // the group-shared rule allows group <= 32
constexpr int kMaxBlock = 128;    // largest block size
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
  float* scores;  // [B, Hq, nb] (group rule: [B, Hkv, nb] group sums)
  float* part;    // [B, Hq, S, d + 4]
  int* ctr;       // [B, Hkv, HC]
  int length;
  int S;          // splits of a chunk's kept blocks
  int NS;         // stages of the key/value ring
};

__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(kFullMask, x, off);
  return x;
}

// ---------------------------------------------------------------------------
// Block scores. CTA = (b, KV head g, head chunk, 32 rows); warp w scores rows
// j0 + 4w .. j0 + 4w + 3 for every query head of the chunk (all of the group's
// heads, summed in head order, in the group-shared rule).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kDecThreads)
decode_score_kernel(Shape s, DecodeArgs a) {
  constexpr int VPL = D / 32;              // head-dim elements per lane
  constexpr int RPW = kMaxBlock / kDecWarps;  // rows of the partial block per warp, at most
  __shared__ __align__(16) float qs[kMaxSelGroup * D];
  __shared__ __align__(16) float msum[kDecWarps][D];
  __shared__ __align__(16) float kmean[D];

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int G = s.group;
  const int HC = s.group_select ? 1 : (G + kDecHeadChunk - 1) / kDecHeadChunk;
  const int L = a.length, i = (L - 1) / s.bs, n = i + 1;
  const int C = (n + 31) / 32;
  int bid = blockIdx.x;
  const int c = bid % C;
  bid /= C;
  const int hc = bid % HC;
  bid /= HC;
  const int g = bid % s.Hkv, b = bid / s.Hkv;
  const int u0 = s.group_select ? 0 : hc * kDecHeadChunk;
  const int Gc = s.group_select ? G : min(kDecHeadChunk, G - u0);

  // the attention kernel may start its prologue now (it waits for this grid
  // to complete before it reads the scores or the counters)
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
  // arrival counters of the attention kernel start at zero every call
  if (blockIdx.x == 0) {
    const int nctr = s.B * s.Hkv * ((G + kDecHeadChunk - 1) / kDecHeadChunk);
    for (int e = tid; e < nctr; e += kDecThreads) a.ctr[e] = 0;
  }

  // Every global load is issued before the first barrier: the pooled rows
  // j < i of this warp, the query rows, and the present keys of block i.
  const int j0 = c * 32, j1 = min(j0 + 32, n);
  const bool own = j1 == n;  // this chunk holds row i, the token's partial block
  const float* const kp_head = a.kp + ((size_t)b * s.Hkv + g) * s.nb * D;
  float kv[4][VPL];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int j = j0 + warp * 4 + rr;
    if (j < i && j < j1) {
      const float* kr = kp_head + (size_t)j * D + lane * VPL;
      if constexpr (VPL == 4) {
        const float4 f = *reinterpret_cast<const float4*>(kr);
        kv[rr][0] = f.x, kv[rr][1] = f.y, kv[rr][2] = f.z, kv[rr][3] = f.w;
      } else {
        const float2 f = *reinterpret_cast<const float2*>(kr);
        kv[rr][0] = f.x, kv[rr][1] = f.y;
      }
    }
  }
  for (int e = tid; e < Gc * D; e += kDecThreads) {
    const int u = e / D, d = e % D;
    qs[e] = __bfloat162float(a.q[((size_t)b * s.Hq + g * G + u0 + u) * D + d]);
  }
  const int r0 = i * s.bs, nrow = L - r0;
  if (own) {
    // mean of the present keys of block i: warp w sums rows w, w + 8, ...
    const __nv_bfloat16* kr = a.k + (((size_t)b * s.Hkv + g) * s.N + r0) * D + lane * VPL;
    uint32_t raw[RPW][VPL / 2];
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      const int r = warp + rr * kDecWarps;
      if (r < nrow) {
        if constexpr (VPL == 4) {
          const uint2 w2 = *reinterpret_cast<const uint2*>(kr + (size_t)r * D);
          raw[rr][0] = w2.x, raw[rr][1] = w2.y;
        } else {
          raw[rr][0] = *reinterpret_cast<const uint32_t*>(kr + (size_t)r * D);
        }
      }
    }
    float acc[VPL];
#pragma unroll
    for (int e = 0; e < VPL; ++e) acc[e] = 0.f;
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      if (warp + rr * kDecWarps < nrow) {
#pragma unroll
        for (int e = 0; e < VPL / 2; ++e) {
          acc[2 * e] += bf_lo(raw[rr][e]);
          acc[2 * e + 1] += bf_hi(raw[rr][e]);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < VPL; ++e) msum[warp][lane * VPL + e] = acc[e];
  }
  __syncthreads();
  if (own && tid < D) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) t += msum[w][tid];
    kmean[tid] = t / (float)nrow;
  }
  __syncthreads();

#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int j = j0 + warp * 4 + rr;
    if (j >= j1) break;
    if (j == i) {
#pragma unroll
      for (int e = 0; e < VPL; ++e) kv[rr][e] = kmean[lane * VPL + e];
    }
    float tot = 0.f;
    for (int u = 0; u < Gc; ++u) {
      const float* qr = qs + u * D + lane * VPL;
      float x = 0.f;
#pragma unroll
      for (int e = 0; e < VPL; ++e) x = __fmaf_rn(qr[e], kv[rr][e], x);
      x = warp_sum(x);
      if (s.group_select) {
        tot = u == 0 ? x : __fadd_rn(tot, x);
      } else if (lane == 0) {
        a.scores[((size_t)b * s.Hq + g * G + u0 + u) * s.nb + j] = x;
      }
    }
    if (s.group_select && lane == 0) a.scores[((size_t)b * s.Hkv + g) * s.nb + j] = tot;
  }
}

// ---------------------------------------------------------------------------
// Attention. Shared memory (dynamic, offsets in 4-byte words, each region on a
// 16-byte boundary):
//   q      [8][D]   the chunk's query rows, fp32; per head the first D/2 words
//                   hold elements 8c..8c+3 of 16-byte chunk c, the last D/2
//                   elements 8c+4..8c+7 (lane-rotated reads hit distinct banks)
//   ublk   [nb]     union of the kept blocks, ascending
//   umask  [nb]     bit u: head u of the chunk keeps that block
//   pbuf   [8][32]  probabilities of a warp's current 32-key chunk
//   wml    [16]     per-warp m, l for the merge
//   wo     [8][D]   per-warp output rows for the merge
//   lcnt   [8]      list lengths; [8] = |union|; [9] = last-arrival flag; [10] abort
//   bars   [4]      one mbarrier (8 bytes) per stage of the ring
//   region          selection scratch (hist [8][256], lists [8][W], mask [nb],
//                   the score rows [8][nb]),
//                   then the key/value ring (NS stages of bs*D*2 bf16 each,
//                   filled by bulk copies that complete on the stage's mbarrier),
//                   then the merge's staging of (m, l) per (head, split)
// ---------------------------------------------------------------------------
__host__ __device__ constexpr int align4(int n) { return (n + 3) & ~3; }
constexpr int kCombHead = kDecHeadChunk * kDecMaxSplit + 2 * kDecHeadChunk;  // merge weights, l, M
constexpr int kMaxStages = 4;

struct AttnSmem {
  int q, ublk, umask, pbuf, wml, wo, lcnt, bars, region, hist, lists, mask, rows, total;
};

__host__ __device__ inline AttnSmem attn_smem(int D, int nb, int W, int bs, int NS) {
  AttnSmem m;
  m.q = 0;
  m.ublk = align4(m.q + kDecHeadChunk * D);
  m.umask = align4(m.ublk + nb);
  m.pbuf = align4(m.umask + nb);
  m.wml = align4(m.pbuf + kDecWarps * 32);
  m.wo = align4(m.wml + 2 * kDecWarps);
  m.lcnt = align4(m.wo + kDecWarps * D);
  m.bars = align4(m.lcnt + 12);
  m.region = align4(m.bars + 2 * kMaxStages);
  m.hist = m.region;
  m.lists = align4(m.hist + kDecWarps * kHistWords);
  m.mask = align4(m.lists + kDecWarps * W);
  m.rows = align4(m.mask + nb);
  const int sel = align4(m.rows + kDecHeadChunk * nb) - m.region;
  const int ring = NS * bs * D;  // K and V, bf16: 2 * bs * D * 2 bytes per stage
  const int comb = kCombHead + kDecHeadChunk * D;  // merge: weights, totals, one staged split
  m.total = m.region + (sel > ring ? (sel > comb ? sel : comb) : (ring > comb ? ring : comb));
  return m;
}

constexpr unsigned long long kDecWaitLimitNs = 1000000000ull;  // 1 s

// Non-suspending test of a phase.
__device__ __forceinline__ bool dbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// A wait with an abort flag uses the workspace header's limit when one is set
// (WsHeader::wait_limit_ns, so that a test can make it give up); the drain
// after an abort (abort_flag null) always allows the default limit. The spin
// polls without suspending and measures SM cycles (fine-grained, unlike the
// global timer), counting 2 cycles per ns: the limit holds at clocks up to
// 2 GHz and is longer below.
__device__ __noinline__ bool dbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            WsHeader* hdr, int where) {
  const long long c0 = clock64();
  unsigned long long limit = kDecWaitLimitNs;
  if (abort_flag != nullptr && hdr != nullptr) {
    const unsigned long long v = *reinterpret_cast<const volatile unsigned long long*>(&hdr->wait_limit_ns);
    if (v != 0ull) limit = v;
  }
  const long long lim_cycles = (long long)(limit < 4000000000ull ? limit : 4000000000ull) * 2;
  for (;;) {
    if (dbar_test(bar, parity)) return true;
    if (abort_flag != nullptr && *abort_flag) return false;
    if (clock64() - c0 > lim_cycles) {
      if (abort_flag != nullptr) *abort_flag = 1;
      raise_error(hdr, DSA_ERR_DEVICE_TIMEOUT, kKernDecode, where, (int)blockIdx.x);
      return false;
    }
  }
}

// The first probe does not suspend, so a stage that has not arrived always
// reaches the bounded spin (and its time limit).
__device__ __forceinline__ bool dbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          WsHeader* hdr, int where) {
  if (dbar_test(bar, parity)) return true;
  return dbar_wait_slow(bar, parity, abort_flag, hdr, where);
}

// bulk copy global -> shared of `bytes` (a multiple of 16, both addresses
// 16-byte aligned), completing as transaction bytes on the mbarrier `bar`
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }

template <int D, int TMAX>
__global__ void __launch_bounds__(kDecThreads)
decode_attn_kernel(Shape s, KBudget kb, DecodeArgs a) {
  constexpr int DPL = D / 32;  // output elements per lane
  constexpr int NCH = D / 8;   // 16-byte chunks of a bf16 key row
  extern __shared__ __align__(16) float sm[];
  const int W = s.W;
  const AttnSmem lay = attn_smem(D, s.nb, W, s.bs, a.NS);
  float* const sq = sm + lay.q;
  int32_t* const ublk = reinterpret_cast<int32_t*>(sm + lay.ublk);
  uint32_t* const umask = reinterpret_cast<uint32_t*>(sm + lay.umask);
  float* const pbuf = sm + lay.pbuf;
  float* const wml = sm + lay.wml;
  float* const wo = sm + lay.wo;
  int32_t* const lcnt = reinterpret_cast<int32_t*>(sm + lay.lcnt);
  uint32_t* const hist = reinterpret_cast<uint32_t*>(sm + lay.hist);
  int32_t* const lists = reinterpret_cast<int32_t*>(sm + lay.lists);
  uint32_t* const mask = reinterpret_cast<uint32_t*>(sm + lay.mask);
  float* const srows = sm + lay.rows;
  float* const region = sm + lay.region;

  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int G = s.group, HC = (G + kDecHeadChunk - 1) / kDecHeadChunk, S = a.S;
  int bid = blockIdx.x;
  const int sp = bid % S;
  bid /= S;
  const int hc = bid % HC;
  bid /= HC;
  const int g = bid % s.Hkv, b = bid / s.Hkv;
  const int u0 = hc * kDecHeadChunk;
  const int Gc = min(kDecHeadChunk, G - u0);
  const int h0 = g * G + u0;  // first query head of the chunk
  const int L = a.length, i = (L - 1) / s.bs, n = i + 1;

  // query rows in the split-chunk layout
  for (int e = tid; e < Gc * D; e += kDecThreads) {
    const int u = e / D, d = e % D, ch = d / 8, w = d % 8;
    sq[u * D + (w < 4 ? ch * 4 + w : D / 2 + ch * 4 + (w - 4))] =
        __bfloat162float(a.q[((size_t)b * s.Hq + h0 + u) * D + d]);
  }

  // the scores and the zeroed counters come from decode_score_kernel (launched
  // as its programmatic dependent: wait for its completion)
  asm volatile("griddepcontrol.wait;\n" ::: "memory");

  // selection: warp u selects head u's row (the group's row once in the
  // group-shared rule); the rows are first copied from the workspace to
  // shared memory by all threads, every load in flight at once
  const int nsel = s.group_select ? 1 : Gc;
  {
    const float* rows = s.group_select ? a.scores + ((size_t)b * s.Hkv + g) * s.nb
                                       : a.scores + ((size_t)b * s.Hq + h0) * s.nb;
    for (int u = 0; u < nsel; ++u) {
#pragma unroll 4
      for (int j = tid; j < n; j += kDecThreads) srows[u * s.nb + j] = __ldcg(rows + (size_t)u * s.nb + j);
    }
    for (int j = tid; j < n; j += kDecThreads) mask[j] = 0u;
  }
  __syncthreads();
  if (warp < nsel) {
    const int k = s.per_head ? kb.k[h0 + warp] : kb.k[0];
    select_row<TMAX>(srows + warp * s.nb, hist + warp * kHistWords, i, k, s.lw, s.ns, W, s.tau, s.c2,
                     lists + warp * W, lcnt + warp, 1, 0, 0, a.hdr, lane);
  }
  __syncthreads();

  // the kept lists leave through split 0
  if (sp == 0 && a.idx != nullptr) {
    for (int e = tid; e < Gc * W; e += kDecThreads) {
      const int u = e / W, p = e % W;
      a.idx[((size_t)b * s.Hq + h0 + u) * W + p] = lists[(s.group_select ? 0 : u) * W + p];
    }
    if (tid < Gc) a.cnt[(size_t)b * s.Hq + h0 + tid] = lcnt[s.group_select ? 0 : tid];
  }
  // union of the kept blocks with the heads that keep each
  const uint32_t all_heads = (1u << Gc) - 1u;
  if (warp < nsel) {
    const int32_t* lst = lists + warp * W;
    for (int e = lane; e < lcnt[warp]; e += 32) {
      const int j = lst[e];
      if (s.group_select) mask[j] = all_heads;
      else atomicOr(&mask[j], 1u << warp);
    }
  }
  __syncthreads();
  if (warp == 0) {
    int U = 0;
    for (int j0 = 0; j0 < n; j0 += 32) {
      const int j = j0 + lane;
      const uint32_t mk = j < n ? mask[j] : 0u;
      const uint32_t bal = __ballot_sync(kFullMask, mk != 0u);
      if (mk != 0u) {
        const int pos = U + __popc(bal & ((1u << lane) - 1u));
        ublk[pos] = j;
        umask[pos] = mk;
      }
      U += __popc(bal);
    }
    if (lane == 0) lcnt[8] = U;
  }
  if (tid == 0) {
    lcnt[10] = 0;
    for (int st = 0; st < a.NS; ++st)
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"((uint32_t)__cvta_generic_to_shared(
                       sm + lay.bars + 2 * st))
                   : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // the bulk copies (async proxy) overwrite what the selection wrote here
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();  // the selection scratch is dead from here: the ring takes the region
  const int U = lcnt[8];
  const int nmine = sp < U ? (U - sp + S - 1) / S : 0;  // union entries sp, sp + S, ...

  // key/value ring: thread 0 fills a stage with two bulk copies (the block's
  // present key rows, then its value rows, each contiguous in the cache)
  const int NS = a.NS;
  const int stage_words = s.bs * D;  // K then V, bf16
  const uint32_t ring_base = (uint32_t)__cvta_generic_to_shared(region);
  const uint32_t bar0 = (uint32_t)__cvta_generic_to_shared(sm + lay.bars);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(lcnt + 10);
  const size_t kv_row0 = ((size_t)b * s.Hkv + g) * s.N;  // cache row of key 0 of this KV head
  auto issue = [&](int e, int stage) {
    const int blk = ublk[sp + e * S];
    const int t0 = blk * s.bs, nr = min(s.bs, L - t0);
    const uint32_t bytes = (uint32_t)nr * D * 2u;
    const uint32_t dk = ring_base + (uint32_t)stage * stage_words * 4u;
    const uint32_t dv = dk + (uint32_t)s.bs * D * 2u;
    const uint32_t bar = bar0 + 8u * stage;
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(2u * bytes)
                 : "memory");
    bulk_g2s(dk, a.k + (kv_row0 + t0) * D, bytes, bar);
    bulk_g2s(dv, a.v + (kv_row0 + t0) * D, bytes, bar);
  };

  // warp -> head: head u = warp % Gc; the warps of a head split its key chunks
  const int u = warp % Gc;
  const int wr = warp / Gc, nw = (kDecWarps - u + Gc - 1) / Gc;
  const float4* const qa4 = reinterpret_cast<const float4*>(sq + u * D);
  const float4* const qb4 = qa4 + NCH;
  const float c2 = s.c2;
  float m = -INFINITY, l = 0.f;
  float o[DPL];
#pragma unroll
  for (int e = 0; e < DPL; ++e) o[e] = 0.f;
  float* const pw = pbuf + warp * 32;

  int issued = 0, landed = 0;  // stages issued and waited for (thread 0's count)
  if (tid == 0) {
    for (; issued < NS - 1 && issued < nmine; ++issued) issue(issued, issued);
  }
  for (int e = 0; e < nmine; ++e) {
    // stage (e + NS - 1) % NS was released by the barrier that ended step e - 1
    if (tid == 0 && e + NS - 1 < nmine && !*abort_flag) {
      issue(e + NS - 1, (e + NS - 1) % NS);
      ++issued;
    }
    const bool ok = dbar_wait(bar0 + 8u * (e % NS), (e / NS) & 1, abort_flag, a.hdr, 1);
    if (ok) landed = e + 1;
    const int ue = sp + e * S;
    const int blk = ublk[ue];
    const int nr = min(s.bs, L - blk * s.bs);
    if (ok && ((umask[ue] >> u) & 1u)) {
      const __nv_bfloat16* const sK = reinterpret_cast<const __nv_bfloat16*>(region + (e % NS) * stage_words);
      const __nv_bfloat16* const sV = sK + s.bs * D;
      for (int c = wr; c * 32 < nr; c += nw) {
        const int key = c * 32 + lane;
        const bool live = key < nr;
        float x = -INFINITY;
        if (live) {
          const uint4* kr = reinterpret_cast<const uint4*>(sK + key * D);
          float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
          for (int c16 = 0; c16 < NCH; ++c16) {
            const int ch = (c16 + lane) & (NCH - 1);
            const uint4 kw = kr[ch];
            const float4 fa = qa4[ch], fb = qb4[ch];
            acc0 = __fmaf_rn(fa.x, bf_lo(kw.x), acc0);
            acc1 = __fmaf_rn(fa.y, bf_hi(kw.x), acc1);
            acc0 = __fmaf_rn(fa.z, bf_lo(kw.y), acc0);
            acc1 = __fmaf_rn(fa.w, bf_hi(kw.y), acc1);
            acc0 = __fmaf_rn(fb.x, bf_lo(kw.z), acc0);
            acc1 = __fmaf_rn(fb.y, bf_hi(kw.z), acc1);
            acc0 = __fmaf_rn(fb.z, bf_lo(kw.w), acc0);
            acc1 = __fmaf_rn(fb.w, bf_hi(kw.w), acc1);
          }
          x = (acc0 + acc1) * c2;
        }
        float mc = x;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mc = fmaxf(mc, __shfl_xor_sync(kFullMask, mc, off));
        const float mn = fmaxf(m, mc);  // finite: key c*32 < nr is live
        const float alpha = exp2f(m - mn);
        const float pr = live ? exp2f(x - mn) : 0.f;
        l = l * alpha + pr;
#pragma unroll
        for (int e2 = 0; e2 < DPL; ++e2) o[e2] *= alpha;
        m = mn;
        pw[lane] = pr;
        __syncwarp();
        const int nk = min(32, nr - c * 32);
        const __nv_bfloat16* vr = sV + (c * 32) * D + lane * DPL;
        int t = 0;
        for (; t + 4 <= nk; t += 4) {
          const float4 p4 = *reinterpret_cast<const float4*>(pw + t);
          const float pp[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            if constexpr (DPL == 4) {
              const uint2 vw = *reinterpret_cast<const uint2*>(vr + (t + q4) * D);
              o[0] = __fmaf_rn(pp[q4], bf_lo(vw.x), o[0]);
              o[1] = __fmaf_rn(pp[q4], bf_hi(vw.x), o[1]);
              o[2] = __fmaf_rn(pp[q4], bf_lo(vw.y), o[2]);
              o[3] = __fmaf_rn(pp[q4], bf_hi(vw.y), o[3]);
            } else {
              const uint32_t vw = *reinterpret_cast<const uint32_t*>(vr + (t + q4) * D);
              o[0] = __fmaf_rn(pp[q4], bf_lo(vw), o[0]);
              o[1] = __fmaf_rn(pp[q4], bf_hi(vw), o[1]);
            }
          }
        }
        for (; t < nk; ++t) {
          const float pt = pw[t];
          if constexpr (DPL == 4) {
            const uint2 vw = *reinterpret_cast<const uint2*>(vr + t * D);
            o[0] = __fmaf_rn(pt, bf_lo(vw.x), o[0]);
            o[1] = __fmaf_rn(pt, bf_hi(vw.x), o[1]);
            o[2] = __fmaf_rn(pt, bf_lo(vw.y), o[2]);
            o[3] = __fmaf_rn(pt, bf_hi(vw.y), o[3]);
          } else {
            const uint32_t vw = *reinterpret_cast<const uint32_t*>(vr + t * D);
            o[0] = __fmaf_rn(pt, bf_lo(vw), o[0]);
            o[1] = __fmaf_rn(pt, bf_hi(vw), o[1]);
          }
        }
        __syncwarp();
      }
    }
    __syncthreads();  // the stage is refilled NS - 1 iterations later
  }
  if (tid == 0 && *abort_flag) {
    // a wait gave up: wait (bounded) for the copies still in flight before the
    // shared memory they write is reused or released
    for (int e = landed; e < issued; ++e)
      if (!dbar_wait(bar0 + 8u * (e % NS), (e / NS) & 1, nullptr, a.hdr, 2)) break;
  }
  __syncthreads();

  // merge the warps of each head; the CTA's partial state per head goes to the workspace
  l = warp_sum(l);
  if (lane == 0) {
    wml[warp] = m;
    wml[kDecWarps + warp] = l;
  }
#pragma unroll
  for (int e2 = 0; e2 < DPL; ++e2) wo[warp * D + lane * DPL + e2] = o[e2];
  __syncthreads();
  const int PS = D + 4;  // partial row: o[0..D), m, l, pad
  for (int e = tid; e < Gc * D; e += kDecThreads) {
    const int uu = e / D, d = e % D;
    float M = -INFINITY;
    for (int w = uu; w < kDecWarps; w += Gc) M = fmaxf(M, wml[w]);
    float lt = 0.f, ot = 0.f;
    if (M > -INFINITY) {
      for (int w = uu; w < kDecWarps; w += Gc) {
        const float f = exp2f(wml[w] - M);
        lt += f * wml[kDecWarps + w];
        ot += f * wo[w * D + d];
      }
    }
    float* prow = a.part + (((size_t)b * s.Hq + h0 + uu) * S + sp) * PS;
    prow[d] = ot;
    if (d == 0) {
      prow[D] = M;
      prow[D + 1] = lt;
    }
  }
  __threadfence();
  __syncthreads();
  int* const ctr = a.ctr + ((size_t)b * s.Hkv + g) * HC + hc;
  if (tid == 0) lcnt[9] = atomicAdd(ctr, 1) == S - 1 ? 1 : 0;
  __syncthreads();
  if (lcnt[9] == 0) return;

  // last CTA of the chunk: merge the S splits of each head in split order.
  // Warp u weighs head u's splits (f_q = 2^(m_q - M), zero for empty ones);
  // the partial rows are then staged in shared memory by asynchronous copies,
  // as many splits at a time as the region holds, and summed from there.
  __threadfence();
  float* const sf = region;                               // [Gc][S] weights
  float* const slt = region + kDecHeadChunk * kDecMaxSplit;  // [Gc] l totals, [Gc] M
  float* const stg = region + kCombHead;                  // staged rows [Gc][SC][D]
  if (warp < Gc) {
    const float* prow = a.part + ((size_t)b * s.Hq + h0 + warp) * S * PS;
    const float m0 = lane < S ? __ldcg(prow + (size_t)lane * PS + D) : -INFINITY;
    const float m1 = lane + 32 < S ? __ldcg(prow + (size_t)(lane + 32) * PS + D) : -INFINITY;
    const float l0 = lane < S ? __ldcg(prow + (size_t)lane * PS + D + 1) : 0.f;
    const float l1 = lane + 32 < S ? __ldcg(prow + (size_t)(lane + 32) * PS + D + 1) : 0.f;
    float M = fmaxf(m0, m1);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, off));
    const float f0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M);
    const float f1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M);
    const float lt = warp_sum(f0 * l0 + f1 * l1);
    if (lane < S) sf[warp * S + lane] = f0;
    if (lane + 32 < S) sf[warp * S + lane + 32] = f1;
    if (lane == 0) {
      slt[warp] = lt;
      slt[kDecHeadChunk + warp] = M;
    }
  }
  const int avail = lay.total - lay.region - kCombHead;
  const int SC = min(S, avail / (Gc * D));  // splits staged per round (>= 1 by the layout)
  constexpr int MI = kDecHeadChunk * D / kDecThreads;  // items e = tid + r * 256 of [Gc][D]
  float ot[MI];
#pragma unroll
  for (int r = 0; r < MI; ++r) ot[r] = 0.f;
  const uint32_t stg_s = (uint32_t)__cvta_generic_to_shared(stg);
  for (int q0 = 0; q0 < S; q0 += SC) {
    const int nq = min(SC, S - q0);
    const int per_row = D / 4;  // 16-byte pieces of a row
    for (int e = tid; e < Gc * nq * per_row; e += kDecThreads) {
      const int row = e / per_row, pc = e % per_row;
      const int uu = row / nq, q = q0 + row % nq;
      cp_async16(stg_s + (uint32_t)(row * D + pc * 4) * 4u,
                 a.part + (((size_t)b * s.Hq + h0 + uu) * S + q) * PS + pc * 4);
    }
    cp_async_commit();
    asm volatile("cp.async.wait_all;\n" ::: "memory");
    __syncthreads();
#pragma unroll 4
    for (int q = 0; q < nq; ++q) {
#pragma unroll
      for (int r = 0; r < MI; ++r) {
        const int e = tid + r * kDecThreads;
        const int uu = e / D, d = e % D;
        if (uu < Gc) ot[r] = __fmaf_rn(sf[uu * S + q0 + q], stg[(uu * nq + q) * D + d], ot[r]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < MI; ++r) {
    const int e = tid + r * kDecThreads;
    if (e < Gc * D) {
      const int uu = e / D, d = e % D;
      const float lt = slt[uu], M = slt[kDecHeadChunk + uu];
      const size_t row = (size_t)b * s.Hq + h0 + uu;
      a.out[row * D + d] = __float2bfloat16_rn(lt > 0.f ? ot[r] / lt : 0.f);
      if (a.lse != nullptr && d == 0) a.lse[row] = lt > 0.f ? M * kLn2Dec + logf(lt) : -INFINITY;
    }
  }
  if (tid == 0) *ctr = 0;
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

// ring depth: about 96 KB of keys and values in flight, 2 to 4 stages
inline int ring_stages(int bs, int D) {
  const int stage_bytes = bs * D * 4;
  const int ns = (96 * 1024) / stage_bytes;
  return ns < 2 ? 2 : ns > 4 ? 4 : ns;
}

template <int D, int TMAX>
cudaError_t launch_decode_d(const Shape& s, const KBudget& kb, DecodeArgs a, cudaStream_t st) {
  const int G = s.group, HC = (G + kDecHeadChunk - 1) / kDecHeadChunk;
  const int n = (a.length - 1) / s.bs + 1;
  // scores
  {
    const long long grid = (long long)s.B * s.Hkv * (s.group_select ? 1 : HC) * ((n + 31) / 32);
    if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    decode_score_kernel<D><<<(unsigned)grid, kDecThreads, 0, st>>>(s, a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // selection + attention + merge
  const long long cells = (long long)s.B * s.Hkv * HC;
  const long long want = (2LL * sm_count() + cells - 1) / cells;
  const int smax = decode_ws_layout(s).smax;
  a.S = (int)(want < 1 ? 1 : want > smax ? smax : want);
  if (a.S > n) a.S = n;
  a.NS = ring_stages(s.bs, D);
  const size_t smem = sizeof(float) * (size_t)attn_smem(D, s.nb, s.W, s.bs, a.NS).total;
  auto f = decode_attn_kernel<D, TMAX>;
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long grid = cells * a.S;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kDecThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, f, s, kb, a);
}

}  // namespace

cudaError_t launch_decode(const Shape& s, const KBudget& kb, const __nv_bfloat16* q,
                          const __nv_bfloat16* k, const __nv_bfloat16* v, const float* kp,
                          int length, __nv_bfloat16* out, float* lse, int32_t* idx, int32_t* cnt,
                          void* ws, cudaStream_t st) {
  const DecodeWs lw = decode_ws_layout(s);
  char* base = static_cast<char*>(ws);
  DecodeArgs a{q, k, v, kp, out, lse, idx, cnt, static_cast<WsHeader*>(ws),
               reinterpret_cast<float*>(base + lw.scores), reinterpret_cast<float*>(base + lw.part),
               reinterpret_cast<int*>(base + lw.ctr), length, 1, 2};
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
