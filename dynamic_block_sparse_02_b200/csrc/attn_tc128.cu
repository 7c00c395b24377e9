// Block-sparse causal attention forward (step 4) for 128x128 blocks on the
// tcgen05 tensor cores, head dim 64 or 128.
//
// What it computes is the same as the other attention kernels: for every
// query block i of (b, query head h), softmax(Q K^T * scale) V over the kept
// key blocks only, causal inside the diagonal block, with K/V of KV head
// h / (Hq/Hkv) ("稀疏注意力 vs Flash Attention v2", section 1; the zblog post's
// 128x128 blocks, section 工程实践建议; "DeepSeek NSA", section 2.2, bf16
// matmul with fp32 accumulation).
//
// With 128-row blocks a query block fills the N side of an MMA by itself, so
// one step takes one kept key block against the whole query block:
//     S^T (128 keys x 128 queries) = K_j (128 x d) . Q^T          (M=128, N=128)
//     O^T (d x 128 queries)       += V_j^T (d x 128 keys) . P^T    (M=d,   N=128)
// Both products run at the full N=128 rate, and each key block crosses into
// shared memory once per query block. The two softmax warpgroups split the
// query columns: warpgroup w owns columns 64w .. 64w+63 of S^T, P^T and O^T
// (per-query maxima and row sums are per column, so the warpgroups never
// exchange data); a thread owns one key (TMEM lane) of S^T and one head-dim
// row of O^T (d = 64: the M=64 accumulator, rows in lanes 0-15 of each
// sub-partition). As in the other kernel the running maxima are raised only
// when a logit exceeds them by more than 2^8.
//
// Work items (one query block each) come from a global counter in
// KV-head-major order, longest rows first. One item is in flight; S^T is
// double-buffered so that the next key block's S^T overlaps this one's
// softmax, and the PV product of a step overlaps the next step's softmax.
//
// Warp roles (384 threads, one persistent CTA per SM):
//   warp 0      K producer: work items, kept lists, the Q tile and the K tiles
//   warp 1      issues S^T = K Q^T     (one thread)
//   warp 2      issues O^T += V^T P^T  (one thread)
//   warp 3      V producer
//   warps 4-11  softmax + epilogue, two warpgroups (query columns 0-63, 64-127)
//
// Shared memory (d = 128): Q 32 KB, one ring of three 32 KB stages that K and V
// tiles share (load 2n is K of step n, load 2n + 1 its V, stage = load mod 3;
// a stage is refilled after the product that read it commits to the stage's
// empty barrier), and two P^T tiles of 32 KB, so that the softmax of step n
// writes its P while the PV product of step n - 1 still reads the other tile.
// Every mbarrier wait is bounded; on expiry the kernel sets
// DSA_ERR_DEVICE_TIMEOUT, stops issuing work, drains and returns.
#include "tc_common.cuh"

namespace dsa {
namespace {

using namespace tc;

constexpr int kBS = 128;
constexpr int kThreads = 384;
constexpr float kTau = 8.0f;   // rescale threshold (log2 units)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D_>
struct Cfg128 {
  static constexpr int D = D_;
  static_assert(D == 64 || D == 128, "head dim");
  static constexpr int DH = D / 64;                 // 128-byte atoms per row
  static constexpr int TileBytes = kBS * D * 2;     // Q, K, V tiles: [DH][128 rows][128 B]
  static constexpr int Atom = kBS * 128;            // one d-atom of a tile
  static constexpr int PBytes = kBS * kBS * 2;      // P^T: [2 query halves][128 keys][128 B]
  static constexpr int NKV = 3;                     // stages of the shared K/V ring
  static constexpr int OffQ = 0;
  static constexpr int OffKV = OffQ + TileBytes;    // NKV stages
  static constexpr int OffP = OffKV + NKV * TileBytes;  // 2 tiles
  static constexpr int OffList = OffP + 2 * PBytes; // [slot][kMaxBlocks] int16
  static constexpr int OffRed = OffList + 2 * kMaxBlocks * 2;  // [wg][4][64] f32
  static constexpr int OffM = OffRed + 2 * 4 * 64 * 4;         // [wg][64] -(running max)
  static constexpr int OffL = OffM + 2 * 64 * 4;               // [wg][64] 1 / row sum
  static constexpr int OffA = OffL + 2 * 64 * 4;               // [wg][64] max increments
  static constexpr int OffBar = OffA + 2 * 64 * 4;
  static constexpr int NumBars = 28;
  static constexpr int OffMisc = OffBar + NumBars * 8;
  static constexpr int SmemBytes = OffMisc + 192 + 1024;
  static_assert(SmemBytes <= 232448, "shared memory budget");
  static constexpr uint32_t TmemCols = 512;         // S^T 2 x 128, O^T 128
  static constexpr uint32_t ColO = 256;
  static constexpr uint32_t IdescS = idesc_bf16(128, 128, 0, 0);  // A = K, B = Q (K-major)
  static constexpr uint32_t IdescPV = idesc_bf16(D, 128, 1, 1);   // A = V^T, B = P^T (MN-major)
};

// The ring's loads are numbered L = 0, 1, 2, ... (2n: K of step n, 2n + 1:
// its V); load L goes to stage L mod 3 as that stage's m-th load, m = L / 3.
// Since 3 is odd, a stage's loads alternate between K and V, and so do its
// readers. Each stage therefore has a pair of full and a pair of empty
// barriers, one per kind: every barrier then has a single waiter that sees
// each of its phases in order (the K producer waits on EMPTY_V, the V
// producer on EMPTY_K, the S issuer on FULL_K, the PV issuer on FULL_V), and
// a load's phase on its own barriers is m / 2, parity (m >> 1) & 1.
enum {
  B_ITEM_FULL = 0,   // [2] slots
  B_ITEM_EMPTY = 2,  // [2]
  B_Q_FULL = 4,
  B_Q_EMPTY = 5,     // the item's last S^T has completed
  B_FULL_K = 6,      // [NKV] a K tile has landed in the stage
  B_FULL_V = 9,      // [NKV] a V tile has landed in the stage
  B_EMPTY_K = 12,    // [NKV] the S^T product that read the stage's K has completed
  B_EMPTY_V = 15,    // [NKV] the PV product that read the stage's V has completed
  B_S_FULL = 18,     // [2] S^T buffer n & 1 written
  B_S_FREE = 20,     // [2] both warpgroups have read S^T buffer n & 1
  B_P_FULL = 22,     // [2] P^T tile n & 1 written (256 arrivals)
  B_P_EMPTY = 24,    // [2] the PV that read P^T tile n & 1 has completed
  B_O_DONE = 26,     // the item's last PV has completed
  B_O_FREE = 27      // the epilogue has read O^T (256 arrivals)
};

struct Item128 {
  int b, h, i, n, diag_last;
};

struct Args128 {
  const int32_t* idx;
  const int32_t* cnt;
  __nv_bfloat16* out;
  float* lse;
  WsHeader* hdr;
  int B, Hq, Hkv, N, nb, W, group;
  int n_items;
  float scale_log2;
};

// Column reductions of 64 columns over a warp (see attn_tc.cu): afterwards
// v[0], v[1] hold columns col0, col0 + 1; col0 is returned.
template <bool kMax>
__device__ __forceinline__ int col_reduce64(float (&v)[64], int lane) {
  int col0 = 0;
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int off = 16 >> s;
    const int half = 64 >> (s + 1);
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < half; ++j) {
      const float send = up ? v[j] : v[j + half];
      const float keep = up ? v[j + half] : v[j];
      const float got = __shfl_xor_sync(0xffffffffu, send, off);
      v[j] = kMax ? fmaxf(keep, got) : (keep + got);
    }
    col0 += up ? half : 0;
  }
  return col0;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc128_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, Args128 a) {
  using C = Cfg128<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + C::OffBar;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + C::OffMisc);
  volatile uint32_t* sTotal = reinterpret_cast<volatile uint32_t*>(smem + C::OffMisc + 8);
  volatile uint32_t* sKMeta = reinterpret_cast<volatile uint32_t*>(smem + C::OffMisc + 16);  // [2]
  volatile uint32_t* sPMeta = reinterpret_cast<volatile uint32_t*>(smem + C::OffMisc + 24);  // [2]
  Item128* sItem = reinterpret_cast<Item128*>(smem + C::OffMisc + 32);  // [2] slots
  volatile CtaFlags* sFlags = reinterpret_cast<volatile CtaFlags*>(smem + C::OffMisc + 176);
  volatile int* sAbort = &sFlags->abort;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  auto bar = [&](int i) { return bars + 8u * i; };
  const WaitCtx wc{sFlags, a.hdr, kKernAttnTc};

  if (threadIdx.x == 0) {
    for (int u = 0; u < 2; ++u) {
      mbar_init(bar(B_ITEM_FULL + u), 1);
      mbar_init(bar(B_ITEM_EMPTY + u), 3);  // V producer + both warpgroups
      mbar_init(bar(B_P_FULL + u), 256);
      mbar_init(bar(B_P_EMPTY + u), 1);
      mbar_init(bar(B_S_FULL + u), 1);
      mbar_init(bar(B_S_FREE + u), 256);
    }
    mbar_init(bar(B_Q_FULL), 1);
    mbar_init(bar(B_Q_EMPTY), 1);
    for (int u = 0; u < C::NKV; ++u) {
      mbar_init(bar(B_FULL_K + u), 1);
      mbar_init(bar(B_FULL_V + u), 1);
      mbar_init(bar(B_EMPTY_K + u), 1);
      mbar_init(bar(B_EMPTY_V + u), 1);
    }
    mbar_init(bar(B_O_DONE), 1);
    mbar_init(bar(B_O_FREE), 256);
    sFlags->abort = 0;
    sFlags->limit_ns = wait_limit(a.hdr);
    *sTotal = 0xffffffffu;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(sTmem)),
                 "r"(C::TmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *sTmem;

  if (warp == 0) {
    // ------------------------------------------------------------------ K producer
    int16_t* const lists = reinterpret_cast<int16_t*>(smem + C::OffList);
    uint32_t n = 0;         // walk step (one kept block per step)
    uint32_t lastK = 0;     // bit u: stage u has had a K load; bit 8 + u: its phase parity
    uint32_t nq = 0;        // Q tiles loaded
    bool ok = true;
    for (int t = 0;; ++t) {
      const int slot = t & 1;
      if (lane == 0 && t >= 2) ok = ok && mbar_wait(bar(B_ITEM_EMPTY + slot), ((t >> 1) - 1) & 1, wc, 1);
      int item = 0;
      if (lane == 0) item = (!ok || *sAbort) ? a.n_items : (int)atomicAdd(&a.hdr->work[0], 1u);
      item = __shfl_sync(0xffffffffu, item, 0);
      if (item >= a.n_items) {
        if (lane == 0) {
          sItem[slot].n = -1;
          mbar_arrive(bar(B_ITEM_FULL + slot));
        }
        break;
      }
      int b, h, i;
      decode_item(item, a.group, a.nb, a.Hkv, b, h, i);
      const size_t row_id = ((size_t)b * a.Hq + h) * a.nb + i;
      int n_raw = a.cnt[row_id];
      if (n_raw < 0 || n_raw > a.W) {
        if (lane == 0) raise_error(a.hdr, DSA_ERR_DEVICE_BOUNDS, kKernAttnTc, (int)row_id, n_raw);
        n_raw = n_raw < 0 ? 0 : a.W;
      }
      const int32_t* lst = a.idx + row_id * a.W;
      int16_t* my_list = lists + slot * kMaxBlocks;
      int cntv = 0;
      for (int base = 0; base < n_raw; base += 32) {
        const int t2 = base + lane;
        const bool in = t2 < n_raw;
        const int j = in ? lst[t2] : -1;
        const bool valid = list_entry_ok(lst, t2, j, i, in);
        if (in && !valid) raise_error(a.hdr, DSA_ERR_DEVICE_BOUNDS, kKernAttnTc, (int)row_id, j);
        const uint32_t m = __ballot_sync(0xffffffffu, valid);
        if (valid) my_list[cntv + __popc(m & ((1u << lane) - 1u))] = (int16_t)j;
        cntv += __popc(m);
      }
      __syncwarp();
      if (lane == 0) {
        Item128& sl = sItem[slot];
        sl.b = b;
        sl.h = h;
        sl.i = i;
        sl.n = cntv;
        sl.diag_last = (cntv > 0 && my_list[cntv - 1] == i) ? 1 : 0;
        mbar_arrive(bar(B_ITEM_FULL + slot));
        if (cntv > 0) {
          // the previous item's last S^T has read the Q tile
          if (nq >= 1) ok = ok && mbar_wait(bar(B_Q_EMPTY), (nq - 1) & 1, wc, 2);
          if (ok) {
            const int qrow = (int)(((size_t)b * a.Hq + h) * a.N + (size_t)i * kBS);
            mbar_expect_tx(bar(B_Q_FULL), C::TileBytes);
#pragma unroll
            for (int hh = 0; hh < C::DH; ++hh)
              tma_load_2d(sbase + C::OffQ + hh * C::Atom, &tmQ, 64 * hh, qrow, bar(B_Q_FULL));
          }
          ++nq;
        }
        const int kvr = (int)(((size_t)b * a.Hkv + h / a.group) * a.N);
        for (int c = 0; c < cntv && ok; ++c, ++n) {
          // load L = 2n into stage L mod 3 once the V that was the stage's
          // previous load (L - 3) has been read
          const uint32_t L = 2 * n, ks = L % C::NKV, m = L / C::NKV;
          if (m > 0) ok = ok && mbar_wait(bar(B_EMPTY_V + ks), ((m - 1) >> 1) & 1, wc, 3);
          if (!ok) break;
          sKMeta[n & 1] = step_meta(0, c == 0, c == cntv - 1, 1);
          mbar_expect_tx(bar(B_FULL_K + ks), C::TileBytes);
          const int row = kvr + my_list[c] * kBS;
#pragma unroll
          for (int hh = 0; hh < C::DH; ++hh)
            tma_load_2d(sbase + C::OffKV + ks * C::TileBytes + hh * C::Atom, &tmK, 64 * hh, row,
                        bar(B_FULL_K + ks));
          lastK = (lastK & ~(0x101u << ks)) | (1u << ks) | (((m >> 1) & 1u) << (8 + ks));
        }
      }
      n = __shfl_sync(0xffffffffu, n, 0);
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
    }
    if (lane == 0) {
      *sTotal = n;
      // drain: every issued load has landed before the CTA may exit
      for (int u = 0; u < C::NKV; ++u)
        if (lastK & (1u << u)) mbar_drain(bar(B_FULL_K + u), (lastK >> (8 + u)) & 1u, a.hdr, kKernAttnTc, 5);
      if (nq > 0) mbar_drain(bar(B_Q_FULL), (nq - 1) & 1, a.hdr, kKernAttnTc, 5);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------------ V producer
    const int16_t* const lists = reinterpret_cast<const int16_t*>(smem + C::OffList);
    if (lane == 0) {
      uint32_t n = 0;
      uint32_t lastV = 0;   // as lastK of the K producer
      bool ok = true;
      for (int t = 0;; ++t) {
        const int slot = t & 1;
        ok = ok && mbar_wait(bar(B_ITEM_FULL + slot), (t >> 1) & 1, wc, 6);
        const Item128 it = sItem[slot];
        const int cntv = ok ? it.n : -1;
        if (cntv < 0) break;
        const int kvr = (int)(((size_t)it.b * a.Hkv + it.h / a.group) * a.N);
        for (int c = 0; c < cntv && ok; ++c, ++n) {
          // load L = 2n + 1 into stage L mod 3 once the K that was the
          // stage's previous load has been read
          const uint32_t L = 2 * n + 1, vs = L % C::NKV, m = L / C::NKV;
          if (m > 0) ok = ok && mbar_wait(bar(B_EMPTY_K + vs), ((m - 1) >> 1) & 1, wc, 4);
          if (!ok) break;
          mbar_expect_tx(bar(B_FULL_V + vs), C::TileBytes);
          const int row = kvr + lists[slot * kMaxBlocks + c] * kBS;
#pragma unroll
          for (int hh = 0; hh < C::DH; ++hh)
            tma_load_2d(sbase + C::OffKV + vs * C::TileBytes + hh * C::Atom, &tmV, 64 * hh, row,
                        bar(B_FULL_V + vs));
          lastV = (lastV & ~(0x101u << vs)) | (1u << vs) | (((m >> 1) & 1u) << (8 + vs));
        }
        mbar_arrive(bar(B_ITEM_EMPTY + slot));  // the slot's list has been read
        if (!ok) break;
      }
      for (int u = 0; u < C::NKV; ++u)
        if (lastV & (1u << u)) mbar_drain(bar(B_FULL_V + u), (lastV >> (8 + u)) & 1u, a.hdr, kKernAttnTc, 5);
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------------ MMA issuers
    const bool is_s = warp == 1;
    if (lane == 0) {
      bool ok = true;
      uint32_t nq = 0;   // S issuer: items started (Q tiles consumed)
      uint32_t no = 0;   // PV issuer: items finished (O^T accumulations completed)
      const uint64_t dK0 = smem_desc(sbase + C::OffKV, 16, 1024);
      const uint64_t dQ0 = smem_desc(sbase + C::OffQ, 16, 1024);
      const uint64_t dV0 = smem_desc(sbase + C::OffKV, C::Atom, 1024);
      const uint64_t dP0 = smem_desc(sbase + C::OffP, C::PBytes / 2, 1024);
      uint32_t n = 0;
      for (;; ++n) {
        const uint32_t u = n & 1;
        if (is_s) {
          const uint32_t L = 2 * n, ks = L % C::NKV;
          const int w = step_wait(bar(B_FULL_K + ks), ((L / C::NKV) >> 1) & 1, sTotal, n, wc, 14);
          if (w <= 0) break;
          const uint32_t meta = sKMeta[u];
          if (meta & 2u) ok = ok && mbar_wait(bar(B_Q_FULL), nq++ & 1, wc, 13);
          // both warpgroups have read the S^T of step n - 2 from this buffer
          if (n >= 2) ok = ok && mbar_wait(bar(B_S_FREE + u), ((n - 2) >> 1) & 1, wc, 15);
          tc_fence_after();
          if (ok) {
            const uint64_t dk = dK0 + (uint64_t)((ks * C::TileBytes) >> 4);
            const uint32_t d = tmem + u * 128;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              tc_mma(d, dk + (uint64_t)(((kk >> 2) * C::Atom + (kk & 3) * 32) >> 4),
                     dQ0 + (uint64_t)(((kk >> 2) * C::Atom + (kk & 3) * 32) >> 4), C::IdescS,
                     kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(B_S_FULL + u));
          tc_commit(bar(B_EMPTY_K + ks));  // the K tile's stage may be refilled
          if (meta & 4u) tc_commit(bar(B_Q_EMPTY));
        } else {
          const int w = step_wait(bar(B_P_FULL + u), (n >> 1) & 1, sTotal, n, wc, 10);
          if (w <= 0) break;
          const uint32_t meta = sPMeta[u];
          const uint32_t L = 2 * n + 1, vs = L % C::NKV;
          ok = ok && mbar_wait(bar(B_FULL_V + vs), ((L / C::NKV) >> 1) & 1, wc, 11);
          // a new item overwrites O^T: the previous item's epilogue has read it
          if ((meta & 2u) && no > 0) ok = ok && mbar_wait(bar(B_O_FREE), (no - 1) & 1, wc, 12);
          tc_fence_after();
          if (ok) {
            const uint64_t dv = dV0 + (uint64_t)((vs * C::TileBytes) >> 4);
            const uint64_t dp = dP0 + (uint64_t)((u * C::PBytes) >> 4);
            const uint32_t d = tmem + C::ColO;
#pragma unroll
            for (int kk = 0; kk < kBS / 16; ++kk)
              tc_mma(d, dv + (uint64_t)(kk * 128), dp + (uint64_t)(kk * 128), C::IdescPV,
                     (kk > 0 || !(meta & 2u)) ? 1u : 0u);
          }
          tc_commit(bar(B_P_EMPTY + u));    // P^T tile u may be rewritten
          tc_commit(bar(B_EMPTY_V + vs));  // the V tile's stage may be refilled
          if (meta & 4u) {
            tc_commit(bar(B_O_DONE));
            ++no;
          }
        }
      }
      // the tensor core has finished every MMA before TMEM is released
      if (n > 0) {
        if (is_s) mbar_drain(bar(B_S_FULL + ((n - 1) & 1)), ((n - 1) >> 1) & 1, a.hdr, kKernAttnTc, 17);
        else mbar_drain(bar(B_P_EMPTY + ((n - 1) & 1)), ((n - 1) >> 1) & 1, a.hdr, kKernAttnTc, 16);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int wg = (warp - 4) / 4;        // query columns 64 wg .. 64 wg + 63
    const int sp = warp & 3;              // TMEM sub-partition
    const int r = sp * 32 + lane;         // key row of S^T
    const int orow = D == 128 ? r : (lane < 16 ? sp * 16 + lane : -1);
    const int bar_id = 1 + wg;
    const int q0 = 64 * wg;
    const uint32_t lane_addr = (uint32_t)(sp * 32) << 16;
    const float c2 = a.scale_log2;
    float* const sRed = reinterpret_cast<float*>(smem + C::OffRed) + wg * 256;
    float* const sNM = reinterpret_cast<float*>(smem + C::OffM) + wg * 64;
    float* const sL = reinterpret_cast<float*>(smem + C::OffL) + wg * 64;
    float* const sA = reinterpret_cast<float*>(smem + C::OffA) + wg * 64;
    uint8_t* const prow0 = smem + C::OffP + wg * (C::PBytes / 2) + r * 128;  // tile 0
    const uint32_t o_addr = tmem + lane_addr + C::ColO + q0;
    float2 l2[32];
    float tmin = INFINITY;
    uint32_t n = 0;     // walk step
    uint32_t no = 0;    // items finished
    for (int t = 0;; ++t) {
      const int slot = t & 1;
      mbar_wait<true>(bar(B_ITEM_FULL + slot), (t >> 1) & 1, wc, 21);
      const Item128 it = sItem[slot];
      const bool stop = wg_any(bar_id, it.n < 0 || *sAbort != 0);
      if (r == 0) mbar_arrive(bar(B_ITEM_EMPTY + slot));
      if (stop) break;
#pragma unroll
      for (int q2 = 0; q2 < 32; ++q2) l2[q2] = make_float2(0.f, 0.f);
      for (int c = 0; c < it.n; ++c, ++n) {
        const uint32_t u = n & 1;
        mbar_wait<true>(bar(B_S_FULL + u), (n >> 1) & 1, wc, 22);
        tc_fence_after();
        const bool diag = (c == it.n - 1) && it.diag_last;
        const uint32_t s_addr = tmem + lane_addr + u * 128 + q0;
        uint32_t raw[64];
        tmem_ld(s_addr, raw);
        bool raise = c == 0;
        if (!raise) {
          float t8[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) t8[e] = __uint_as_float(raw[e]);
#pragma unroll
          for (int q = 8; q < 64; ++q) t8[q & 7] = fmaxf(t8[q & 7], __uint_as_float(raw[q]));
          const float mx = fmaxf(fmaxf(fmaxf(t8[0], t8[1]), fmaxf(t8[2], t8[3])),
                                 fmaxf(fmaxf(t8[4], t8[5]), fmaxf(t8[6], t8[7])));
          if (wg_any(bar_id, mx > tmin)) {
            bool part[8] = {false, false, false, false, false, false, false, false};
#pragma unroll
            for (int q4 = 0; q4 < 16; ++q4) {
              const float4 nm = reinterpret_cast<const float4*>(sNM)[q4];
              const float mm[4] = {nm.x, nm.y, nm.z, nm.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int q = 4 * q4 + e;
                part[q & 7] |= (__fmaf_rn(__uint_as_float(raw[q]), c2, mm[e]) > kTau) && !(diag && r > q0 + q);
              }
            }
            const bool big = ((part[0] | part[1]) | (part[2] | part[3])) | ((part[4] | part[5]) | (part[6] | part[7]));
            raise = wg_any(bar_id, big);
          }
        }
        if (raise) {
#pragma unroll
          for (int q4 = 0; q4 < 16; ++q4) {
            const float4 nm = c == 0 ? make_float4(0.f, 0.f, 0.f, 0.f) : reinterpret_cast<const float4*>(sNM)[q4];
            const float mm[4] = {nm.x, nm.y, nm.z, nm.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int q = 4 * q4 + e;
              const bool vis = !(diag && r > q0 + q);
              raw[q] = __float_as_uint(vis ? __fmaf_rn(__uint_as_float(raw[q]), c2, mm[e]) : -INFINITY);
            }
          }
          float* dv = reinterpret_cast<float*>(raw);
          const int col0 = col_reduce64<true>(*reinterpret_cast<float(*)[64]>(dv), lane);
          sRed[sp * 64 + col0] = dv[0];
          sRed[sp * 64 + col0 + 1] = dv[1];
          wg_sync(bar_id);
          if (r < 64) {
            const float mx = fmaxf(fmaxf(sRed[r], sRed[64 + r]), fmaxf(sRed[128 + r], sRed[192 + r]));
            const float inc = c == 0 ? mx : fmaxf(mx, 0.f);
            sA[r] = inc;
            sNM[r] = c == 0 ? -mx : sNM[r] - inc;
          }
          wg_sync(bar_id);
          {
            float mn = INFINITY;
#pragma unroll
            for (int q4 = 0; q4 < 16; ++q4) {
              const float4 nm = reinterpret_cast<const float4*>(sNM)[q4];
              mn = fminf(mn, fminf(fminf(-nm.x, -nm.y), fminf(-nm.z, -nm.w)));
            }
            tmin = c2 > 0.f ? (mn + kTau) / c2 : INFINITY;
          }
          if (c > 0) {
            // O^T holds every earlier step's contribution (the PV of step n - 1
            // has completed) before it is rescaled
            mbar_wait<true>(bar(B_P_EMPTY + ((n - 1) & 1)), ((n - 1) >> 1) & 1, wc, 20);
            tc_fence_after();
            tmem_ld(o_addr, raw);
#pragma unroll
            for (int q2 = 0; q2 < 32; ++q2) {
              const float2 al = make_float2(ex2(-sA[2 * q2]), ex2(-sA[2 * q2 + 1]));
              l2[q2] = __fmul2_rn(l2[q2], al);
              const float2 o = __fmul2_rn(make_float2(__uint_as_float(raw[2 * q2]), __uint_as_float(raw[2 * q2 + 1])), al);
              raw[2 * q2] = __float_as_uint(o.x);
              raw[2 * q2 + 1] = __float_as_uint(o.y);
            }
            tmem_st(o_addr, raw);
          }
          tmem_ld(s_addr, raw);
        }
        tc_fence_before();
        mbar_arrive(bar(B_S_FREE + u));
        // P = 2^(S * scale - m) in bf16, packed into registers first; the
        // single P^T tile is rewritten once the PV of step n - 1 has read it
        uint32_t pw[32];
        {
          const float2 c22 = make_float2(c2, c2);
#pragma unroll
          for (int q4 = 0; q4 < 16; ++q4) {
            const float4 nm4 = reinterpret_cast<const float4*>(sNM)[q4];
            const float2 nm[2] = {make_float2(nm4.x, nm4.y), make_float2(nm4.z, nm4.w)};
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int q = 4 * q4 + 2 * e;
              const float2 d2 = __ffma2_rn(make_float2(__uint_as_float(raw[q]), __uint_as_float(raw[q + 1])), c22, nm[e]);
              float p0 = ex2(d2.x), p1 = ex2(d2.y);
              if (diag) {
                p0 = r > q0 + q ? 0.f : p0;
                p1 = r > q0 + q + 1 ? 0.f : p1;
              }
              pw[q >> 1] = pack_bf16(p0, p1);
              l2[q >> 1].x = add_lo(l2[q >> 1].x, pw[q >> 1]);
              l2[q >> 1].y = add_hi(l2[q >> 1].y, pw[q >> 1]);
            }
          }
        }
        // P^T tile n & 1 was read by the PV of step n - 2
        if (n >= 2) mbar_wait<true>(bar(B_P_EMPTY + u), ((n - 2) >> 1) & 1, wc, 24);
        uint8_t* const prow = prow0 + u * C::PBytes;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          *reinterpret_cast<uint4*>(prow + ((cc ^ (r & 7)) << 4)) =
              make_uint4(pw[4 * cc], pw[4 * cc + 1], pw[4 * cc + 2], pw[4 * cc + 3]);
        if (r == 0 && wg == 0) sPMeta[u] = step_meta(0, c == 0, c == it.n - 1, 1);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(bar(B_P_FULL + u));
      }
      // ---------------------------------------------------------------- epilogue
      if (it.n > 0) {
        mbar_wait<true>(bar(B_O_DONE), no & 1, wc, 23);
      }
      tc_fence_after();
      {
        float* lf = reinterpret_cast<float*>(l2);
        const int col0 = col_reduce64<false>(*reinterpret_cast<float(*)[64]>(lf), lane);
        sRed[sp * 64 + col0] = lf[0];
        sRed[sp * 64 + col0 + 1] = lf[1];
      }
      wg_sync(bar_id);
      float lsum = 0.f;
      if (r < 64) {
        lsum = (sRed[r] + sRed[64 + r]) + (sRed[128 + r] + sRed[192 + r]);
        sL[r] = lsum > 0.f ? 1.0f / lsum : 0.f;
      }
      wg_sync(bar_id);
      const size_t row0 = ((size_t)it.b * a.Hq + it.h) * a.N + (size_t)it.i * kBS + q0;
      {
        uint32_t o[64];
        if (it.n > 0) {
          tmem_ld(o_addr, o);
        } else {
#pragma unroll
          for (int q = 0; q < 64; ++q) o[q] = 0u;
        }
        tc_fence_before();
        if (it.n > 0) {
          mbar_arrive(bar(B_O_FREE));  // O^T may be overwritten by the next item
          ++no;
        }
        if (orow >= 0) {
          __nv_bfloat16* const dst = a.out + row0 * D + orow;
#pragma unroll
          for (int q = 0; q < 64; ++q) dst[(size_t)q * D] = __float2bfloat16_rn(__uint_as_float(o[q]) * sL[q]);
        }
      }
      if (a.lse != nullptr && r < 64)
        a.lse[row0 + r] = (it.n > 0 && lsum > 0.f) ? (-sNM[r] * kLn2 + logf(lsum)) : -INFINITY;
      wg_sync(bar_id);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TmemCols)
                 : "memory");
  }
}

template <int D>
cudaError_t launch128(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                      const __nv_bfloat16* v, const int32_t* idx, const int32_t* cnt,
                      __nv_bfloat16* out, float* lse, WsHeader* hdr, cudaStream_t st) {
  using C = Cfg128<D>;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, (unsigned long long)s.B * s.Hq * s.N, D, kBS) ||
      !make_map(&mk, k, (unsigned long long)s.B * s.Hkv * s.N, D, kBS) ||
      !make_map(&mv, v, (unsigned long long)s.B * s.Hkv * s.N, D, kBS))
    return cudaErrorInvalidValue;
  Args128 a;
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
  a.n_items = s.B * s.Hq * s.nb;
  a.scale_log2 = s.scale * kLog2e;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(attn_tc128_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(&hdr->work[0], 0, sizeof(unsigned int), st);
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < sms ? a.n_items : sms;
  attn_tc128_kernel<D><<<grid, kThreads, C::SmemBytes, st>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_tc128(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                              const __nv_bfloat16* v, const int32_t* idx, const int32_t* cnt,
                              __nv_bfloat16* out, float* lse, WsHeader* hdr, cudaStream_t st) {
  if (s.bs != kBS) return cudaErrorNotSupported;
  if (s.d == 128) return launch128<128>(s, q, k, v, idx, cnt, out, lse, hdr, st);
  return launch128<64>(s, q, k, v, idx, cnt, out, lse, hdr, st);
}

}  // namespace dsa
