// Backward of the block-sparse causal attention on the tcgen05 tensor cores
// (64x64 blocks, head dim 64 or 128): dQ, dK, dV over the kept blocks with the
// kept lists held fixed. The gradient is the one written out in attn_bwd.cu
// (the DeepSeek NSA article, section 2.2, trains with the sparse pattern):
//   P = 2^(S * c2 - lse2),  dS = P * (dP - D),  D_r = dO_r . O_r,
//   dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO.
//
// Both passes have one shape. A work item has two fixed tiles F1, F2 of 64
// rows and a list of 128-row chunks X1, X2 streamed through shared memory:
//     A1  = X1 . F1^T              (M=128, N=64, K=d)   on TMEM
//     A2  = X2 . F2^T              (M=128, N=64, K=d)
//     P   = 2^(A1 * c2 - lse2),  G = P * (A2 - D)      (bf16, to shared memory)
//     Acc1 += X1^T . G             (M=d, N=64, K=128 rows)
//     Acc2 += X2^T . P             (dK/dV pass only)
//   dQ pass (item = query block (b, h, i)): F = (Q_i, dO_i), X = two kept key
//     blocks (K, V); A1 = S^T, A2 = dP^T, G = dS^T, Acc1 = dQ^T. lse2 and D
//     belong to the 64 query columns.
//   dK/dV pass (item = key block (b, g, j)): F = (K_j, V_j), X = the Q and dO
//     rows of two (query head, query block) pairs that keep j, taken in the
//     order of the transposed lists; A1 = S, A2 = dP, G = dS, Acc1 = dK^T,
//     Acc2 = dV^T. lse2 and D belong to the 128 streamed rows.
// Every sum runs in list order: the results are deterministic.
//
// One item is in flight; A1/A2 are double-buffered in TMEM so that the next
// chunk's products overlap this chunk's elementwise step, and the X rings are
// as deep as shared memory allows (a chunk's X1 stage stays busy from its load
// until its Acc products complete). The list entries of the dK/dV pass come
// through a 32-entry register window per producer warp, and the chunk rows'
// lse2 / D arrive by bulk copies on the chunk's barrier. Warp roles (384 threads, one persistent CTA/SM):
//   warp 0      X1 producer: work items, lists, F tiles, X1 chunks (and, in the
//               dK/dV pass, the lse2 / D values of the chunk's rows)
//   warp 1      issues A1 and A2 (one thread)
//   warp 2      issues Acc1 and Acc2 (one thread)
//   warp 3      X2 producer
//   warps 4-11  elementwise step and epilogue; warpgroup w owns the 32
//               columns 32w .. 32w+31 of A1, A2, G, P and the accumulators
// Every mbarrier wait is bounded; on expiry the kernel sets
// DSA_ERR_DEVICE_TIMEOUT, stops issuing work, drains and returns.
#include "tc_common.cuh"

namespace dsa {
namespace {

using namespace tc;

constexpr int kBS = 64;
constexpr int kRows = 128;    // rows of a streamed chunk (two blocks / two pairs)
constexpr int kThreads = 384;

template <int D_, bool DKV_>
struct BCfg {
  static constexpr int D = D_;
  static constexpr bool DKV = DKV_;
  static constexpr int DH = D / 64;
  static constexpr int FBytes = kBS * D * 2;        // F1 or F2: [DH][64 rows][128 B]
  static constexpr int FAtom = kBS * 128;
  static constexpr int XBytes = kRows * D * 2;      // a stage of X1 or X2: [DH][128 rows][128 B]
  static constexpr int XAtom = kRows * 128;
  static constexpr int GBytes = kRows * kBS * 2;    // G or P: [128 rows][64 columns] bf16
  // Ring depths. A stage of X1 is held from its load through the A products,
  // the elementwise step and the Acc products, so X1 gets the deepest ring
  // that shared memory allows; in the dQ pass X2 (V) is released right after
  // the A products and G is single-buffered to make room.
  static constexpr int NX1 = D == 64 ? 4 : (DKV ? 2 : 3);
  static constexpr int NX2 = D == 64 ? (DKV ? 4 : 3) : 2;
  static constexpr int NG = (DKV || D == 64) ? 2 : 1;
  static constexpr int NP = DKV ? 1 : 0;            // P tiles
  static constexpr int OffF1 = 0;
  static constexpr int OffF2 = OffF1 + FBytes;
  static constexpr int OffX1 = OffF2 + FBytes;
  static constexpr int OffX2 = OffX1 + NX1 * XBytes;
  static constexpr int OffG = OffX2 + NX2 * XBytes;
  static constexpr int OffP = OffG + NG * GBytes;
  static constexpr int OffList = OffP + NP * GBytes;                 // dQ: [slot][kMaxBlocks] int16
  static constexpr int ListBytes = DKV ? 0 : 2 * kMaxBlocks * 2;
  // dQ: [slot][64] float2 (lse2, D) of the query columns;
  // dK/dV: [stage][2][128] floats (lse2 row values, then D row values)
  static constexpr int OffLD = OffList + ListBytes;
  static constexpr int LDBytes = DKV ? NX1 * 2 * kRows * 4 : 2 * kBS * 8;
  static constexpr int OffPair = OffLD + LDBytes;                    // dK/dV: [stage][2] pair ids
  static constexpr int OffBar = OffPair + 32;
  static constexpr int NumBars = 40;
  static constexpr int OffMisc = OffBar + NumBars * 8;
  static constexpr int SmemBytes = OffMisc + 128 + 1024;
  static_assert(SmemBytes <= 232448, "shared memory budget");
  static_assert(NX1 <= 4 && NX2 <= 4 && NG <= 2, "barrier arrays");
  static constexpr uint32_t TmemCols = 512;
  // TMEM columns: A1[2] at 0, 64; A2[2] at 128, 192; Acc1 at 256; Acc2 at 320
  static constexpr uint32_t IdescA = idesc_bf16(kRows, kBS, 0, 0);  // X (K-major) . F^T (K-major)
  static constexpr uint32_t IdescAcc = idesc_bf16(D, kBS, 1, 1);    // X^T (MN-major) . G (MN-major)
};

enum {
  B_ITEM_FULL = 0,   // [2]
  B_ITEM_EMPTY = 2,  // [2]
  B_F_FULL = 4,
  B_F_EMPTY = 5,     // the item's last A products have completed
  B_A_FULL = 6,      // [2] A1 and A2 of the step written
  B_A_FREE = 8,      // [2] both warpgroups have read them (256 arrivals)
  B_G_FULL = 10,     // [NG] G of the step written (256 arrivals)
  B_G_EMPTY = 12,    // [NG] the Acc products that read it have completed
  B_P_FULL = 14,     // dK/dV pass: P of the step written (256 arrivals)
  B_P_EMPTY = 15,
  B_ACC_DONE = 16,   // the item's last Acc products have completed
  B_ACC_FREE = 17,   // the epilogue has read the accumulators (256 arrivals)
  B_X1_FULL = 18,    // [NX1]
  B_X1_EMPTY = 22,   // [NX1] the Acc products that read the stage have completed
  B_X2_FULL = 26,    // [NX2]
  B_X2_EMPTY = 30    // [NX2] the last products that read the stage have completed
};

struct BItem {
  int b, h, i, n, diag_last;  // dQ: query block (b, h, i); dK/dV: key block (b, g = h, j = i)
  long long pair_base;        // dK/dV: start of the item's pair list in BwdTcArgs::pairs
};
static_assert(sizeof(BItem) == 32, "item slot size");

// Start of the pair list of key block kb = (b, g, j): column j can be kept only
// by the G (nb - j) rows (u, i >= j), so the lists of one (b, g) are packed
// at offsets G * sum_{j' < j} (nb - j').
__device__ __forceinline__ long long pair_offset(const BwdTcArgs& a, size_t kb) {
  const long long nb = a.nb, G = a.group;
  const long long bg = (long long)(kb / a.nb), j = (long long)(kb % a.nb);
  return bg * G * (nb * (nb + 1) / 2) + G * (j * nb - j * (j - 1) / 2);
}

// Untiled bulk copy global -> shared completing on an mbarrier (both
// addresses 16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
               : "memory");
}

// A warp's window of 32 consecutive entries of a pair list, one per lane.
struct PairWindow {
  int base = -1 << 30;
  int val = -1;
  // entry e of the list (every lane calls with the same e)
  __device__ __forceinline__ int get(const int32_t* list, int count, int e, int lane) {
    if (e < base || e >= base + 32) {
      base = e;
      val = (e + lane < count) ? list[e + lane] : -1;
    }
    return __shfl_sync(0xffffffffu, val, e - base);
  }
};

template <bool DKV>
__device__ __forceinline__ void decode_bwd_item(const BwdTcArgs& a, int item, int& b, int& h, int& i) {
  if (!DKV) {
    decode_item(item, a.group, a.nb, a.Hkv, b, h, i);
  } else {
    // key blocks in ascending j (a column j can only be kept by rows i >= j,
    // so the long columns come first), the (batch, KV head) pairs interleaved
    const int bh = a.B * a.Hkv;
    i = item / bh;
    const int r = item - i * bh;
    b = r / a.Hkv;
    h = r - b * a.Hkv;
  }
}

template <int D, bool DKV>
__global__ void __launch_bounds__(kThreads, 1)
bwd_tc_kernel(const __grid_constant__ CUtensorMap tmF1, const __grid_constant__ CUtensorMap tmF2,
              const __grid_constant__ CUtensorMap tmX1, const __grid_constant__ CUtensorMap tmX2,
              BwdTcArgs a) {
  using C = BCfg<D, DKV>;
  constexpr int NX1 = C::NX1, NX2 = C::NX2, NG = C::NG;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + C::OffBar;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + C::OffMisc);
  volatile uint32_t* sTotal = reinterpret_cast<volatile uint32_t*>(smem + C::OffMisc + 8);
  volatile uint32_t* sXMeta = reinterpret_cast<volatile uint32_t*>(smem + C::OffMisc + 16);  // [NX1]
  volatile uint32_t* sGMeta = reinterpret_cast<volatile uint32_t*>(smem + C::OffMisc + 32);  // [NG]
  BItem* sItem = reinterpret_cast<BItem*>(smem + C::OffMisc + 40);                          // [2]
  volatile CtaFlags* sFlags = reinterpret_cast<volatile CtaFlags*>(smem + C::OffMisc + 104);
  volatile int* sAbort = &sFlags->abort;
  float* const sLDf = reinterpret_cast<float*>(smem + C::OffLD);
  float2* const sLD2 = reinterpret_cast<float2*>(smem + C::OffLD);
  int* const sPair = reinterpret_cast<int*>(smem + C::OffPair);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  auto bar = [&](int i) { return bars + 8u * i; };
  const WaitCtx wc{sFlags, a.hdr, kKernAttnBwd};

  if (threadIdx.x == 0) {
    for (int u = 0; u < 2; ++u) {
      mbar_init(bar(B_ITEM_FULL + u), 1);
      mbar_init(bar(B_ITEM_EMPTY + u), 3);  // X2 producer + both warpgroups
      mbar_init(bar(B_A_FULL + u), 1);
      mbar_init(bar(B_A_FREE + u), 256);
    }
    for (int u = 0; u < NG; ++u) {
      mbar_init(bar(B_G_FULL + u), 256);
      mbar_init(bar(B_G_EMPTY + u), 1);
    }
    for (int u = 0; u < NX1; ++u) {
      mbar_init(bar(B_X1_FULL + u), 1);
      mbar_init(bar(B_X1_EMPTY + u), 1);
    }
    for (int u = 0; u < NX2; ++u) {
      mbar_init(bar(B_X2_FULL + u), 1);
      mbar_init(bar(B_X2_EMPTY + u), 1);
    }
    mbar_init(bar(B_F_FULL), 1);
    mbar_init(bar(B_F_EMPTY), 1);
    mbar_init(bar(B_P_FULL), 256);
    mbar_init(bar(B_P_EMPTY), 1);
    mbar_init(bar(B_ACC_DONE), 1);
    mbar_init(bar(B_ACC_FREE), 256);
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
  const int n_items = DKV ? a.B * a.Hkv * a.nb : a.B * a.Hq * a.nb;

  if (warp == 0) {
    // ------------------------------------------------------------------ X1 producer
    int16_t* const lists = reinterpret_cast<int16_t*>(smem + C::OffList);
    uint32_t n = 0;       // walk step (one chunk per step)
    uint32_t nf = 0;      // F tile pairs loaded
    uint32_t lastX = 0;   // bit u: stage u has an issued load; bit 8+u: its parity
    bool ok = true;
    for (int t = 0;; ++t) {
      const int slot = t & 1;
      if (lane == 0 && t >= 2) ok = ok && mbar_wait(bar(B_ITEM_EMPTY + slot), ((t >> 1) - 1) & 1, wc, 1);
      int item = 0;
      if (lane == 0) item = (!ok || *sAbort) ? n_items : (int)atomicAdd(&a.hdr->work[0], 1u);
      item = __shfl_sync(0xffffffffu, item, 0);
      if (item >= n_items) {
        if (lane == 0) {
          sItem[slot].n = -1;
          mbar_arrive(bar(B_ITEM_FULL + slot));
        }
        break;
      }
      int b, h, i;
      decode_bwd_item<DKV>(a, item, b, h, i);
      int cntv = 0, diag_last = 0;
      long long pair_base = 0;
      if (!DKV) {
        // the query block's kept list, out-of-range and out-of-order entries dropped (and flagged)
        const size_t row_id = ((size_t)b * a.Hq + h) * a.nb + i;
        int n_raw = a.cnt[row_id];
        if (n_raw < 0 || n_raw > a.W) {
          if (lane == 0) raise_error(a.hdr, DSA_ERR_DEVICE_BOUNDS, kKernAttnBwd, (int)row_id, n_raw);
          n_raw = n_raw < 0 ? 0 : a.W;
        }
        const int32_t* lst = a.idx + row_id * a.W;
        int16_t* my_list = lists + slot * kMaxBlocks;
        for (int base = 0; base < n_raw; base += 32) {
          const int t2 = base + lane;
          const bool in = t2 < n_raw;
          const int j = in ? lst[t2] : -1;
          const bool valid = list_entry_ok(lst, t2, j, i, in);
          if (in && !valid) raise_error(a.hdr, DSA_ERR_DEVICE_BOUNDS, kKernAttnBwd, (int)row_id, j);
          const uint32_t m = __ballot_sync(0xffffffffu, valid);
          if (valid) my_list[cntv + __popc(m & ((1u << lane) - 1u))] = (int16_t)j;
          cntv += __popc(m);
        }
        __syncwarp();
        diag_last = (cntv > 0 && my_list[cntv - 1] == i) ? 1 : 0;
        // lse2 and D of the 64 query rows
        const size_t q0 = ((size_t)b * a.Hq + h) * a.N + (size_t)i * kBS;
        for (int r = lane; r < kBS; r += 32)
          sLD2[slot * kBS + r] = make_float2(a.lse2[q0 + r], a.drow[q0 + r]);
      } else {
        const size_t kb = ((size_t)b * a.Hkv + h) * a.nb + i;
        cntv = a.npairs[kb];
        pair_base = pair_offset(a, kb);
      }
      __syncwarp();
      if (lane == 0) {
        BItem& sl = sItem[slot];
        sl.b = b;
        sl.h = h;
        sl.i = i;
        sl.n = cntv;
        sl.diag_last = diag_last;
        sl.pair_base = pair_base;
        mbar_arrive(bar(B_ITEM_FULL + slot));
        if (cntv > 0) {
          // the previous item's last A products have read the F tiles
          if (nf >= 1) ok = ok && mbar_wait(bar(B_F_EMPTY), (nf - 1) & 1, wc, 2);
          if (ok) {
            const int frow = DKV ? (int)(((size_t)b * a.Hkv + h) * a.N + (size_t)i * kBS)
                                 : (int)(((size_t)b * a.Hq + h) * a.N + (size_t)i * kBS);
            mbar_expect_tx(bar(B_F_FULL), 2 * C::FBytes);
#pragma unroll
            for (int hh = 0; hh < C::DH; ++hh) {
              tma_load_2d(sbase + C::OffF1 + hh * C::FAtom, &tmF1, 64 * hh, frow, bar(B_F_FULL));
              tma_load_2d(sbase + C::OffF2 + hh * C::FAtom, &tmF2, 64 * hh, frow, bar(B_F_FULL));
            }
          }
          ++nf;
        }
      }
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
      // the chunks: two kept key blocks (dQ) or two pairs (dK/dV) each
      const int steps = (cntv + 1) >> 1;
      const int16_t* my_list = lists + slot * kMaxBlocks;
      const int32_t* plist = a.pairs + pair_base;
      PairWindow win;
      for (int c = 0; c < steps && ok; ++c, ++n) {
        const uint32_t u = n % NX1;
        const int nblk = min(2, cntv - 2 * c);
        int rows[2] = {0, 0}, pid[2] = {-1, -1};
        if (!DKV) {
          const int kvr = (int)(((size_t)b * a.Hkv + h / a.group) * a.N);
          for (int bb = 0; bb < nblk; ++bb) rows[bb] = kvr + my_list[2 * c + bb] * kBS;
        } else {
          // pair p = u_head * nb + i_q: rows of query head g*G + u_head, block i_q
          for (int bb = 0; bb < 2; ++bb) {
            const int pv = win.get(plist, cntv, 2 * c + bb, lane);
            if (bb < nblk) {
              pid[bb] = pv;
              const int uh = pv / a.nb, iq = pv - uh * a.nb;
              rows[bb] = (int)(((size_t)b * a.Hq + h * a.group + uh) * a.N + (size_t)iq * kBS);
            }
          }
        }
        if (lane == 0) {
          if (n >= (uint32_t)NX1) ok = mbar_wait(bar(B_X1_EMPTY + u), ((n / NX1) - 1) & 1, wc, 3);
          if (ok) {
            sXMeta[u] = step_meta(0, c == 0, c == steps - 1, nblk);
            if (DKV) {
              sPair[2 * u] = pid[0];
              sPair[2 * u + 1] = pid[1];
            }
            mbar_expect_tx(bar(B_X1_FULL + u), nblk * (kBS * D * 2 + (DKV ? 2 * kBS * 4 : 0)));
            for (int bb = 0; bb < nblk; ++bb) {
#pragma unroll
              for (int hh = 0; hh < C::DH; ++hh)
                tma_load_2d(sbase + C::OffX1 + u * C::XBytes + hh * C::XAtom + bb * kBS * 128, &tmX1, 64 * hh,
                            rows[bb], bar(B_X1_FULL + u));
              if (DKV) {
                // lse2 and D of the pair's 64 rows (contiguous, 256-byte aligned)
                const uint32_t ld = sbase + C::OffLD + u * (2 * kRows * 4) + bb * kBS * 4;
                bulk_load(ld, a.lse2 + rows[bb], kBS * 4, bar(B_X1_FULL + u));
                bulk_load(ld + kRows * 4, a.drow + rows[bb], kBS * 4, bar(B_X1_FULL + u));
              }
            }
            lastX = (lastX & ~(0x101u << u)) | (1u << u) | (((n / NX1) & 1u) << (8 + u));
          }
        }
        ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
        if (!ok) break;
      }
      n = __shfl_sync(0xffffffffu, n, 0);
    }
    if (lane == 0) {
      *sTotal = n;
      for (int u = 0; u < NX1; ++u)
        if (lastX & (1u << u)) mbar_drain(bar(B_X1_FULL + u), (lastX >> (8 + u)) & 1u, a.hdr, kKernAttnBwd, 5);
      if (nf > 0) mbar_drain(bar(B_F_FULL), (nf - 1) & 1, a.hdr, kKernAttnBwd, 5);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------------ X2 producer
    const int16_t* const lists = reinterpret_cast<const int16_t*>(smem + C::OffList);
    uint32_t n = 0;
    uint32_t lastX = 0;
    bool ok = true;
    for (int t = 0;; ++t) {
      const int slot = t & 1;
      // every lane waits, so that every lane's reads of the slot come after it
      ok = ok && mbar_wait(bar(B_ITEM_FULL + slot), (t >> 1) & 1, wc, 6);
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
      const BItem it = sItem[slot];
      const int cntv = ok ? it.n : -1;
      if (cntv < 0) break;
      const int steps = (cntv + 1) >> 1;
      const int32_t* plist = a.pairs + it.pair_base;
      PairWindow win;
      for (int c = 0; c < steps && ok; ++c, ++n) {
        const uint32_t u = n % NX2;
        const int nblk = min(2, cntv - 2 * c);
        int rows[2] = {0, 0};
        for (int bb = 0; bb < 2; ++bb) {
          if (!DKV) {
            if (bb < nblk)
              rows[bb] = (int)(((size_t)it.b * a.Hkv + it.h / a.group) * a.N) + lists[slot * kMaxBlocks + 2 * c + bb] * kBS;
          } else {
            const int pv = win.get(plist, cntv, 2 * c + bb, lane);
            const int uh = pv / a.nb, iq = pv - uh * a.nb;
            if (bb < nblk) rows[bb] = (int)(((size_t)it.b * a.Hq + it.h * a.group + uh) * a.N + (size_t)iq * kBS);
          }
        }
        if (lane == 0) {
          if (n >= (uint32_t)NX2) ok = mbar_wait(bar(B_X2_EMPTY + u), ((n / NX2) - 1) & 1, wc, 4);
          if (ok) {
            mbar_expect_tx(bar(B_X2_FULL + u), nblk * kBS * D * 2);
            for (int bb = 0; bb < nblk; ++bb) {
#pragma unroll
              for (int hh = 0; hh < C::DH; ++hh)
                tma_load_2d(sbase + C::OffX2 + u * C::XBytes + hh * C::XAtom + bb * kBS * 128, &tmX2, 64 * hh,
                            rows[bb], bar(B_X2_FULL + u));
            }
            lastX = (lastX & ~(0x101u << u)) | (1u << u) | (((n / NX2) & 1u) << (8 + u));
          }
        }
        ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
        if (!ok) break;
      }
      n = __shfl_sync(0xffffffffu, n, 0);
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_ITEM_EMPTY + slot));
      if (!ok) break;
    }
    if (lane == 0) {
      for (int u = 0; u < NX2; ++u)
        if (lastX & (1u << u)) mbar_drain(bar(B_X2_FULL + u), (lastX >> (8 + u)) & 1u, a.hdr, kKernAttnBwd, 5);
    }
  } else if (warp == 1 || warp == 2) {
    // ------------------------------------------------------------------ MMA issuers
    const bool is_a = warp == 1;
    if (lane == 0) {
      bool ok = true;
      uint32_t nf = 0;    // issuer A: items started
      uint32_t nacc = 0;  // issuer B: items finished
      const uint64_t dX1k = smem_desc(sbase + C::OffX1, 16, 1024);  // K-major views
      const uint64_t dX2k = smem_desc(sbase + C::OffX2, 16, 1024);
      const uint64_t dF1 = smem_desc(sbase + C::OffF1, 16, 1024);
      const uint64_t dF2 = smem_desc(sbase + C::OffF2, 16, 1024);
      const uint64_t dX1m = smem_desc(sbase + C::OffX1, C::XAtom, 1024);  // MN-major views
      const uint64_t dX2m = smem_desc(sbase + C::OffX2, C::XAtom, 1024);
      const uint64_t dG = smem_desc(sbase + C::OffG, C::GBytes, 1024);
      const uint64_t dP = smem_desc(sbase + C::OffP, C::GBytes, 1024);
      uint32_t n = 0;
      for (;; ++n) {
        const uint32_t u1 = n % NX1, u2 = n % NX2, ua = n & 1, ug = n % NG;
        if (is_a) {
          const int w = step_wait(bar(B_X1_FULL + u1), (n / NX1) & 1, sTotal, n, wc, 14);
          if (w <= 0) break;
          const uint32_t meta = sXMeta[u1];
          if (meta & 2u) ok = ok && mbar_wait(bar(B_F_FULL), nf++ & 1, wc, 13);
          ok = ok && mbar_wait(bar(B_X2_FULL + u2), (n / NX2) & 1, wc, 12);
          if (n >= 2) ok = ok && mbar_wait(bar(B_A_FREE + ua), ((n - 2) >> 1) & 1, wc, 15);
          tc_fence_after();
          if (ok) {
            const uint64_t x1 = dX1k + (uint64_t)((u1 * C::XBytes) >> 4);
            const uint64_t x2 = dX2k + (uint64_t)((u2 * C::XBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t xo = ((kk >> 2) * C::XAtom + (kk & 3) * 32) >> 4;
              const uint32_t fo = ((kk >> 2) * C::FAtom + (kk & 3) * 32) >> 4;
              tc_mma(tmem + ua * 64, x1 + xo, dF1 + fo, C::IdescA, kk > 0 ? 1u : 0u);
            }
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t xo = ((kk >> 2) * C::XAtom + (kk & 3) * 32) >> 4;
              const uint32_t fo = ((kk >> 2) * C::FAtom + (kk & 3) * 32) >> 4;
              tc_mma(tmem + 128 + ua * 64, x2 + xo, dF2 + fo, C::IdescA, kk > 0 ? 1u : 0u);
            }
          }
          tc_commit(bar(B_A_FULL + ua));
          if (!DKV) tc_commit(bar(B_X2_EMPTY + u2));  // V is read only by A2
          if (meta & 4u) tc_commit(bar(B_F_EMPTY));
        } else {
          const int w = step_wait(bar(B_G_FULL + ug), (n / NG) & 1, sTotal, n, wc, 10);
          if (w <= 0) break;
          const uint32_t meta = sGMeta[ug];
          const bool first = (meta & 2u) != 0;
          // a new item overwrites the accumulators: the previous epilogue has read them
          if (first && nacc > 0) ok = ok && mbar_wait(bar(B_ACC_FREE), (nacc - 1) & 1, wc, 11);
          tc_fence_after();
          // only the chunk's loaded rows enter (the rest of the stage is stale)
          const int ksteps = (int)(meta >> 3) * (kBS / 16);
          if (ok) {
            const uint64_t x1 = dX1m + (uint64_t)((u1 * C::XBytes) >> 4);
            const uint64_t g = dG + (uint64_t)((ug * C::GBytes) >> 4);
            for (int kk = 0; kk < ksteps; ++kk)
              tc_mma(tmem + 256, x1 + (uint64_t)(kk * 128), g + (uint64_t)(kk * 128), C::IdescAcc,
                     (kk > 0 || !first) ? 1u : 0u);
          }
          tc_commit(bar(B_G_EMPTY + ug));
          tc_commit(bar(B_X1_EMPTY + u1));
          if (DKV) {
            ok = ok && mbar_wait(bar(B_P_FULL), n & 1, wc, 9);
            tc_fence_after();
            if (ok) {
              const uint64_t x2 = dX2m + (uint64_t)((u2 * C::XBytes) >> 4);
              for (int kk = 0; kk < ksteps; ++kk)
                tc_mma(tmem + 320, x2 + (uint64_t)(kk * 128), dP + (uint64_t)(kk * 128), C::IdescAcc,
                       (kk > 0 || !first) ? 1u : 0u);
            }
            tc_commit(bar(B_P_EMPTY));
            tc_commit(bar(B_X2_EMPTY + u2));
          }
          if (meta & 4u) {
            tc_commit(bar(B_ACC_DONE));
            ++nacc;
          }
        }
      }
      // the tensor core has finished every MMA before TMEM is released: wait for
      // a commit issued after this thread's last MMA
      if (n > 0) {
        const uint32_t m = n - 1;
        if (is_a) mbar_drain(bar(B_A_FULL + (m & 1)), (m >> 1) & 1, a.hdr, kKernAttnBwd, 17);
        else if (DKV) mbar_drain(bar(B_P_EMPTY), m & 1, a.hdr, kKernAttnBwd, 16);
        else mbar_drain(bar(B_G_EMPTY + m % NG), (m / NG) & 1, a.hdr, kKernAttnBwd, 16);
      }
    }
  } else {
    // ------------------------------------------------------------------ elementwise + epilogue
    const int wg = (warp - 4) / 4;         // columns 32 wg .. 32 wg + 31
    const int sp = warp & 3;
    const int r = sp * 32 + lane;          // row of A1 / A2 (a key in dQ, a query row in dK/dV)
    const int orow = D == 128 ? r : (lane < 16 ? sp * 16 + lane : -1);  // head-dim row of the accumulators
    const int bar_id = 1 + wg;
    const int col0 = 32 * wg;
    const uint32_t lane_addr = (uint32_t)(sp * 32) << 16;
    const float c2 = a.c2;
    // 16-byte chunk cc (8 columns) of row r of a G / P tile sits at cc ^ (r & 7)
    uint8_t* const grow0 = smem + C::OffG + r * 128;
    uint8_t* const prow = smem + C::OffP + r * 128;
    uint32_t n = 0;
    uint32_t nacc = 0;
    for (int t = 0;; ++t) {
      const int slot = t & 1;
      mbar_wait<true>(bar(B_ITEM_FULL + slot), (t >> 1) & 1, wc, 21);
      const BItem it = sItem[slot];
      const bool stop = wg_any(bar_id, it.n < 0 || *sAbort != 0);
      // per-column lse2 and D (dQ pass), read before the slot is released
      float2 ldc[32];
      if (!DKV) {
#pragma unroll
        for (int k = 0; k < 32; ++k) ldc[k] = sLD2[slot * kBS + col0 + k];
      }
      wg_sync(bar_id);
      if (r == 0) mbar_arrive(bar(B_ITEM_EMPTY + slot));
      if (stop) break;
      const int steps = (it.n + 1) >> 1;
      for (int c = 0; c < steps; ++c, ++n) {
        const uint32_t ua = n & 1, u1 = n % NX1, ug = n % NG;
        const int nblk = min(2, it.n - 2 * c);
        const int blk = r / kBS, rl = r % kBS;
        const bool valid = blk < nblk;
        bool diag;
        float2 ldr = make_float2(0.f, 0.f);
        if (!DKV) {
          diag = (c == steps - 1) && it.diag_last && (blk == nblk - 1);
        } else {
          // this row's lse2 / D and pair, loaded with the X1 chunk
          mbar_wait<true>(bar(B_X1_FULL + u1), (n / NX1) & 1, wc, 25);
          ldr = make_float2(sLDf[u1 * 2 * kRows + r], sLDf[u1 * 2 * kRows + kRows + r]);
          const int pid = sPair[2 * u1 + (blk & 1)];
          diag = valid && (pid % a.nb) == it.i;
        }
        mbar_wait<true>(bar(B_A_FULL + ua), (n >> 1) & 1, wc, 22);
        tc_fence_after();
        uint32_t s[32], dp[32];
        tmem_ld(tmem + lane_addr + ua * 64 + col0, s);
        tmem_ld(tmem + lane_addr + 128 + ua * 64 + col0, dp);
        tc_fence_before();
        mbar_arrive(bar(B_A_FREE + ua));
        // P and G in bf16, packed in pairs of columns (two-wide fp32 math; a
        // row outside the chunk's loaded blocks is all zeros, the causal mask
        // applies in the diagonal block only)
        uint32_t gw[16], pw[16];
        if (!valid) {
#pragma unroll
          for (int k2 = 0; k2 < 16; ++k2) gw[k2] = pw[k2] = 0u;
        } else {
          const float2 c22 = make_float2(c2, c2);
#pragma unroll
          for (int k2 = 0; k2 < 16; ++k2) {
            const int k = 2 * k2, col = col0 + k;
            const float2 nl = DKV ? make_float2(-ldr.x, -ldr.x) : make_float2(-ldc[k].x, -ldc[k + 1].x);
            const float2 dv2 = DKV ? make_float2(ldr.y, ldr.y) : make_float2(ldc[k].y, ldc[k + 1].y);
            const float2 x2 = __ffma2_rn(make_float2(__uint_as_float(s[k]), __uint_as_float(s[k + 1])), c22, nl);
            float p0 = ex2(x2.x), p1 = ex2(x2.y);
            if (diag) {
              // dQ: row r is key rl, columns are queries; dK/dV: row r is query
              // rl, columns are keys
              if (DKV ? col > rl : rl > col) p0 = 0.f;
              if (DKV ? col + 1 > rl : rl > col + 1) p1 = 0.f;
            }
            const float2 dd = make_float2(__uint_as_float(dp[k]) - dv2.x, __uint_as_float(dp[k + 1]) - dv2.y);
            const float2 g2 = __fmul2_rn(make_float2(p0, p1), dd);
            if (DKV) pw[k2] = pack_bf16(p0, p1);
            gw[k2] = pack_bf16(g2.x, g2.y);
          }
        }
        // G: the tile was read by the Acc products of step n - NG
        if (n >= (uint32_t)NG) mbar_wait<true>(bar(B_G_EMPTY + ug), ((n / NG) - 1) & 1, wc, 24);
        uint8_t* const grow = grow0 + ug * C::GBytes;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          *reinterpret_cast<uint4*>(grow + (((4 * wg + cc) ^ (r & 7)) << 4)) =
              make_uint4(gw[4 * cc], gw[4 * cc + 1], gw[4 * cc + 2], gw[4 * cc + 3]);
        if (r == 0 && wg == 0) sGMeta[ug] = step_meta(0, c == 0, c == steps - 1, nblk);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(bar(B_G_FULL + ug));
        if (DKV) {
          // P: the single tile was read by the Acc2 products of step n - 1
          if (n >= 1) mbar_wait<true>(bar(B_P_EMPTY), (n - 1) & 1, wc, 26);
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            *reinterpret_cast<uint4*>(prow + (((4 * wg + cc) ^ (r & 7)) << 4)) =
                make_uint4(pw[4 * cc], pw[4 * cc + 1], pw[4 * cc + 2], pw[4 * cc + 3]);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          tc_fence_before();
          mbar_arrive(bar(B_P_FULL));
        }
      }
      // ---------------------------------------------------------------- epilogue
      uint32_t acc1[32], acc2[32];
      if (it.n > 0) {
        mbar_wait<true>(bar(B_ACC_DONE), nacc & 1, wc, 23);
        tc_fence_after();
        tmem_ld(tmem + lane_addr + 256 + col0, acc1);
        if (DKV) tmem_ld(tmem + lane_addr + 320 + col0, acc2);
        tc_fence_before();
        mbar_arrive(bar(B_ACC_FREE));
        ++nacc;
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) acc1[k] = acc2[k] = 0u;
      }
      if (orow >= 0) {
        // rows of the output block: 64 query rows (dQ) or 64 key rows (dK, dV);
        // this thread writes head-dim element orow of the warpgroup's 32 rows
        const size_t row0 = DKV ? (((size_t)it.b * a.Hkv + it.h) * a.N + (size_t)it.i * kBS + col0)
                                : (((size_t)it.b * a.Hq + it.h) * a.N + (size_t)it.i * kBS + col0);
        __nv_bfloat16* const d1 = (DKV ? a.dk : a.dq) + row0 * D + orow;
#pragma unroll
        for (int k = 0; k < 32; ++k) d1[(size_t)k * D] = __float2bfloat16_rn(__uint_as_float(acc1[k]) * a.scale);
        if (DKV) {
          __nv_bfloat16* const d2 = a.dv + row0 * D + orow;
#pragma unroll
          for (int k = 0; k < 32; ++k) d2[(size_t)k * D] = __float2bfloat16_rn(__uint_as_float(acc2[k]));
        }
      }
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

// Transposed lists as pair lists: one warp per key block (b, g, j) writes the
// bit positions u * nb + i of its bitmap, ascending, at pair_off[(b, g, j)].
__global__ void __launch_bounds__(256) bwd_pairs_kernel(BwdTcArgs a) {
  const size_t kb = (size_t)blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (kb >= (size_t)a.B * a.Hkv * a.nb) return;
  const uint32_t* bits = a.colbits + kb * a.cw;
  int32_t* out = a.pairs + pair_offset(a, kb);
  int total = 0;
  for (int w0 = 0; w0 < a.cw; w0 += 32) {
    const int w = w0 + lane;
    const uint32_t word = w < a.cw ? bits[w] : 0u;
    const int cntw = __popc(word);
    int pre = cntw;  // inclusive prefix over the lanes
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, pre, off);
      if (lane >= off) pre += y;
    }
    int pos = total + pre - cntw;
    uint32_t m = word;
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1;
      out[pos++] = w * 32 + bit;
    }
    total += __shfl_sync(0xffffffffu, pre, 31);
  }
  if (lane == 0) a.npairs[kb] = total;
}

template <int D, bool DKV>
cudaError_t launch_pass(const BwdTcArgs& a, const CUtensorMap& f1, const CUtensorMap& f2,
                        const CUtensorMap& x1, const CUtensorMap& x2, int sms, cudaStream_t st) {
  using C = BCfg<D, DKV>;
  cudaError_t e = cudaFuncSetAttribute(bwd_tc_kernel<D, DKV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(&a.hdr->work[0], 0, sizeof(unsigned int), st);
  if (e != cudaSuccess) return e;
  const long long items = DKV ? (long long)a.B * a.Hkv * a.nb : (long long)a.B * a.Hq * a.nb;
  const int grid = (int)(items < sms ? items : sms);
  bwd_tc_kernel<D, DKV><<<grid, kThreads, C::SmemBytes, st>>>(f1, f2, x1, x2, a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_bwd_tc_d(const BwdTcArgs& a, cudaStream_t st) {
  CUtensorMap mq, mdo, mk, mv;
  const unsigned long long qrows = (unsigned long long)a.B * a.Hq * a.N;
  const unsigned long long krows = (unsigned long long)a.B * a.Hkv * a.N;
  // boxes of 64 rows: every tile here is a whole 64-row block
  if (!make_map(&mq, a.q, qrows, D, kBS) || !make_map(&mdo, a.dout, qrows, D, kBS) ||
      !make_map(&mk, a.k, krows, D, kBS) || !make_map(&mv, a.v, krows, D, kBS))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  {
    const size_t kbs = (size_t)a.B * a.Hkv * a.nb;
    bwd_pairs_kernel<<<(unsigned)((kbs + 7) / 8), 256, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if ((e = launch_pass<D, false>(a, mq, mdo, mk, mv, sms, st)) != cudaSuccess) return e;
  return launch_pass<D, true>(a, mk, mv, mq, mdo, sms, st);
}

}  // namespace

bool attn_bwd_tc_supported(const Shape& s) {
  const unsigned long long rows = (unsigned long long)s.B * s.Hq * s.N;
  return s.bs == kBS && (s.d == 64 || s.d == 128) && rows < (1ull << 31) && encode_fn() != nullptr;
}

cudaError_t launch_attn_bwd_tc(const Shape& s, const BwdTcArgs& a, cudaStream_t st) {
  if (!attn_bwd_tc_supported(s)) return cudaErrorNotSupported;
  if (s.d == 128) return launch_bwd_tc_d<128>(a, st);
  return launch_bwd_tc_d<64>(a, st);
}

}  // namespace dsa
