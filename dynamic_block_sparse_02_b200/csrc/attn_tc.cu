// Block-sparse causal attention forward (step 4) on the 5th-generation tensor
// cores (tcgen05 + TMEM + TMA), for 32x32 and 64x64 blocks and head dim 64
// or 128 (one kernel template; 128x128 blocks run in attn_tc128.cu).
//
// What it computes is the same as the warp-MMA kernel: for every query block
// i of (b, query head h), softmax(Q K^T * scale) V over the kept key blocks
// only, causal inside the diagonal block, with K/V of KV head h / (Hq/Hkv)
// ("稀疏注意力 vs Flash Attention v2", section 1; FlashAttention-style online
// softmax; "DeepSeek NSA", section 2.2, bf16 matmul with fp32 accumulation).
//
// Shape of the computation on sm_100a. A query block has only bs = 32 or 64
// rows, and every (head, query block) keeps its own list of key blocks, so
// stacking query blocks into one 128-row MMA would multiply masked work.
// Instead the kernel computes transposed products whose 128-row side is the
// keys of 128/bs kept blocks (a "chunk"):
//     S^T (128 keys x bs queries) = K_chunk (128 x d) . Q^T        (M=128, N=bs)
//     O^T (d x bs queries)       += V_chunk^T (d x 128 keys) . P^T (M=d, N=bs)
// so the score MMAs run at M=128 without any wasted rows (at N=64 an MMA
// reads 6 KB of shared memory per 128x64x16 step, which bounds the tensor
// pipe at 2/3 of its N>=128 rate). With d = 64 the PV product is an M=64 MMA,
// whose accumulator row m sits in TMEM lane (m % 16) + 32 (m / 16). In TMEM a
// thread of a softmax warpgroup owns one key (lane) of S^T and one head-dim
// row of O^T. The softmax maximum
// is per query (a TMEM column), i.e. across threads; it is kept as a running
// value per query that is only raised when some logit exceeds it by more than
// 2^8 (decided by a warpgroup vote), which keeps P in [0, 2^8] and makes the
// cross-thread reduction and the rescale of O rare. Row sums are kept per
// thread and reduced once per query block.
//
// Warp roles (384 threads, one persistent CTA per SM):
//   warp 0        TMA producer: work items, kept lists, Q and K tiles
//   warp 1        issues S^T = K Q^T      (one thread)
//   warp 2        issues O^T += V^T P^T   (one thread)
//   warp 3        TMA producer of the V tiles
//   warps 4-7     softmax + epilogue of stream 0
//   warps 8-11    softmax + epilogue of stream 1
// A single issuing thread cannot issue N=64 MMAs as fast as the tensor core
// retires them, nor tensor-TMA loads as fast as L2 fills shared memory, so the
// two products and the K and V loads each come from their own warp. Two streams of work
// items (each with its own Q tile, TMEM S buffers, O accumulator and P tile)
// alternate chunk by chunk, so that one stream's softmax, rescale and
// epilogue overlap the other stream's MMAs. The producer and both issuers walk
// the same deterministic interleaving of (stream, chunk) steps, which is also
// the order of the shared K and V rings.
// Work items come from a global counter in KV-head-major order (the CTAs
// running at one time gather K/V of one KV head, which stays in L2), longest
// rows first inside a KV head.
//
// Every wait on an mbarrier is bounded (about 2 s); on expiry the kernel sets
// DSA_ERR_DEVICE_TIMEOUT in the workspace header, stops issuing work, drains
// and returns.
#include "tc_common.cuh"

namespace dsa {
namespace {

using namespace tc;

constexpr int kChunk = 128;    // keys per S^T tile
constexpr int kThreads = 384;
constexpr int kStreams = 2;
constexpr float kTau = 8.0f;   // rescale threshold (log2 units)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr int kMaxPT = 6;      // most P tiles of any shape
constexpr int kNumBars = 50;

// Sizes and shared-memory map for bs x bs blocks and head dim d. Every tile is
// a stack of 128-byte swizzle atoms [d / 64][rows][128 B] (K-major rows of
// 64 head-dim elements), except P^T: [128 keys][bs queries] bf16, MN-major,
// one 128-byte swizzled row per key for bs = 64 and one 64-byte swizzled row
// for bs = 32.
template <int BS_, int D_>
struct Cfg {
  static constexpr int BS = BS_, D = D_;
  static_assert((BS == 32 || BS == 64) && (D == 64 || D == 128), "shape");
  static constexpr int NBC = kChunk / BS;            // kept blocks per chunk
  static constexpr int DH = D / 64;                  // 128-byte atoms per row
  static constexpr int QBytes = BS * D * 2;
  static constexpr int KVBytes = kChunk * D * 2;
  static constexpr int KVAtom = kChunk * 128;        // bytes of one d-atom of a K/V stage
  static constexpr int QAtom = BS * 128;             // bytes of one d-atom of a Q tile
  static constexpr int PRow = BS * 2;                // bytes per key row of P^T
  static constexpr int PBytes = kChunk * PRow;
  static constexpr uint32_t PLayout = BS == 64 ? 2u : 4u;  // 128- / 64-byte swizzle
  // K and V ring stages: 16 KB stages (d = 64) need a deeper ring to hide the
  // copy latency behind the short steps; 32 KB stages fill shared memory at 2.
  static constexpr int NSTG = D == 64 ? 4 : 2;
  static constexpr int OffQ = 0;                           // one per stream
  static constexpr int OffK = OffQ + kStreams * QBytes;    // NSTG ring stages
  static constexpr int OffV = OffK + NSTG * KVBytes;       // NSTG ring stages
  // P tiles shared by the two streams (as many as shared memory holds, <= kMaxPT)
  static constexpr int PT = (BS == 64 && D == 128) ? 3 : (BS == 64 ? 4 : 6);
  static constexpr int OffP = OffV + NSTG * KVBytes;       // [PT]
  static constexpr int OffList = OffP + PT * PBytes;       // [stream][slot][kMaxBlocks] int16
  static constexpr int OffRed = OffList + kStreams * 2 * kMaxBlocks * 2;  // [stream][4][BS] f32
  static constexpr int OffM = OffRed + kStreams * 4 * BS * 4;  // [stream][BS] -(running max)
  static constexpr int OffL = OffM + kStreams * BS * 4;        // [stream][BS] 1 / row sum
  static constexpr int OffA = OffL + kStreams * BS * 4;        // [stream][BS] max increments
  static constexpr int OffBar = OffA + kStreams * BS * 4;      // mbarriers
  static constexpr int OffMisc = OffBar + kNumBars * 8;        // tmem base, item slots, step ids, wait flags
  static constexpr int SmemBytes = OffMisc + 192 + 1024;       // + alignment slack
  static_assert(PT <= kMaxPT, "P tiles");
  static_assert(QBytes % 1024 == 0 && KVBytes % 1024 == 0 && PBytes % 1024 == 0, "atom alignment");
  static_assert(SmemBytes <= 232448, "shared memory budget");
  // TMEM columns per stream: two S^T buffers and the O^T accumulator.
  static constexpr uint32_t TmemCols = 6 * BS <= 256 ? 256u : 512u;
  static constexpr uint32_t IdescS = idesc_bf16(128, BS, 0, 0);   // A = K, B = Q (both K-major)
  static constexpr uint32_t IdescPV = idesc_bf16(D, BS, 1, 1);    // A = V^T, B = P^T (MN-major)
  __device__ static __forceinline__ uint32_t col_s(int stream, uint32_t buf) {
    return stream * 3 * BS + buf * BS;
  }
  __device__ static __forceinline__ uint32_t col_o(int stream) { return stream * 3 * BS + 2 * BS; }
};

// barrier indices ([stream] or [stream][slot|buffer] or [stage])
enum {
  B_ITEM_FULL = 0,    // [2][2]
  B_ITEM_EMPTY = 4,   // [2][2]
  B_Q_FULL = 8,       // [2]
  B_Q_EMPTY = 10,     // [2]
  B_S_FULL = 12,      // [2][2]
  B_S_FREE = 16,      // [2][2]
  B_P_FULL = 20,      // [PT <= kMaxPT]
  B_P_EMPTY = 26,     // [PT]
  B_O_DONE = 32,      // [2]: the last PV of a stream's item has finished
  B_K_FULL = 34,      // [NSTG <= 4]
  B_K_EMPTY = 38,     // [NSTG] the S^T that read the stage has completed
  B_V_FULL = 42,      // [NSTG]
  B_V_EMPTY = 46      // [NSTG] the PV that read the stage has completed
};

// P tiles: step n of the (stream, chunk) walk writes tile n % PT, whose
// previous reader was step n - PT; the S^T issuer publishes each step's
// index next to its S^T buffer (sStep[stream][buffer]).

struct ItemSlot {
  int b, h, i, n, diag_last;
};

struct TcArgs {
  const int32_t* idx;
  const int32_t* cnt;
  __nv_bfloat16* out;
  float* lse;
  WsHeader* hdr;
  int B, Hq, Hkv, N, nb, W, group;
  int n_items;
  float scale_log2;
};

// Column-wise reductions over the 32 lanes of a warp for NC columns held one
// per register: afterwards v[0 .. NC/32) hold the reduced values of columns
// col0 .. col0 + NC/32 - 1; col0 is returned.
template <int NC, bool kMax>
__device__ __forceinline__ int warp_col_reduce(float (&v)[NC], int lane) {
  int col0 = 0;
#pragma unroll
  for (int s = 0; s < 5; ++s) {
    const int off = 16 >> s;     // lane distance of this round
    const int half = NC >> (s + 1);  // columns kept after this round
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

template <int BS, int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, TcArgs a) {
  using C = Cfg<BS, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + C::OffBar;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + C::OffMisc);
  volatile CtaFlags* sFlags = reinterpret_cast<volatile CtaFlags*>(smem + C::OffMisc + 176);
  volatile int* sAbort = &sFlags->abort;
  ItemSlot* sItem = reinterpret_cast<ItemSlot*>(smem + C::OffMisc + 16);  // [stream][slot]
  volatile uint32_t* sStep = reinterpret_cast<volatile uint32_t*>(smem + C::OffMisc + 112);  // [stream][S buffer]
  // step count of the whole walk, published by the K producer when it ends
  volatile uint32_t* sTotal = reinterpret_cast<volatile uint32_t*>(smem + C::OffMisc + 8);
  // per K stage and per P tile: stream and position of the step they hold
  volatile uint32_t* sKMeta = reinterpret_cast<volatile uint32_t*>(smem + C::OffMisc + 128);  // [NSTG]
  volatile uint32_t* sPMeta = reinterpret_cast<volatile uint32_t*>(smem + C::OffMisc + 144);  // [PT]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  auto bar = [&](int idx) { return bars + 8u * idx; };
  const WaitCtx wc{sFlags, a.hdr, kKernAttnTc};

  if (threadIdx.x == 0) {
    for (int x = 0; x < kStreams; ++x) {
      for (int u = 0; u < 2; ++u) {
        mbar_init(bar(B_ITEM_FULL + 2 * x + u), 1);
        mbar_init(bar(B_ITEM_EMPTY + 2 * x + u), 2);  // V producer + softmax
        mbar_init(bar(B_S_FULL + 2 * x + u), 2);  // MMA commit + step-id publication
        mbar_init(bar(B_S_FREE + 2 * x + u), 128);
      }
      mbar_init(bar(B_Q_FULL + x), 1);
      mbar_init(bar(B_Q_EMPTY + x), 1);
      mbar_init(bar(B_O_DONE + x), 1);
    }
    for (int u = 0; u < C::NSTG; ++u) {
      mbar_init(bar(B_K_FULL + u), 1);
      mbar_init(bar(B_K_EMPTY + u), 1);
      mbar_init(bar(B_V_FULL + u), 1);
      mbar_init(bar(B_V_EMPTY + u), 1);
    }
    for (int t = 0; t < C::PT; ++t) {
      mbar_init(bar(B_P_FULL + t), 128);
      mbar_init(bar(B_P_EMPTY + t), 1);
    }
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

  if (warp < 4) {
    if (warp == 0) {
      // ---------------------------------------------------------------- K producer
      // Fetches work items, compacts their kept lists into the item slot,
      // publishes them, and loads the Q tiles and the K tiles.
      int16_t* const lists = reinterpret_cast<int16_t*>(smem + C::OffList);
      uint32_t gk = 0;
      Pair<uint32_t> gq = {0u, 0u};
      // bit u set: ring stage (or Q buffer) u has an issued load; bit 8+u: its phase parity
      uint32_t lastK = 0, lastQ = 0;
      Pair<int> kvrow = {0, 0};
      Pair<int> nkept = {0, 0};
      bool ok = true;
      Walk<C::NBC> wk;
      wk.init();
      for (;;) {
        const int x = wk.pick();
        if (x < 0) break;
        if (wk.C.get(x) < 0) {
          // open the stream's next item: fetch it, compact its list, publish it
          const int tx = wk.t.get(x);
          const int slot = tx & 1;
          if (lane == 0 && tx >= 2)
            ok = ok && mbar_wait(bar(B_ITEM_EMPTY + 2 * x + slot), ((tx >> 1) - 1) & 1, wc, 1);
          int item = 0;
          if (lane == 0) item = (!ok || *sAbort) ? a.n_items : (int)atomicAdd(&a.hdr->work[0], 1u);
          item = __shfl_sync(0xffffffffu, item, 0);
          if (item >= a.n_items) {
            if (lane == 0) {
              sItem[2 * x + slot].n = -1;
              mbar_arrive(bar(B_ITEM_FULL + 2 * x + slot));
            }
            wk.done.set(x, 1);
            continue;
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
          int16_t* my_list = lists + (2 * x + slot) * kMaxBlocks;
          int n = 0;
          for (int base = 0; base < n_raw; base += 32) {
            const int t2 = base + lane;
            const bool in = t2 < n_raw;
            const int j = in ? lst[t2] : -1;
            const bool valid = list_entry_ok(lst, t2, j, i, in);
            if (in && !valid) raise_error(a.hdr, DSA_ERR_DEVICE_BOUNDS, kKernAttnTc, (int)row_id, j);
            const uint32_t m = __ballot_sync(0xffffffffu, valid);
            if (valid) my_list[n + __popc(m & ((1u << lane) - 1u))] = (int16_t)j;
            n += __popc(m);
          }
          __syncwarp();
          if (lane == 0) {
            ItemSlot& sl = sItem[2 * x + slot];
            sl.b = b;
            sl.h = h;
            sl.i = i;
            sl.n = n;
            sl.diag_last = (n > 0 && my_list[n - 1] == i) ? 1 : 0;
            mbar_arrive(bar(B_ITEM_FULL + 2 * x + slot));
            if (n > 0) {
              const uint32_t gqx = gq.get(x);
              if (gqx >= 1) ok = ok && mbar_wait(bar(B_Q_EMPTY + x), (gqx - 1) & 1, wc, 2);
              if (ok) {
                const int qrow = (int)(((size_t)b * a.Hq + h) * a.N + (size_t)i * BS);
                mbar_expect_tx(bar(B_Q_FULL + x), C::QBytes);
                const uint32_t dq = sbase + C::OffQ + x * C::QBytes;
#pragma unroll
                for (int hh = 0; hh < C::DH; ++hh)
                  tma_load_2d(dq + hh * C::QAtom, &tmQ, 64 * hh, qrow, bar(B_Q_FULL + x));
                lastQ = (lastQ & ~(0x101u << x)) | (1u << x) | ((gqx & 1u) << (8 + x));
              }
              gq.inc(x);
            }
          }
          __syncwarp();
          kvrow.set(x, (int)(((size_t)b * a.Hkv + h / a.group) * a.N));
          nkept.set(x, n);
          wk.open(x, n);
          continue;
        }
        // one step: the K tile of chunk c of stream x
        if (lane == 0 && ok) {
          const int c = wk.c.get(x);
          const int nblk = min(C::NBC, nkept.get(x) - C::NBC * c);
          const int kvr = kvrow.get(x);
          const int16_t* my_list = lists + (2 * x + (wk.t.get(x) & 1)) * kMaxBlocks;
          const uint32_t ks = gk % C::NSTG;
          // the stage's previous tile was read by the S^T of load gk - NSTG
          if (gk >= (uint32_t)C::NSTG) ok = ok && mbar_wait(bar(B_K_EMPTY + ks), ((gk / C::NSTG) - 1) & 1, wc, 3);
          if (ok) {
            sKMeta[ks] = step_meta(x, c == 0, c == wk.C.get(x) - 1, nblk);
            mbar_expect_tx(bar(B_K_FULL + ks), nblk * BS * D * 2);
            const uint32_t dk = sbase + C::OffK + ks * C::KVBytes;
            for (int bb = 0; bb < nblk; ++bb) {
              const int row = kvr + my_list[C::NBC * c + bb] * BS;
#pragma unroll
              for (int hh = 0; hh < C::DH; ++hh)
                tma_load_2d(dk + hh * C::KVAtom + bb * BS * 128, &tmK, 64 * hh, row, bar(B_K_FULL + ks));
            }
            lastK = (lastK & ~(0x101u << ks)) | (1u << ks) | (((gk / C::NSTG) & 1u) << (8 + ks));
          }
        }
        ++gk;
        ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
        wk.advance(x);
      }
      if (lane == 0) *sTotal = gk;
      // drain: every issued load has landed before the CTA may exit
      if (lane == 0) {
        for (int u = 0; u < C::NSTG; ++u)
          if (lastK & (1u << u)) mbar_drain(bar(B_K_FULL + u), (lastK >> (8 + u)) & 1u, a.hdr, kKernAttnTc, 5);
        for (int u = 0; u < kStreams; ++u)
          if (lastQ & (1u << u)) mbar_drain(bar(B_Q_FULL + u), (lastQ >> (8 + u)) & 1u, a.hdr, kKernAttnTc, 5);
      }
    } else if (warp == 3) {
      // ---------------------------------------------------------------- V producer
      // Walks the same steps; reads each item's kept list from its slot and
      // releases the slot after the item's last V tile has been issued.
      const int16_t* const lists = reinterpret_cast<const int16_t*>(smem + C::OffList);
      if (lane == 0) {
        uint32_t gv = 0;
        uint32_t lastV = 0;
        Pair<int> kvrow = {0, 0};
        Pair<int> nkept = {0, 0};
        bool ok = true;
        Walk<C::NBC> wk;
        wk.init();
        for (;;) {
          const int x = wk.pick();
          if (x < 0) break;
          if (wk.C.get(x) < 0) {
            const int tx = wk.t.get(x);
            const int slot = tx & 1;
            ok = ok && mbar_wait(bar(B_ITEM_FULL + 2 * x + slot), (tx >> 1) & 1, wc, 6);
            const ItemSlot it = sItem[2 * x + slot];
            const int n = ok ? it.n : -1;
            if (n <= 0) mbar_arrive(bar(B_ITEM_EMPTY + 2 * x + slot));
            if (n < 0) {
              wk.done.set(x, 1);
              continue;
            }
            kvrow.set(x, (int)(((size_t)it.b * a.Hkv + it.h / a.group) * a.N));
            nkept.set(x, n);
            wk.open(x, n);
            continue;
          }
          const int c = wk.c.get(x);
          const int slot = wk.t.get(x) & 1;
          const int nblk = min(C::NBC, nkept.get(x) - C::NBC * c);
          const uint32_t vs = gv % C::NSTG;
          // the stage's previous tile was read by the PV of step gv - NSTG
          if (gv >= (uint32_t)C::NSTG) ok = ok && mbar_wait(bar(B_V_EMPTY + vs), ((gv / C::NSTG) - 1) & 1, wc, 4);
          if (ok) {
            const int16_t* my_list = lists + (2 * x + slot) * kMaxBlocks;
            const int kvr = kvrow.get(x);
            mbar_expect_tx(bar(B_V_FULL + vs), nblk * BS * D * 2);
            const uint32_t dv = sbase + C::OffV + vs * C::KVBytes;
            for (int bb = 0; bb < nblk; ++bb) {
              const int row = kvr + my_list[C::NBC * c + bb] * BS;
#pragma unroll
              for (int hh = 0; hh < C::DH; ++hh)
                tma_load_2d(dv + hh * C::KVAtom + bb * BS * 128, &tmV, 64 * hh, row, bar(B_V_FULL + vs));
            }
            lastV = (lastV & ~(0x101u << vs)) | (1u << vs) | (((gv / C::NSTG) & 1u) << (8 + vs));
          }
          ++gv;
          if (c == wk.C.get(x) - 1) mbar_arrive(bar(B_ITEM_EMPTY + 2 * x + slot));
          wk.advance(x);
        }
        for (int u = 0; u < C::NSTG; ++u)
          if (lastV & (1u << u)) mbar_drain(bar(B_V_FULL + u), (lastV >> (8 + u)) & 1u, a.hdr, kKernAttnTc, 5);
      }
    } else if (warp == 1 || warp == 2) {
      // ---------------------------------------------------------------- MMA issuers
      const bool is_s = warp == 1;
      if (lane == 0) {
        Pair<uint32_t> gs = {0u, 0u};   // S^T uses per stream (buffer = gs & 1)
        Pair<uint32_t> gq = {0u, 0u};   // Q tiles per stream
        bool ok = true;
        // descriptor templates: k-steps only advance the 14-bit start-address field
        const uint64_t dK0 = smem_desc(sbase + C::OffK, 16, 1024);
        const uint64_t dQ0 = smem_desc(sbase + C::OffQ, 16, 1024);
        const uint64_t dV0 = smem_desc(sbase + C::OffV, C::KVAtom, 1024);
        const uint64_t dP0 = smem_desc(sbase + C::OffP, C::PBytes, 8 * C::PRow, C::PLayout);
        // Walk step n: its stream and item position come with its data, from the
        // K producer beside the K stage (S^T issuer) and from the softmax beside
        // the P tile (PV issuer).
        uint32_t n = 0;
        for (;; ++n) {
          if (is_s) {
            const uint32_t ks = n % C::NSTG;
            const int w = step_wait(bar(B_K_FULL + ks), (n / C::NSTG) & 1, sTotal, n, wc, 14);
            if (w <= 0) break;
            const uint32_t meta = sKMeta[ks];
            const int x = (int)(meta & 1u);
            const uint32_t gsx = gs.get(x);
            const uint32_t sb = gsx & 1;
            if (meta & 2u) ok = ok && mbar_wait(bar(B_Q_FULL + x), gq.inc(x) & 1, wc, 13);
            if (gsx >= 2) ok = ok && mbar_wait(bar(B_S_FREE + 2 * x + sb), ((gsx >> 1) - 1) & 1, wc, 15);
            tc_fence_after();
            if (ok) {
              const uint64_t dk = dK0 + (uint64_t)((ks * C::KVBytes) >> 4);
              const uint64_t dq = dQ0 + (uint64_t)((x * C::QBytes) >> 4);
              const uint32_t d = tmem + C::col_s(x, sb);
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk)
                tc_mma(d, dk + (uint64_t)(((kk >> 2) * C::KVAtom + (kk & 3) * 32) >> 4),
                       dq + (uint64_t)(((kk >> 2) * C::QAtom + (kk & 3) * 32) >> 4), C::IdescS,
                       kk > 0 ? 1u : 0u);
            }
            sStep[2 * x + sb] = n;
            tc_commit(bar(B_S_FULL + 2 * x + sb));
            tc_commit(bar(B_K_EMPTY + ks));           // K stage ks may be refilled
            mbar_arrive(bar(B_S_FULL + 2 * x + sb));  // releases the step id
            if (meta & 4u) tc_commit(bar(B_Q_EMPTY + x));
            gs.inc(x);
          } else {
            const uint32_t vs = n % C::NSTG;
            const uint32_t pt = n % C::PT, pu = n / C::PT;
            const int w = step_wait(bar(B_P_FULL + pt), pu & 1, sTotal, n, wc, 10);
            if (w <= 0) break;
            const uint32_t meta = sPMeta[pt];
            const int x = (int)(meta & 1u);
            ok = ok && mbar_wait(bar(B_V_FULL + vs), (n / C::NSTG) & 1, wc, 11);
            tc_fence_after();
            if (ok) {
              // only the chunk's kept blocks enter: the rest of the stage is stale
              const int ksteps = (int)(meta >> 3) * (BS / 16);
              const uint32_t acc0 = (meta & 2u) ? 0u : 1u;
              const uint64_t dv = dV0 + (uint64_t)((vs * C::KVBytes) >> 4);
              const uint64_t dp = dP0 + (uint64_t)((pt * C::PBytes) >> 4);
              const uint32_t d = tmem + C::col_o(x);
              // k-step kk: 16 keys, i.e. 16 rows of 128 B of V and 16 rows of P^T
              if (ksteps == kChunk / 16) {
#pragma unroll
                for (int kk = 0; kk < kChunk / 16; ++kk)
                  tc_mma(d, dv + (uint64_t)(kk * 128), dp + (uint64_t)(kk * C::PRow), C::IdescPV,
                         kk > 0 ? 1u : acc0);
              } else {
                for (int kk = 0; kk < ksteps; ++kk)
                  tc_mma(d, dv + (uint64_t)(kk * 128), dp + (uint64_t)(kk * C::PRow), C::IdescPV,
                         kk > 0 ? 1u : acc0);
              }
            }
            tc_commit(bar(B_P_EMPTY + pt));  // P tile pt may be rewritten
            tc_commit(bar(B_V_EMPTY + vs));  // V stage vs may be refilled
            if (meta & 4u) tc_commit(bar(B_O_DONE + x));
          }
        }
        const uint32_t gv = n;
        // the tensor core has finished every MMA before TMEM is released
        if (!is_s && gv > 0)
          mbar_drain(bar(B_P_EMPTY + (gv - 1) % C::PT), ((gv - 1) / C::PT) & 1, a.hdr, kKernAttnTc, 16);
        for (int x = 0; x < kStreams; ++x) {
          const uint32_t ns = gs.get(x);
          if (is_s && ns > 0)
            mbar_drain(bar(B_S_FULL + 2 * x + ((ns - 1) & 1)), ((ns - 1) >> 1) & 1, a.hdr, kKernAttnTc, 17);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    constexpr int NQ4 = BS / 4;
    const int x = (warp - 4) / 4;        // stream
    const int sp = warp & 3;             // TMEM sub-partition: lanes 32*sp ..
    const int r = sp * 32 + lane;        // key row of S^T
    // head-dim row of O^T this thread holds (M = 128: lane r; M = 64: lanes 0-15
    // of each sub-partition hold rows 16 sp .. 16 sp + 15), or -1
    const int orow = D == 128 ? r : (lane < 16 ? sp * 16 + lane : -1);
    const int bar_id = 1 + x;
    const uint32_t lane_addr = (uint32_t)(sp * 32) << 16;
    const float c2 = a.scale_log2;
    float* const sRed = reinterpret_cast<float*>(smem + C::OffRed) + x * 4 * BS;
    float* const sNM = reinterpret_cast<float*>(smem + C::OffM) + x * BS;  // -(running max)
    float* const sL = reinterpret_cast<float*>(smem + C::OffL) + x * BS;
    float* const sA = reinterpret_cast<float*>(smem + C::OffA) + x * BS;
    float2 l2[BS / 2];  // this thread's share of the row sums, queries 2j and 2j+1
    float tmin = INFINITY;  // smallest (m + kTau) / scale over the queries
    uint32_t gs = 0;
    uint32_t go = 0;      // items of this stream whose O^T has been completed
    uint32_t lastn = 0;   // walk step of this stream's previous tile
    // wait until the PV of walk step n has finished
    auto wait_step_pv = [&](uint32_t n) {
      mbar_wait<true>(bar(B_P_EMPTY + n % C::PT), (n / C::PT) & 1, wc, 20);
    };
    for (int t = 0;; ++t) {
      const int slot = t & 1;
      mbar_wait<true>(bar(B_ITEM_FULL + 2 * x + slot), (t >> 1) & 1, wc, 21);
      const ItemSlot it = sItem[2 * x + slot];
      // one decision for the whole warpgroup (also orders the slot reads before the release)
      const bool stop = wg_any(bar_id, it.n < 0 || *sAbort != 0);
      if (r == 0) mbar_arrive(bar(B_ITEM_EMPTY + 2 * x + slot));
      if (stop) break;
      const int Cn = (it.n + C::NBC - 1) / C::NBC;
#pragma unroll
      for (int q2 = 0; q2 < BS / 2; ++q2) l2[q2] = make_float2(0.f, 0.f);
      for (int c = 0; c < Cn; ++c) {
        const uint32_t sb = gs & 1;
        mbar_wait<true>(bar(B_S_FULL + 2 * x + sb), (gs >> 1) & 1, wc, 22);
        tc_fence_after();
        const uint32_t n_step = sStep[2 * x + sb];  // this tile's walk step
        const int nblk = min(C::NBC, it.n - C::NBC * c);
        const int blk = r / BS, kl = r % BS;
        const bool valid = blk < nblk;  // this lane holds a kept key of the tile
        const bool diag = (c == Cn - 1) && it.diag_last && (blk == nblk - 1);
        const uint32_t s_addr = tmem + lane_addr + C::col_s(x, sb);
        uint32_t raw[BS];
        tmem_ld(s_addr, raw);
        // Raise the running maxima when some visible logit exceeds them by more
        // than 2^kTau. Cheap sufficient test first: no S value of this lane
        // above the smallest per-query threshold (m + kTau) / scale.
        bool raise = c == 0;
        if (!raise) {
          float mx = -INFINITY;
          if (valid) {
            float t8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) t8[e] = __uint_as_float(raw[e]);
#pragma unroll
            for (int q = 8; q < BS; ++q) t8[q & 7] = fmaxf(t8[q & 7], __uint_as_float(raw[q]));
            mx = fmaxf(fmaxf(fmaxf(t8[0], t8[1]), fmaxf(t8[2], t8[3])),
                       fmaxf(fmaxf(t8[4], t8[5]), fmaxf(t8[6], t8[7])));
          }
          if (wg_any(bar_id, mx > tmin)) {
            // exact test, query by query
            bool part[8] = {false, false, false, false, false, false, false, false};
            if (valid) {
#pragma unroll
              for (int q4 = 0; q4 < NQ4; ++q4) {
                const float4 nm = reinterpret_cast<const float4*>(sNM)[q4];
                const float mm[4] = {nm.x, nm.y, nm.z, nm.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int q = 4 * q4 + e;
                  part[q & 7] |= (__fmaf_rn(__uint_as_float(raw[q]), c2, mm[e]) > kTau) && !(diag && kl > q);
                }
              }
            }
            const bool big = ((part[0] | part[1]) | (part[2] | part[3])) | ((part[4] | part[5]) | (part[6] | part[7]));
            raise = wg_any(bar_id, big);
          }
        }
        if (raise) {
          // column maxima of d = S * scale - m over this tile's visible keys
#pragma unroll
          for (int q4 = 0; q4 < NQ4; ++q4) {
            const float4 nm = c == 0 ? make_float4(0.f, 0.f, 0.f, 0.f) : reinterpret_cast<const float4*>(sNM)[q4];
            const float mm[4] = {nm.x, nm.y, nm.z, nm.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int q = 4 * q4 + e;
              const bool vis = valid && !(diag && kl > q);
              raw[q] = __float_as_uint(vis ? __fmaf_rn(__uint_as_float(raw[q]), c2, mm[e]) : -INFINITY);
            }
          }
          float* dv = reinterpret_cast<float*>(raw);
          const int col0 = warp_col_reduce<BS, true>(*reinterpret_cast<float(*)[BS]>(dv), lane);
#pragma unroll
          for (int e = 0; e < BS / 32; ++e) sRed[sp * BS + col0 + e] = dv[e];
          wg_sync(bar_id);
          if (r < BS) {
            const float mx = fmaxf(fmaxf(sRed[r], sRed[BS + r]), fmaxf(sRed[2 * BS + r], sRed[3 * BS + r]));
            const float inc = c == 0 ? mx : fmaxf(mx, 0.f);
            sA[r] = inc;
            sNM[r] = c == 0 ? -mx : sNM[r] - inc;
          }
          wg_sync(bar_id);
          // smallest raise threshold of the new maxima
          {
            float mn = INFINITY;
#pragma unroll
            for (int q4 = 0; q4 < NQ4; ++q4) {
              const float4 nm = reinterpret_cast<const float4*>(sNM)[q4];
              mn = fminf(mn, fminf(fminf(-nm.x, -nm.y), fminf(-nm.z, -nm.w)));
            }
            tmin = c2 > 0.f ? (mn + kTau) / c2 : INFINITY;
          }
          if (c > 0) {
            // O^T must hold every earlier tile's contribution before it is rescaled
            wait_step_pv(lastn);
            tc_fence_after();
            tmem_ld(tmem + lane_addr + C::col_o(x), raw);
#pragma unroll
            for (int q2 = 0; q2 < BS / 2; ++q2) {
              const float2 al = make_float2(ex2(-sA[2 * q2]), ex2(-sA[2 * q2 + 1]));
              l2[q2] = __fmul2_rn(l2[q2], al);
              const float2 o = __fmul2_rn(make_float2(__uint_as_float(raw[2 * q2]), __uint_as_float(raw[2 * q2 + 1])), al);
              raw[2 * q2] = __float_as_uint(o.x);
              raw[2 * q2 + 1] = __float_as_uint(o.y);
            }
            tmem_st(tmem + lane_addr + C::col_o(x), raw);
          }
          tmem_ld(s_addr, raw);  // the tile again, for the exponentials
        }
        tc_fence_before();
        mbar_arrive(bar(B_S_FREE + 2 * x + sb));  // the S^T buffer may be refilled
        ++gs;
        // P = 2^(S * scale - m) in bf16, row r of the MN-major P^T tile; the row
        // sums add the same bf16 values. The tile was last read by step n - PT.
        if (n_step >= (uint32_t)C::PT) wait_step_pv(n_step - C::PT);
        uint8_t* const prow = smem + C::OffP + (n_step % C::PT) * C::PBytes + r * C::PRow;
        // 16-byte chunk cc of this key row sits at chunk cc ^ (row bits of the swizzle)
        const int swz = BS == 64 ? (r & 7) : ((r >> 1) & 3);
        if (!valid) {
#pragma unroll
          for (int cc = 0; cc < BS / 8; ++cc)
            *reinterpret_cast<uint4*>(prow + ((cc ^ swz) << 4)) = make_uint4(0u, 0u, 0u, 0u);
        } else {
          const float2 c22 = make_float2(c2, c2);
          // The maxima of group cc + 1 are read before the P store of group cc:
          // a shared load that follows a shared store would wait for it.
          float4 n0 = reinterpret_cast<const float4*>(sNM)[0];
          float4 n1 = reinterpret_cast<const float4*>(sNM)[1];
#pragma unroll
          for (int cc = 0; cc < BS / 8; ++cc) {
            const float2 nm[4] = {make_float2(n0.x, n0.y), make_float2(n0.z, n0.w), make_float2(n1.x, n1.y),
                                  make_float2(n1.z, n1.w)};
            if (cc < BS / 8 - 1) {
              n0 = reinterpret_cast<const float4*>(sNM)[2 * cc + 2];
              n1 = reinterpret_cast<const float4*>(sNM)[2 * cc + 3];
            }
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int q = cc * 8 + 2 * e;
              const float2 d2 = __ffma2_rn(make_float2(__uint_as_float(raw[q]), __uint_as_float(raw[q + 1])), c22, nm[e]);
              float p0 = ex2(d2.x), p1 = ex2(d2.y);
              if (diag) {
                p0 = kl > q ? 0.f : p0;
                p1 = kl > q + 1 ? 0.f : p1;
              }
              w[e] = pack_bf16(p0, p1);
              l2[q >> 1].x = add_lo(l2[q >> 1].x, w[e]);
              l2[q >> 1].y = add_hi(l2[q >> 1].y, w[e]);
            }
            *reinterpret_cast<uint4*>(prow + ((cc ^ swz) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        if (r == 0) sPMeta[n_step % C::PT] = step_meta(x, c == 0, c == Cn - 1, nblk);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(bar(B_P_FULL + n_step % C::PT));
        lastn = n_step;
      }
      // ---------------------------------------------------------------- epilogue
      if (Cn > 0) {
        // the item's last PV has finished: O^T is complete
        mbar_wait<true>(bar(B_O_DONE + x), go & 1, wc, 23);
        ++go;
      }
      tc_fence_after();
      {
        float* lf = reinterpret_cast<float*>(l2);
        const int col0 = warp_col_reduce<BS, false>(*reinterpret_cast<float(*)[BS]>(lf), lane);
#pragma unroll
        for (int e = 0; e < BS / 32; ++e) sRed[sp * BS + col0 + e] = lf[e];
      }
      wg_sync(bar_id);
      float lsum = 0.f;
      if (r < BS) {
        lsum = (sRed[r] + sRed[BS + r]) + (sRed[2 * BS + r] + sRed[3 * BS + r]);
        sL[r] = lsum > 0.f ? 1.0f / lsum : 0.f;
      }
      wg_sync(bar_id);
      const size_t row0 = ((size_t)it.b * a.Hq + it.h) * a.N + (size_t)it.i * BS;
      {
        uint32_t o[BS];
        if (Cn > 0) {
          tmem_ld(tmem + lane_addr + C::col_o(x), o);
        } else {
#pragma unroll
          for (int q = 0; q < BS; ++q) o[q] = 0u;
        }
        tc_fence_before();
        // this thread holds head-dim element orow of the bs output rows: each
        // warp store covers consecutive head-dim elements of one row
        if (orow >= 0) {
          __nv_bfloat16* const dst = a.out + row0 * D + orow;
#pragma unroll
          for (int q = 0; q < BS; ++q) dst[(size_t)q * D] = __float2bfloat16_rn(__uint_as_float(o[q]) * sL[q]);
        }
      }
      if (a.lse != nullptr && r < BS)
        a.lse[row0 + r] = (Cn > 0 && lsum > 0.f) ? (-sNM[r] * kLn2 + logf(lsum)) : -INFINITY;
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

template <int BS, int D>
cudaError_t launch_shape(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                         const __nv_bfloat16* v, const int32_t* idx, const int32_t* cnt,
                         __nv_bfloat16* out, float* lse, WsHeader* hdr, cudaStream_t st) {
  using C = Cfg<BS, D>;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, (unsigned long long)s.B * s.Hq * s.N, D, BS) ||
      !make_map(&mk, k, (unsigned long long)s.B * s.Hkv * s.N, D, BS) ||
      !make_map(&mv, v, (unsigned long long)s.B * s.Hkv * s.N, D, BS))
    return cudaErrorInvalidValue;
  TcArgs a;
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
  e = cudaFuncSetAttribute(attn_tc_kernel<BS, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(&hdr->work[0], 0, sizeof(unsigned int), st);
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < sms ? a.n_items : sms;
  attn_tc_kernel<BS, D><<<grid, kThreads, C::SmemBytes, st>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(const Shape& s) {
  // TMA row coordinates are 32-bit
  const unsigned long long rows = (unsigned long long)s.B * s.Hq * s.N;
  if (rows >= (1ull << 31) || encode_fn() == nullptr) return false;
  return (s.bs == 32 || s.bs == 64 || s.bs == 128) && (s.d == 64 || s.d == 128);
}

cudaError_t launch_attn_tc(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, const int32_t* idx, const int32_t* cnt,
                           __nv_bfloat16* out, float* lse, WsHeader* hdr, cudaStream_t st) {
  if (!attn_tc_supported(s)) return cudaErrorNotSupported;
  if (s.bs == 128) return launch_attn_tc128(s, q, k, v, idx, cnt, out, lse, hdr, st);
  if (s.bs == 64 && s.d == 128) return launch_shape<64, 128>(s, q, k, v, idx, cnt, out, lse, hdr, st);
  if (s.bs == 64 && s.d == 64) return launch_shape<64, 64>(s, q, k, v, idx, cnt, out, lse, hdr, st);
  if (s.bs == 32 && s.d == 128) return launch_shape<32, 128>(s, q, k, v, idx, cnt, out, lse, hdr, st);
  return launch_shape<32, 64>(s, q, k, v, idx, cnt, out, lse, hdr, st);
}

}  // namespace dsa
