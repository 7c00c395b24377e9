// Block-sparse causal attention forward (step 4) on the 5th-generation tensor
// cores (tcgen05 + TMEM + TMA), for 64x64 blocks and head dim 128.
//
// What it computes is the same as the warp-MMA kernel: for every query block
// i of (b, query head h), softmax(Q K^T * scale) V over the kept key blocks
// only, causal inside the diagonal block, with K/V of KV head h / (Hq/Hkv)
// ("稀疏注意力 vs Flash Attention v2", section 1; FlashAttention-style online
// softmax; "DeepSeek NSA", section 2.2, bf16 matmul with fp32 accumulation).
//
// Shape of the computation on sm_100a. A query block has only 64 rows, and
// every (head, query block) keeps its own list of key blocks, so stacking
// two query blocks into one 128-row MMA would multiply masked work. Instead
// the kernel computes transposed products whose 128-row side is the keys of
// two kept blocks:
//     S^T (128 keys x 64 queries) = K_pair (128 x d) . Q^T        (M=128, N=64)
//     O^T (d=128 x 64 queries)   += V_pair^T (128 x 128 keys) . P^T (M=128, N=64)
// so every tcgen05.mma runs at M=128 without any wasted rows (at N=64 an MMA
// reads 6 KB of shared memory per 128x64x16 step, which bounds the tensor
// pipe at 2/3 of its N>=128 rate). In TMEM a thread of a softmax warpgroup
// owns one key (lane) of S^T and one head-dim row of O^T. The softmax maximum
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
#include <cuda.h>

#include "dsa_internal.cuh"

namespace dsa {
namespace {

constexpr int kBS = 64;        // query / key block
constexpr int kD = 128;        // head dim
constexpr int kChunk = 128;    // keys per S^T tile (two blocks)
constexpr int kThreads = 384;
constexpr int kStreams = 2;
constexpr float kTau = 8.0f;   // rescale threshold (log2 units)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

// Shared memory map (bytes from a 1024-byte aligned base).
constexpr int kQBytes = kBS * kD * 2;         // 16 KB: [2 d-halves][64 rows][128 B]
constexpr int kKVBytes = kChunk * kD * 2;     // 32 KB: [2 d-halves][128 rows][128 B]
constexpr int kPBytes = kChunk * kBS * 2;     // 16 KB: [128 keys][64 queries] bf16
constexpr int kOffQ = 0;                                  // one per stream
constexpr int kOffK = kOffQ + kStreams * kQBytes;         // 2 ring stages
constexpr int kOffV = kOffK + 2 * kKVBytes;               // 2 ring stages
constexpr int kPTiles = 3;                                // P tiles shared by the streams
constexpr int kOffP = kOffV + 2 * kKVBytes;               // [kPTiles]
constexpr int kOffList = kOffP + kPTiles * kPBytes;       // [stream][slot][kMaxBlocks] int16
constexpr int kOffRed = kOffList + kStreams * 2 * kMaxBlocks * 2;  // [stream][4][64] f32
constexpr int kOffM = kOffRed + kStreams * 4 * 64 * 4;    // [stream][64] -(running max)
constexpr int kOffL = kOffM + kStreams * 64 * 4;          // [stream][64] 1 / row sum
constexpr int kOffA = kOffL + kStreams * 64 * 4;          // [stream][64] max increments
constexpr int kOffBar = kOffA + kStreams * 64 * 4;        // mbarriers
constexpr int kNumBars = 36;
constexpr int kOffMisc = kOffBar + kNumBars * 8;          // tmem base, abort flag, item slots, step ids
constexpr int kSmemBytes = kOffMisc + 160 + 1024;         // + alignment slack
static_assert(kSmemBytes <= 232448, "shared memory budget");

// barrier indices ([stream] or [stream][slot|buffer] or [stage])
enum {
  B_ITEM_FULL = 0,    // [2][2]
  B_ITEM_EMPTY = 4,   // [2][2]
  B_Q_FULL = 8,       // [2]
  B_Q_EMPTY = 10,     // [2]
  B_K_FULL = 12,      // [2]
  B_K_EMPTY = 14,     // [2] spare: a K stage is free once its S^T has completed (S_FULL)
  B_V_FULL = 16,      // [2]
  B_V_EMPTY = 18,     // [2] spare: a V stage is free once its PV has completed (P_EMPTY)
  B_S_FULL = 20,      // [2][2]
  B_S_FREE = 24,      // [2][2]
  B_P_FULL = 28,      // [kPTiles]
  B_P_EMPTY = 31,     // [kPTiles]
  B_O_DONE = 34       // [2]: the last PV of a stream's item has finished
};

// P tiles: step n of the (stream, chunk) walk writes tile n % kPTiles, whose
// previous reader was step n - kPTiles; the S^T issuer publishes each step's
// index next to its S^T buffer (sStep[stream][buffer]).

// TMEM columns per stream: two S^T buffers and the O^T accumulator.
constexpr uint32_t kTmemCols = 512;
__device__ __forceinline__ uint32_t col_s(int stream, uint32_t buf) { return stream * 192 + buf * 64; }
__device__ __forceinline__ uint32_t col_o(int stream) { return stream * 192 + 128; }

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

// ----------------------------------------------------------------------------
// PTX helpers
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait. Returns false (and raises the CTA abort flag and the device
// error) when the phase does not complete within the limit, or at once when
// the CTA is already aborting. The first probe is inlined; the spin loop is
// out of line so that callers keep their registers on the fast path.
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                            WsHeader* hdr, int where) {
  const unsigned long long t0 = now_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*abort_flag) return false;
      if (now_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        raise_error(hdr, DSA_ERR_DEVICE_TIMEOUT, kKernAttnTc, where, (int)blockIdx.x);
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          WsHeader* hdr, int where) {
  if (mbar_try(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, abort_flag, hdr, where);
}

// Step metadata word: stream, first and last chunk of the item, kept blocks in the chunk.
__device__ __forceinline__ uint32_t step_meta(int x, bool first, bool last, int nblk) {
  return (uint32_t)x | (first ? 2u : 0u) | (last ? 4u : 0u) | ((uint32_t)nblk << 3);
}

// Waits for a barrier phase that belongs to walk step n. Returns 1 when the
// phase completed, 0 when the walk has fewer than n + 1 steps (the step and
// its phase never come), -1 when the kernel is aborting or the wait timed out.
__device__ __noinline__ int step_wait_slow(uint32_t bar, uint32_t parity, volatile uint32_t* total,
                                           uint32_t n, volatile int* abort_flag, WsHeader* hdr,
                                           int where) {
  const unsigned long long t0 = now_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return 1;
    if (*total <= n) return 0;
    if ((it & 63u) == 0u) {
      if (*abort_flag) return -1;
      if (now_ns() - t0 > kWaitLimitNs) {
        *abort_flag = 1;
        raise_error(hdr, DSA_ERR_DEVICE_TIMEOUT, kKernAttnTc, where, (int)blockIdx.x);
        return -1;
      }
    }
  }
}

__device__ __forceinline__ int step_wait(uint32_t bar, uint32_t parity, volatile uint32_t* total,
                                         uint32_t n, volatile int* abort_flag, WsHeader* hdr,
                                         int where) {
  if (mbar_try(bar, parity)) return 1;
  return step_wait_slow(bar, parity, total, n, abort_flag, hdr, where);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 64 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]),
        "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]),
        "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
        "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]),
        "=r"(r[63])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,"
      "%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,"
      "%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]),
      "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]),
      "r"(r[30]), "r"(r[31]), "r"(r[32]), "r"(r[33]), "r"(r[34]), "r"(r[35]), "r"(r[36]),
      "r"(r[37]), "r"(r[38]), "r"(r[39]), "r"(r[40]), "r"(r[41]), "r"(r[42]), "r"(r[43]),
      "r"(r[44]), "r"(r[45]), "r"(r[46]), "r"(r[47]), "r"(r[48]), "r"(r[49]), "r"(r[50]),
      "r"(r[51]), "r"(r[52]), "r"(r[53]), "r"(r[54]), "r"(r[55]), "r"(r[56]), "r"(r[57]),
      "r"(r[58]), "r"(r[59]), "r"(r[60]), "r"(r[61]), "r"(r[62]), "r"(r[63])
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// c + (low / high bf16 half of w), one mixed-precision add (fp32 result, round to nearest)
__device__ __forceinline__ float add_lo(float c, uint32_t w) {
  float d;
  asm("{ .reg .b16 lo, hi; mov.b32 {lo, hi}, %1; add.rn.f32.bf16 %0, lo, %2; }" : "=f"(d) : "r"(w), "f"(c));
  return d;
}
__device__ __forceinline__ float add_hi(float c, uint32_t w) {
  float d;
  asm("{ .reg .b16 lo, hi; mov.b32 {lo, hi}, %1; add.rn.f32.bf16 %0, hi, %2; }" : "=f"(d) : "r"(w), "f"(c));
  return d;
}

// Named barrier over the 128 threads of one softmax warpgroup (id 1 + stream),
// optionally OR-reducing a predicate.
__device__ __forceinline__ void softmax_sync(int id) {
  asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
}
__device__ __forceinline__ bool softmax_any(int id, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %2, 0;\n\t"
      "bar.red.or.pred q, %1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(id), "r"((uint32_t)pred)
      : "memory");
  return r != 0;
}

// Shared-memory matrix descriptor (sm_100 format, 128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor: bf16 x bf16 -> fp32, M=128, N=64.
constexpr uint32_t idesc_mn(uint32_t a_mn_major, uint32_t b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn_major << 15) | (b_mn_major << 16) |
         ((uint32_t)(kBS >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
constexpr uint32_t kIdescS = idesc_mn(0, 0);   // A = K (K-major), B = Q (K-major)
constexpr uint32_t kIdescPV = idesc_mn(1, 1);  // A = V^T (MN-major), B = P^T (MN-major)

// Column-wise reductions over the 32 lanes of a warp for 64 columns held one
// per register: after the call, v[0] and v[1] hold the reduced values of
// columns col0 and col0+1, col0 = 2 * (bit-reversed pattern of the lane).
template <bool kMax>
__device__ __forceinline__ int warp_col_reduce(float (&v)[64], int lane) {
#define DSA_RED(OFF, HALF)                                                     \
  {                                                                            \
    const bool up = (lane & OFF) != 0;                                         \
    _Pragma("unroll") for (int j = 0; j < HALF; ++j) {                         \
      const float send = up ? v[j] : v[j + HALF];                              \
      const float keep = up ? v[j + HALF] : v[j];                              \
      const float got = __shfl_xor_sync(0xffffffffu, send, OFF);               \
      v[j] = kMax ? fmaxf(keep, got) : (keep + got);                           \
    }                                                                          \
  }
  DSA_RED(16, 32)
  DSA_RED(8, 16)
  DSA_RED(4, 8)
  DSA_RED(2, 4)
  DSA_RED(1, 2)
#undef DSA_RED
  return ((lane >> 4) & 1) * 32 + ((lane >> 3) & 1) * 16 + ((lane >> 2) & 1) * 8 +
         ((lane >> 1) & 1) * 4 + (lane & 1) * 2;
}

__device__ __forceinline__ void decode_item(const TcArgs& a, int item, int& b, int& h, int& i) {
  // KV-head-major; inside a KV head, query blocks from the last (longest) down;
  // the group's query heads interleaved.
  const int per_kv = a.group * a.nb;
  const int bk = item / per_kv;
  const int rem = item - bk * per_kv;
  b = bk / a.Hkv;
  const int kvh = bk - b * a.Hkv;
  i = a.nb - 1 - rem / a.group;
  h = kvh * a.group + rem % a.group;
}

// Two per-stream values kept in registers (a runtime-indexed array would live
// in local memory).
template <class T>
struct Pair {
  T v0, v1;
  __device__ __forceinline__ T get(int x) const { return x ? v1 : v0; }
  __device__ __forceinline__ void set(int x, T v) {
    if (x) v1 = v;
    else v0 = v;
  }
  __device__ __forceinline__ T inc(int x) {  // post-increment
    const T old = get(x);
    set(x, old + 1);
    return old;
  }
};

// The (stream, chunk) walk shared by the producer and both MMA issuers.
// Streams alternate one chunk at a time; a stream whose item has no chunks
// moves on to its next item without taking a step; once one stream runs out
// of items the other takes every remaining step.
struct Walk {
  Pair<int> t;     // item counter of the stream (slot = t & 1)
  Pair<int> c;     // next chunk of the current item
  Pair<int> C;     // chunks of the current item; -1: no item open
  Pair<int> done;
  int turn;
  __device__ __forceinline__ void init() {
    t = {0, 0};
    c = {0, 0};
    C = {-1, -1};
    done = {0, 0};
    turn = 0;
  }
  // Chooses the stream of the next step; -1 when both are finished.
  __device__ __forceinline__ int pick() const {
    int x = turn;
    if (done.get(x)) x ^= 1;
    return done.get(x) ? -1 : x;
  }
  // Opens an item of n kept blocks on stream x (n = 0: closed at once).
  __device__ __forceinline__ void open(int x, int n) {
    const int chunks = (n + 1) >> 1;
    c.set(x, 0);
    if (chunks == 0) {
      C.set(x, -1);
      t.inc(x);
    } else {
      C.set(x, chunks);
    }
  }
  // After a step of stream x: advance, and close the item after its last chunk.
  __device__ __forceinline__ void advance(int x) {
    turn = x ^ 1;
    const int nc = c.get(x) + 1;
    if (nc == C.get(x)) {
      c.set(x, 0);
      C.set(x, -1);
      t.inc(x);
    } else {
      c.set(x, nc);
    }
  }
};

__global__ void __launch_bounds__(kThreads, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bars = sbase + kOffBar;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* sAbort = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  ItemSlot* sItem = reinterpret_cast<ItemSlot*>(smem + kOffMisc + 16);  // [stream][slot]
  volatile uint32_t* sStep = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc + 112);  // [stream][S buffer]
  // step count of the whole walk, published by the K producer when it ends
  volatile uint32_t* sTotal = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc + 8);
  // per K stage and per P tile: stream and position of the step they hold
  volatile uint32_t* sKMeta = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc + 128);  // [2]
  volatile uint32_t* sPMeta = reinterpret_cast<volatile uint32_t*>(smem + kOffMisc + 136);  // [kPTiles]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  auto bar = [&](int idx) { return bars + 8u * idx; };

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
      mbar_init(bar(B_K_FULL + x), 1);
      mbar_init(bar(B_K_EMPTY + x), 1);
      mbar_init(bar(B_V_FULL + x), 1);
      mbar_init(bar(B_V_EMPTY + x), 1);
    }
    for (int t = 0; t < kPTiles; ++t) {
      mbar_init(bar(B_P_FULL + t), 128);
      mbar_init(bar(B_P_EMPTY + t), 1);
    }
    *sAbort = 0;
    *sTotal = 0xffffffffu;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(sTmem)),
                 "r"(kTmemCols)
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
      int16_t* const lists = reinterpret_cast<int16_t*>(smem + kOffList);
      uint32_t gk = 0;
      Pair<uint32_t> gq = {0u, 0u};
      Pair<uint32_t> gs = {0u, 0u};  // S^T uses per stream, as counted by the S issuer
      // per K stage u: bit 8u: loaded once; bits 8u+1..: s_full barrier index and
      // parity of the S^T step that read it (the stage is free once that completes)
      uint32_t kuse = 0;
      // bit u set: ring stage u has an issued load; bit 2+u: its phase parity
      uint32_t lastK = 0, lastQ = 0;
      Pair<int> kvrow = {0, 0};
      Pair<int> nkept = {0, 0};
      bool ok = true;
      Walk wk;
      wk.init();
      for (;;) {
        const int x = wk.pick();
        if (x < 0) break;
        if (wk.C.get(x) < 0) {
          // open the stream's next item: fetch it, compact its list, publish it
          const int tx = wk.t.get(x);
          const int slot = tx & 1;
          if (lane == 0 && tx >= 2)
            ok = ok && mbar_wait(bar(B_ITEM_EMPTY + 2 * x + slot), ((tx >> 1) - 1) & 1, sAbort, a.hdr, 1);
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
          decode_item(a, item, b, h, i);
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
            const bool valid = in && j >= 0 && j <= i;
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
              if (gqx >= 1) ok = ok && mbar_wait(bar(B_Q_EMPTY + x), (gqx - 1) & 1, sAbort, a.hdr, 2);
              if (ok) {
                const int qrow = (int)(((size_t)b * a.Hq + h) * a.N + (size_t)i * kBS);
                mbar_expect_tx(bar(B_Q_FULL + x), kQBytes);
                const uint32_t dq = sbase + kOffQ + x * kQBytes;
                tma_load_2d(dq, &tmQ, 0, qrow, bar(B_Q_FULL + x));
                tma_load_2d(dq + kQBytes / 2, &tmQ, 64, qrow, bar(B_Q_FULL + x));
                lastQ = (lastQ & ~(5u << x)) | (1u << x) | ((gqx & 1u) << (2 + x));
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
          const int nblk = min(2, nkept.get(x) - 2 * c);
          const int kvr = kvrow.get(x);
          const int16_t* my_list = lists + (2 * x + (wk.t.get(x) & 1)) * kMaxBlocks;
          const uint32_t ks = gk & 1;
          const uint32_t prev = (kuse >> (8 * ks)) & 0xffu;
          if (prev & 1u) ok = ok && mbar_wait(bar(B_S_FULL + (prev >> 2)), (prev >> 1) & 1u, sAbort, a.hdr, 3);
          if (ok) {
            sKMeta[ks] = step_meta(x, c == 0, c == wk.C.get(x) - 1, nblk);
            mbar_expect_tx(bar(B_K_FULL + ks), nblk * (kKVBytes / 2));
            const uint32_t dk = sbase + kOffK + ks * kKVBytes;
            for (int bb = 0; bb < nblk; ++bb) {
              const int row = kvr + my_list[2 * c + bb] * kBS;
              tma_load_2d(dk + bb * (kKVBytes / 4), &tmK, 0, row, bar(B_K_FULL + ks));
              tma_load_2d(dk + kKVBytes / 2 + bb * (kKVBytes / 4), &tmK, 64, row, bar(B_K_FULL + ks));
            }
            lastK = (lastK & ~(5u << ks)) | (1u << ks) | (((gk >> 1) & 1u) << (2 + ks));
          }
          // the S^T step of this K tile writes buffer gs & 1 of stream x
          const uint32_t gsx = gs.get(x);
          const uint32_t use = 1u | (((gsx >> 1) & 1u) << 1) | ((uint32_t)(2 * x + (gsx & 1)) << 2);
          kuse = (kuse & ~(0xffu << (8 * ks))) | (use << (8 * ks));
        }
        gs.inc(x);
        ++gk;
        ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
        wk.advance(x);
      }
      if (lane == 0) *sTotal = gk;
      // drain: every issued load has landed before the CTA may exit
      if (lane == 0) {
        volatile int no_abort = 0;
        for (int u = 0; u < 2; ++u) {
          if (lastK & (1u << u)) mbar_wait(bar(B_K_FULL + u), (lastK >> (2 + u)) & 1u, &no_abort, a.hdr, 5);
          if (lastQ & (1u << u)) mbar_wait(bar(B_Q_FULL + u), (lastQ >> (2 + u)) & 1u, &no_abort, a.hdr, 5);
        }
      }
    } else if (warp == 3) {
      // ---------------------------------------------------------------- V producer
      // Walks the same steps; reads each item's kept list from its slot and
      // releases the slot after the item's last V tile has been issued.
      const int16_t* const lists = reinterpret_cast<const int16_t*>(smem + kOffList);
      if (lane == 0) {
        uint32_t gv = 0;
        uint32_t lastV = 0;
        Pair<int> kvrow = {0, 0};
        Pair<int> nkept = {0, 0};
        bool ok = true;
        Walk wk;
        wk.init();
        for (;;) {
          const int x = wk.pick();
          if (x < 0) break;
          if (wk.C.get(x) < 0) {
            const int tx = wk.t.get(x);
            const int slot = tx & 1;
            ok = ok && mbar_wait(bar(B_ITEM_FULL + 2 * x + slot), (tx >> 1) & 1, sAbort, a.hdr, 6);
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
          const int nblk = min(2, nkept.get(x) - 2 * c);
          const uint32_t vs = gv & 1;
          // the stage's previous tile belongs to step gv - 2, whose PV also freed its P tile
          if (gv >= 2)
            ok = ok && mbar_wait(bar(B_P_EMPTY + (gv - 2) % kPTiles), ((gv - 2) / kPTiles) & 1, sAbort, a.hdr, 4);
          if (ok) {
            const int16_t* my_list = lists + (2 * x + slot) * kMaxBlocks;
            const int kvr = kvrow.get(x);
            mbar_expect_tx(bar(B_V_FULL + vs), nblk * (kKVBytes / 2));
            const uint32_t dv = sbase + kOffV + vs * kKVBytes;
            for (int bb = 0; bb < nblk; ++bb) {
              const int row = kvr + my_list[2 * c + bb] * kBS;
              tma_load_2d(dv + bb * (kKVBytes / 4), &tmV, 0, row, bar(B_V_FULL + vs));
              tma_load_2d(dv + kKVBytes / 2 + bb * (kKVBytes / 4), &tmV, 64, row, bar(B_V_FULL + vs));
            }
            lastV = (lastV & ~(5u << vs)) | (1u << vs) | (((gv >> 1) & 1u) << (2 + vs));
          }
          ++gv;
          if (c == wk.C.get(x) - 1) mbar_arrive(bar(B_ITEM_EMPTY + 2 * x + slot));
          wk.advance(x);
        }
        volatile int no_abort = 0;
        for (int u = 0; u < 2; ++u)
          if (lastV & (1u << u)) mbar_wait(bar(B_V_FULL + u), (lastV >> (2 + u)) & 1u, &no_abort, a.hdr, 5);
      }
    } else if (warp == 1 || warp == 2) {
      // ---------------------------------------------------------------- MMA issuers
      const bool is_s = warp == 1;
      if (lane == 0) {
        Pair<uint32_t> gs = {0u, 0u};   // S^T uses per stream (buffer = gs & 1)
        Pair<uint32_t> gq = {0u, 0u};   // Q tiles per stream
        bool ok = true;
        // descriptor templates: k-steps only advance the 14-bit start-address field
        const uint64_t dK0 = smem_desc(sbase + kOffK, 16, 1024);
        const uint64_t dQ0 = smem_desc(sbase + kOffQ, 16, 1024);
        const uint64_t dV0 = smem_desc(sbase + kOffV, kKVBytes / 2, 1024);
        const uint64_t dP0 = smem_desc(sbase + kOffP, kPBytes, 1024);
        // Walk step n: its stream and item position come with its data, from the
        // K producer beside the K stage (S^T issuer) and from the softmax beside
        // the P tile (PV issuer).
        uint32_t n = 0;
        for (;; ++n) {
          if (is_s) {
            const uint32_t ks = n & 1;
            const int w = step_wait(bar(B_K_FULL + ks), (n >> 1) & 1, sTotal, n, sAbort, a.hdr, 14);
            if (w <= 0) break;
            const uint32_t meta = sKMeta[ks];
            const int x = (int)(meta & 1u);
            const uint32_t gsx = gs.get(x);
            const uint32_t sb = gsx & 1;
            if (meta & 2u) ok = ok && mbar_wait(bar(B_Q_FULL + x), gq.inc(x) & 1, sAbort, a.hdr, 13);
            if (gsx >= 2)
              ok = ok && mbar_wait(bar(B_S_FREE + 2 * x + sb), ((gsx >> 1) - 1) & 1, sAbort, a.hdr, 15);
            tc_fence_after();
            if (ok) {
              const uint64_t dk = dK0 + (uint64_t)((ks * kKVBytes) >> 4);
              const uint64_t dq = dQ0 + (uint64_t)((x * kQBytes) >> 4);
              const uint32_t d = tmem + col_s(x, sb);
#pragma unroll
              for (int kk = 0; kk < kD / 16; ++kk)
                tc_mma(d, dk + (uint64_t)(((kk >> 2) * (kKVBytes / 2) + (kk & 3) * 32) >> 4),
                       dq + (uint64_t)(((kk >> 2) * (kQBytes / 2) + (kk & 3) * 32) >> 4), kIdescS,
                       kk > 0 ? 1u : 0u);
            }
            sStep[2 * x + sb] = n;
            tc_commit(bar(B_S_FULL + 2 * x + sb));  // also frees K stage ks
            mbar_arrive(bar(B_S_FULL + 2 * x + sb));  // releases the step id
            if (meta & 4u) tc_commit(bar(B_Q_EMPTY + x));
            gs.inc(x);
          } else {
            const uint32_t vs = n & 1;
            const uint32_t pt = n % kPTiles, pu = n / kPTiles;
            const int w = step_wait(bar(B_P_FULL + pt), pu & 1, sTotal, n, sAbort, a.hdr, 10);
            if (w <= 0) break;
            const uint32_t meta = sPMeta[pt];
            const int x = (int)(meta & 1u);
            ok = ok && mbar_wait(bar(B_V_FULL + vs), (n >> 1) & 1, sAbort, a.hdr, 11);
            tc_fence_after();
            if (ok) {
              const int ksteps = (int)(meta >> 3) * (kBS / 16);
              const uint32_t acc0 = (meta & 2u) ? 0u : 1u;
              const uint64_t dv = dV0 + (uint64_t)((vs * kKVBytes) >> 4);
              const uint64_t dp = dP0 + (uint64_t)((pt * kPBytes) >> 4);
              const uint32_t d = tmem + col_o(x);
              if (ksteps == 2 * (kBS / 16)) {
#pragma unroll
                for (int kk = 0; kk < 2 * (kBS / 16); ++kk)
                  tc_mma(d, dv + (uint64_t)(kk * 128), dp + (uint64_t)(kk * 128), kIdescPV,
                         kk > 0 ? 1u : acc0);
              } else {
#pragma unroll
                for (int kk = 0; kk < kBS / 16; ++kk)
                  tc_mma(d, dv + (uint64_t)(kk * 128), dp + (uint64_t)(kk * 128), kIdescPV,
                         kk > 0 ? 1u : acc0);
              }
            }
            tc_commit(bar(B_P_EMPTY + pt));  // frees P tile pt and V stage vs
            if (meta & 4u) tc_commit(bar(B_O_DONE + x));
          }
        }
        const uint32_t gv = n;
        // the tensor core has finished every MMA before TMEM is released
        volatile int no_abort = 0;
        if (!is_s && gv > 0)
          mbar_wait(bar(B_P_EMPTY + (gv - 1) % kPTiles), ((gv - 1) / kPTiles) & 1, &no_abort, a.hdr, 16);
        for (int x = 0; x < kStreams; ++x) {
          const uint32_t ns = gs.get(x);
          if (is_s && ns > 0)
            mbar_wait(bar(B_S_FULL + 2 * x + ((ns - 1) & 1)), ((ns - 1) >> 1) & 1, &no_abort, a.hdr, 17);
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax + epilogue
    const int x = (warp - 4) / 4;        // stream
    const int sp = warp & 3;             // TMEM sub-partition: lanes 32*sp ..
    const int r = sp * 32 + lane;        // key row of S^T / head-dim row of O^T
    const int bar_id = 1 + x;
    const uint32_t lane_addr = (uint32_t)(sp * 32) << 16;
    const float c2 = a.scale_log2;
    float* const sRed = reinterpret_cast<float*>(smem + kOffRed) + x * 256;
    float* const sNM = reinterpret_cast<float*>(smem + kOffM) + x * 64;  // -(running max)
    float* const sL = reinterpret_cast<float*>(smem + kOffL) + x * 64;
    float* const sA = reinterpret_cast<float*>(smem + kOffA) + x * 64;
    float2 l2[32];  // this thread's share of the row sums, queries 2j and 2j+1
    float tmin = INFINITY;  // smallest (m + kTau) / scale over the queries
    uint32_t gs = 0;
    uint32_t go = 0;      // items of this stream whose O^T has been completed
    uint32_t lastn = 0;   // walk step of this stream's previous tile
    // wait until the PV of walk step n has finished
    auto wait_step_pv = [&](uint32_t n) {
      mbar_wait(bar(B_P_EMPTY + n % kPTiles), (n / kPTiles) & 1, sAbort, a.hdr, 20);
    };
    for (int t = 0;; ++t) {
      const int slot = t & 1;
      mbar_wait(bar(B_ITEM_FULL + 2 * x + slot), (t >> 1) & 1, sAbort, a.hdr, 21);
      const ItemSlot it = sItem[2 * x + slot];
      // one decision for the whole warpgroup (also orders the slot reads before the release)
      const bool stop = softmax_any(bar_id, it.n < 0 || *sAbort != 0);
      if (r == 0) mbar_arrive(bar(B_ITEM_EMPTY + 2 * x + slot));
      if (stop) break;
      const int C = (it.n + 1) >> 1;
#pragma unroll
      for (int q2 = 0; q2 < 32; ++q2) l2[q2] = make_float2(0.f, 0.f);
      for (int c = 0; c < C; ++c) {
        const uint32_t sb = gs & 1;
        mbar_wait(bar(B_S_FULL + 2 * x + sb), (gs >> 1) & 1, sAbort, a.hdr, 22);
        tc_fence_after();
        const uint32_t n_step = sStep[2 * x + sb];  // this tile's walk step
        const int nblk = min(2, it.n - 2 * c);
        const int blk = r / kBS, kl = r % kBS;
        const bool valid = blk < nblk;  // this lane holds a kept key of the tile
        const bool diag = (c == C - 1) && it.diag_last && (blk == nblk - 1);
        const uint32_t s_addr = tmem + lane_addr + col_s(x, sb);
        uint32_t raw[64];
        tmem_ld64(s_addr, raw);
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
            for (int q = 8; q < 64; ++q) t8[q & 7] = fmaxf(t8[q & 7], __uint_as_float(raw[q]));
            mx = fmaxf(fmaxf(fmaxf(t8[0], t8[1]), fmaxf(t8[2], t8[3])),
                       fmaxf(fmaxf(t8[4], t8[5]), fmaxf(t8[6], t8[7])));
          }
          if (softmax_any(bar_id, mx > tmin)) {
            // exact test, query by query
            bool part[8] = {false, false, false, false, false, false, false, false};
            if (valid) {
#pragma unroll
              for (int q4 = 0; q4 < 16; ++q4) {
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
            raise = softmax_any(bar_id, big);
          }
        }
        if (raise) {
          // column maxima of d = S * scale - m over this tile's visible keys
#pragma unroll
          for (int q4 = 0; q4 < 16; ++q4) {
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
          const int col0 = warp_col_reduce<true>(*reinterpret_cast<float(*)[64]>(dv), lane);
          sRed[sp * 64 + col0] = dv[0];
          sRed[sp * 64 + col0 + 1] = dv[1];
          softmax_sync(bar_id);
          if (r < 64) {
            const float mx = fmaxf(fmaxf(sRed[r], sRed[64 + r]), fmaxf(sRed[128 + r], sRed[192 + r]));
            const float inc = c == 0 ? mx : fmaxf(mx, 0.f);
            sA[r] = inc;
            sNM[r] = c == 0 ? -mx : sNM[r] - inc;
          }
          softmax_sync(bar_id);
          // smallest raise threshold of the new maxima
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
            // O^T must hold every earlier tile's contribution before it is rescaled
            wait_step_pv(lastn);
            tc_fence_after();
            tmem_ld64(tmem + lane_addr + col_o(x), raw);
#pragma unroll
            for (int q2 = 0; q2 < 32; ++q2) {
              const float2 al = make_float2(ex2(-sA[2 * q2]), ex2(-sA[2 * q2 + 1]));
              l2[q2] = __fmul2_rn(l2[q2], al);
              const float2 o = __fmul2_rn(make_float2(__uint_as_float(raw[2 * q2]), __uint_as_float(raw[2 * q2 + 1])), al);
              raw[2 * q2] = __float_as_uint(o.x);
              raw[2 * q2 + 1] = __float_as_uint(o.y);
            }
            tmem_st64(tmem + lane_addr + col_o(x), raw);
          }
          tmem_ld64(s_addr, raw);  // the tile again, for the exponentials
        }
        tc_fence_before();
        mbar_arrive(bar(B_S_FREE + 2 * x + sb));  // the S^T buffer may be refilled
        ++gs;
        // P = 2^(S * scale - m) in bf16, row r of the MN-major P^T tile; the row
        // sums add the same bf16 values. The tile was last read by step n - kPTiles.
        if (n_step >= (uint32_t)kPTiles) wait_step_pv(n_step - kPTiles);
        uint8_t* const prow = smem + kOffP + (n_step % kPTiles) * kPBytes + r * 128;
        if (!valid) {
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
            *reinterpret_cast<uint4*>(prow + ((cc ^ (r & 7)) << 4)) = make_uint4(0u, 0u, 0u, 0u);
        } else {
          const float2 c22 = make_float2(c2, c2);
          // The maxima of group cc + 1 are read before the P store of group cc:
          // a shared load that follows a shared store would wait for it.
          float4 n0 = reinterpret_cast<const float4*>(sNM)[0];
          float4 n1 = reinterpret_cast<const float4*>(sNM)[1];
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const float2 nm[4] = {make_float2(n0.x, n0.y), make_float2(n0.z, n0.w), make_float2(n1.x, n1.y),
                                  make_float2(n1.z, n1.w)};
            if (cc < 7) {
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
            *reinterpret_cast<uint4*>(prow + ((cc ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        if (r == 0) sPMeta[n_step % kPTiles] = step_meta(x, c == 0, c == C - 1, nblk);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        tc_fence_before();
        mbar_arrive(bar(B_P_FULL + n_step % kPTiles));
        lastn = n_step;
      }
      // ---------------------------------------------------------------- epilogue
      if (C > 0) {
        // the item's last PV has finished: O^T is complete
        mbar_wait(bar(B_O_DONE + x), go & 1, sAbort, a.hdr, 23);
        ++go;
      }
      tc_fence_after();
      {
        float* lf = reinterpret_cast<float*>(l2);
        const int col0 = warp_col_reduce<false>(*reinterpret_cast<float(*)[64]>(lf), lane);
        sRed[sp * 64 + col0] = lf[0];
        sRed[sp * 64 + col0 + 1] = lf[1];
      }
      softmax_sync(bar_id);
      float lsum = 0.f;
      if (r < 64) {
        lsum = (sRed[r] + sRed[64 + r]) + (sRed[128 + r] + sRed[192 + r]);
        sL[r] = lsum > 0.f ? 1.0f / lsum : 0.f;
      }
      softmax_sync(bar_id);
      const size_t row0 = ((size_t)it.b * a.Hq + it.h) * a.N + (size_t)it.i * kBS;
      {
        uint32_t o[64];
        if (C > 0) {
          tmem_ld64(tmem + lane_addr + col_o(x), o);
        } else {
#pragma unroll
          for (int q = 0; q < 64; ++q) o[q] = 0u;
        }
        tc_fence_before();
        // thread r holds column r of the 64 output rows: each warp store covers
        // 32 consecutive head-dim elements of one row
        __nv_bfloat16* const dst = a.out + row0 * kD + r;
#pragma unroll
        for (int q = 0; q < 64; ++q) dst[(size_t)q * kD] = __float2bfloat16_rn(__uint_as_float(o[q]) * sL[q]);
      }
      if (a.lse != nullptr && r < 64)
        a.lse[row0 + r] = (C > 0 && lsum > 0.f) ? (-sNM[r] * kLn2 + logf(lsum)) : -INFINITY;
      softmax_sync(bar_id);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D map over a [rows][128] bf16 tensor, 64 x 64 boxes, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, unsigned long long rows) {
  EncodeTiledFn f = encode_fn();
  if (f == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)kBS};
  cuuint32_t estr[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool attn_tc_supported(const Shape& s) {
  // TMA row coordinates are 32-bit
  const unsigned long long rows = (unsigned long long)s.B * s.Hq * s.N;
  return s.bs == kBS && s.d == kD && rows < (1ull << 31) && encode_fn() != nullptr;
}

cudaError_t launch_attn_tc(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, const int32_t* idx, const int32_t* cnt,
                           __nv_bfloat16* out, float* lse, WsHeader* hdr, cudaStream_t st) {
  if (!attn_tc_supported(s)) return cudaErrorNotSupported;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, (unsigned long long)s.B * s.Hq * s.N) ||
      !make_map(&mk, k, (unsigned long long)s.B * s.Hkv * s.N) ||
      !make_map(&mv, v, (unsigned long long)s.B * s.Hkv * s.N))
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
  e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(&hdr->work[0], 0, sizeof(unsigned int), st);
  if (e != cudaSuccess) return e;
  const int grid = a.n_items < sms ? a.n_items : sms;
  attn_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace dsa
