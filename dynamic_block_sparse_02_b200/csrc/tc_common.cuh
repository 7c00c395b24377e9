// PTX helpers shared by the tcgen05 kernels: mbarriers with bounded waits,
// tensor-TMA loads, tcgen05 MMA / commit / TMEM loads and stores, shared
// memory matrix descriptors and instruction descriptors, and the host-side
// tensor-map encoder.
#pragma once

#include <cuda.h>

#include "dsa_internal.cuh"

namespace dsa {
namespace tc {

// Default limit of every bounded wait (ns); a workspace header may lower it
// (WsHeader::wait_limit_ns) so that a test can make a wait give up.
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;

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

// Per-CTA state of the bounded waits, in shared memory: the abort flag (set
// by the first wait that gives up; every later wait returns at once) and the
// wait limit, read only on the slow path so that it occupies no register.
struct CtaFlags {
  int abort;
  int pad;
  unsigned long long limit_ns;
};

// What a bounded wait needs to know (passed by value; no local memory).
struct WaitCtx {
  volatile CtaFlags* f;
  WsHeader* hdr;
  int kernel;
};

// Bounded wait. Returns false (and raises the CTA abort flag and the device
// error) when the phase does not complete within the limit, or at once when
// the CTA is already aborting. The first probe is inlined; the spin loop is
// out of line so that callers keep their registers on the fast path. A
// try_wait may itself suspend for a while, so the limit and the abort flag are
// checked after the first failed probe and then every 8 probes.
template <bool kInline>
__device__ __forceinline__ bool mbar_wait_spin(uint32_t bar, uint32_t parity, volatile CtaFlags* f,
                                               WsHeader* hdr, int kernel, int where) {
  const unsigned long long t0 = now_ns();
  const unsigned long long limit = f->limit_ns;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if (it == 1u || (it & 7u) == 0u) {
      if (f->abort) return false;
      if (now_ns() - t0 > limit) {
        f->abort = 1;
        raise_error(hdr, DSA_ERR_DEVICE_TIMEOUT, kernel, where, (int)blockIdx.x);
        return false;
      }
    }
  }
}

static __device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile CtaFlags* f,
                                            WsHeader* hdr, int kernel, int where) {
  return mbar_wait_spin<false>(bar, parity, f, hdr, kernel, where);
}

// kInline: the spin loop is inlined (for warps that run after setmaxnreg.inc,
// where ptxas cannot call out of line), else it is called out of line so that
// the caller keeps its registers on the fast path.
template <bool kInline = false>
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, WaitCtx w, int where) {
  if (mbar_try(bar, parity)) return true;
  if (kInline) return mbar_wait_spin<true>(bar, parity, w.f, w.hdr, w.kernel, where);
  return mbar_wait_slow(bar, parity, w.f, w.hdr, w.kernel, where);
}

// Wait used while draining (after an abort or at the end): it ignores the
// abort flag and always allows the default limit, so that every copy and MMA
// already issued has landed before shared memory or TMEM is given up. Returns
// false only if even that limit passes (reported as a timeout).
__device__ __forceinline__ bool mbar_drain(uint32_t bar, uint32_t parity, WsHeader* hdr, int kernel,
                                        int where) {
  const unsigned long long t0 = now_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it == 1u || (it & 7u) == 0u) && now_ns() - t0 > kDefaultWaitNs) {
      raise_error(hdr, DSA_ERR_DEVICE_TIMEOUT, kernel, where, (int)blockIdx.x);
      return false;
    }
  }
}

// Waits for a barrier phase that belongs to walk step n. Returns 1 when the
// phase completed, 0 when the walk has fewer than n + 1 steps (the step and
// its phase never come), -1 when the kernel is aborting or the wait timed out.
static __device__ __noinline__ int step_wait_slow(uint32_t bar, uint32_t parity, volatile uint32_t* total,
                                           uint32_t n, volatile CtaFlags* f, WsHeader* hdr,
                                           int kernel, int where) {
  const unsigned long long t0 = now_ns();
  const unsigned long long limit = f->limit_ns;
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return 1;
    if (*total <= n) return 0;
    if (it == 1u || (it & 7u) == 0u) {
      if (f->abort) return -1;
      if (now_ns() - t0 > limit) {
        f->abort = 1;
        raise_error(hdr, DSA_ERR_DEVICE_TIMEOUT, kernel, where, (int)blockIdx.x);
        return -1;
      }
    }
  }
}

__device__ __forceinline__ int step_wait(uint32_t bar, uint32_t parity, volatile uint32_t* total,
                                         uint32_t n, WaitCtx w, int where) {
  if (mbar_try(bar, parity)) return 1;
  return step_wait_slow(bar, parity, total, n, w.f, w.hdr, w.kernel, where);
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

// D (TMEM) (+)= A (shared) . B (shared), kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// TMEM loads and stores of 32 or 64 consecutive fp32 columns of this warp's
// 32 lanes (shape 32x32b), followed by the wait. The register arrays are bound
// to the asm operands element by element through array references, so they
// stay in registers.
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  tmem_wait_ld();
}

__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[64]) {
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
  tmem_wait_ld();
}

__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
      "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]),
      "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]),
      "r"(r[30]), "r"(r[31])
      : "memory");
  tmem_wait_st();
}

__device__ __forceinline__ void tmem_st(uint32_t taddr, const uint32_t (&r)[64]) {
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
  tmem_wait_st();
}

// Register rebalancing between warpgroups (every thread of the warpgroup
// executes it). The counts of all warpgroups must add up to at most the
// registers the block was launched with.
template <int N>
__device__ __forceinline__ void reg_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void reg_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
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

// Named barrier over the 128 threads of one warpgroup, optionally OR-reducing
// a predicate.
__device__ __forceinline__ void wg_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }
__device__ __forceinline__ bool wg_any(int id, bool pred) {
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

// Shared-memory matrix descriptor (sm_100 format). layout: 2 = 128-byte
// swizzle, 4 = 64-byte swizzle. lbo / sbo in bytes: for a K-major operand
// sbo is the stride between 8-row groups; for an MN-major operand lbo is the
// stride between swizzle atoms along M/N and sbo between 8-row groups along K.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout = 2) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}

// Instruction descriptor of kind::f16: bf16 x bf16 -> fp32, shape M x N,
// A / B K-major (0) or MN-major (1).
constexpr uint32_t idesc_bf16(int M, int N, uint32_t a_mn_major, uint32_t b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (a_mn_major << 15) | (b_mn_major << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
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

// The (stream, chunk) walk shared by the producers and both MMA issuers.
// Streams alternate one chunk at a time; a stream whose item has no chunks
// moves on to its next item without taking a step; once one stream runs out
// of items the other takes every remaining step. An item of n kept blocks has
// ceil(n / per_chunk) chunks.
template <int kPerChunk>
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
    const int chunks = (n + kPerChunk - 1) / kPerChunk;
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

// Step metadata word: stream, first and last chunk of the item, kept blocks in the chunk.
__device__ __forceinline__ uint32_t step_meta(int x, bool first, bool last, int nblk) {
  return (uint32_t)x | (first ? 2u : 0u) | (last ? 4u : 0u) | ((uint32_t)nblk << 3);
}

// Work item order shared by the attention kernels: KV-head-major; inside a
// KV head, query blocks from the last (longest) down; the group's query heads
// interleaved.
__device__ __forceinline__ void decode_item(int item, int group, int nb, int Hkv, int& b, int& h,
                                            int& i) {
  const int per_kv = group * nb;
  const int bk = item / per_kv;
  const int rem = item - bk * per_kv;
  b = bk / Hkv;
  const int kvh = bk - b * Hkv;
  i = nb - 1 - rem / group;
  h = kvh * group + rem % group;
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
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

// 2-D map over a [rows][d] bf16 tensor: boxes of 64 d-elements x box_rows
// rows, 128-byte swizzle (one box row = one 128-byte swizzle row).
inline bool make_map(CUtensorMap* m, const void* base, unsigned long long rows, int d, int box_rows) {
  EncodeTiledFn f = encode_fn();
  if (f == nullptr) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return f(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Wait limit a kernel uses: the header's value when set, else the default.
__device__ __forceinline__ unsigned long long wait_limit(const WsHeader* hdr) {
  if (hdr == nullptr) return kDefaultWaitNs;
  const unsigned long long v = *reinterpret_cast<const volatile unsigned long long*>(&hdr->wait_limit_ns);
  return v == 0ull ? kDefaultWaitNs : v;
}

}  // namespace tc
}  // namespace dsa
