// Internal declarations shared by the kernels and the C-ABI host code.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/dsa.h"

namespace dsa {

// Workspace header (the first kHeaderBytes of the caller's workspace).
struct WsHeader {
  int status;           // first device-side error (dsa_status value), 0 = none
  int detail[3];        // kernel id and a coordinate of the first error
  unsigned int work[8]; // work counters of persistent kernels (reset per call)
  unsigned long long wait_limit_ns;  // limit of the kernels' bounded waits; 0 = default (2 s)
};
constexpr size_t kHeaderBytes = 256;
static_assert(sizeof(WsHeader) <= kHeaderBytes, "header too large");

constexpr int kMaxBlocks = 1024;  // largest nb = N / block
constexpr int kMaxHeads = 256;    // largest Hq when k_per_head is given

// Kernel ids reported in WsHeader::detail[0].
enum KernelId { kKernPool = 1, kKernScore = 2, kKernSelect = 3, kKernAttnMma = 4, kKernAttnTc = 5,
                kKernDecode = 6, kKernAttnBwd = 7 };

// Derived, validated problem description.
struct Shape {
  int B, Hq, Hkv, N, d, bs, nb, group, W;
  int lw, ns;
  float scale;
  int kmax_head;
  bool per_head;
  bool group_select;  // DSA_SELECT_GROUP_TOPK: one list per KV head, copied to its query heads
  float tau;          // DSA_SELECT_THRESHOLD: tau (0 in the other modes)
  float c2;           // scale * log2(e): block logits in base 2
};

// Per-head top-k budgets passed by value to the kernels.
struct KBudget {
  int32_t k[kMaxHeads];
};

// Device-side error reporting: the first error wins.
__device__ __forceinline__ void raise_error(WsHeader* hdr, int status, int kernel, int a, int b) {
  if (hdr == nullptr) return;
  if (atomicCAS(&hdr->status, 0, status) == 0) {
    hdr->detail[0] = kernel;
    hdr->detail[1] = a;
    hdr->detail[2] = b;
  }
}

// Entry t = j of a caller's kept list lst (in: t < the row's count): it is
// used only if 0 <= j <= i and j is greater than the entry before it in the
// list (rows are ascending without repeats); other entries are skipped and
// flagged by the caller. The entry before is read again from the list (the
// same cache line, no state carried between entries).
__device__ __forceinline__ bool list_entry_ok(const int32_t* lst, int t, int j, int i, bool in) {
  return in && j >= 0 && j <= i && (t == 0 || j > lst[t - 1]);
}

// Launchers (return cudaSuccess or the launch error).
cudaError_t launch_pool(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k, float* qp,
                        float* kp, cudaStream_t st);
cudaError_t launch_scores(const Shape& s, const float* qp, const float* kp, float* scores,
                          cudaStream_t st);
cudaError_t launch_score_select(const Shape& s, const KBudget& kb, const float* qp, const float* kp,
                                int32_t* idx, int32_t* cnt, WsHeader* hdr, cudaStream_t st);
cudaError_t launch_select(const Shape& s, const KBudget& kb, const float* scores, int32_t* idx,
                          int32_t* cnt, WsHeader* hdr, cudaStream_t st);
// Pooling of key blocks [j0, j1) of every (batch, KV head) of a cache of nb blocks.
cudaError_t launch_pool_range(const Shape& s, const __nv_bfloat16* k, float* kp, int j0, int j1,
                              cudaStream_t st);
// Decode workspace after the header: fp32 scores [B, Hq, nb] (per-head rows;
// the group-shared rule uses the first B*Hkv rows for the groups' sums), fp32
// partial softmax states [B, Hq, kDecMaxSplit', d + 4] (output row, m, l) with
// kDecMaxSplit' = min(kDecMaxSplit, nb) splits of a head's kept blocks, and one
// arrival counter per (batch, KV head, chunk of 8 query heads).
constexpr int kDecMaxSplit = 64;
constexpr int kDecHeadChunk = 8;
struct DecodeWs {
  size_t scores, part, ctr, total;
  int smax;
};
inline size_t ws_round_up(size_t x) { return (x + 255) / 256 * 256; }
inline DecodeWs decode_ws_layout(const Shape& s) {
  DecodeWs w;
  w.smax = s.nb < kDecMaxSplit ? s.nb : kDecMaxSplit;
  const int hc = (s.group + kDecHeadChunk - 1) / kDecHeadChunk;
  size_t off = kHeaderBytes;
  w.scores = off;
  off += ws_round_up((size_t)s.B * s.Hq * s.nb * sizeof(float));
  w.part = off;
  off += ws_round_up((size_t)s.B * s.Hq * w.smax * (s.d + 4) * sizeof(float));
  w.ctr = off;
  off += ws_round_up((size_t)s.B * s.Hkv * hc * sizeof(int));
  w.total = off;
  return w;
}

// Backward workspace after the header: fp32 D_r = dO_r . O_r and base-2 lse
// per query row [B, Hq, N], and the transposed kept lists, one bitmap of
// cw = ceil(G * nb / 32) words per key block [B, Hkv, nb, cw].
// For the tensor-core backward also the transposed lists as pair lists
// (int32 bit positions, G (nb - j) slots for key block j, packed per (b, g):
// [B, Hkv, G nb (nb + 1) / 2]) and their lengths [B, Hkv, nb].
struct BwdWs {
  size_t drow, lse2, colbits, pairs, npairs, total;
  int cw;
};
inline BwdWs bwd_ws_layout(const Shape& s) {
  BwdWs w;
  w.cw = (s.group * s.nb + 31) / 32;
  size_t off = kHeaderBytes;
  w.drow = off;
  off += ws_round_up((size_t)s.B * s.Hq * s.N * sizeof(float));
  w.lse2 = off;
  off += ws_round_up((size_t)s.B * s.Hq * s.N * sizeof(float));
  w.colbits = off;
  off += ws_round_up((size_t)s.B * s.Hkv * s.nb * w.cw * sizeof(uint32_t));
  w.pairs = off;
  off += ws_round_up((size_t)s.B * s.Hkv * s.group * ((size_t)s.nb * (s.nb + 1) / 2) * sizeof(int32_t));
  w.npairs = off;
  off += ws_round_up((size_t)s.B * s.Hkv * s.nb * sizeof(int32_t));
  w.total = off;
  return w;
}

// Arguments of the tensor-core backward (attn_bwd_tc.cu).
struct BwdTcArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* dout;
  const int32_t* idx;
  const int32_t* cnt;
  const float* drow;   // D_r = dO_r . O_r
  const float* lse2;   // lse * log2(e), +inf for a row with no visible key
  const uint32_t* colbits;
  int32_t* pairs;
  int32_t* npairs;
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  WsHeader* hdr;
  int B, Hq, Hkv, N, nb, W, group, cw;
  float scale, c2;
};
bool attn_bwd_tc_supported(const Shape& s);
// dQ, dK, dV on the tensor cores, after the D / lse2 and bitmap kernels.
cudaError_t launch_attn_bwd_tc(const Shape& s, const BwdTcArgs& a, cudaStream_t st);

// Backward of the sparse attention over the kept blocks (dQ, dK, dV).
cudaError_t launch_attn_bwd(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                            const __nv_bfloat16* v, const __nv_bfloat16* o, const float* lse,
                            const __nv_bfloat16* dout, const int32_t* idx, const int32_t* cnt,
                            __nv_bfloat16* dq, __nv_bfloat16* dk, __nv_bfloat16* dv, void* ws,
                            bool use_tc, cudaStream_t st);

// Decode step: one query token per (batch, query head) at position length - 1.
cudaError_t launch_decode(const Shape& s, const KBudget& kb, const __nv_bfloat16* q,
                          const __nv_bfloat16* k, const __nv_bfloat16* v, const float* kp,
                          int length, __nv_bfloat16* out, float* lse, int32_t* idx, int32_t* cnt,
                          void* ws, cudaStream_t st);
cudaError_t launch_attn_mma(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                            const __nv_bfloat16* v, const int32_t* idx, const int32_t* cnt,
                            __nv_bfloat16* out, float* lse, WsHeader* hdr, cudaStream_t st);
bool attn_tc_supported(const Shape& s);
// 128x128 blocks (attn_tc128.cu); called by launch_attn_tc.
cudaError_t launch_attn_tc128(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                              const __nv_bfloat16* v, const int32_t* idx, const int32_t* cnt,
                              __nv_bfloat16* out, float* lse, WsHeader* hdr, cudaStream_t st);
cudaError_t launch_attn_tc(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, const int32_t* idx, const int32_t* cnt,
                           __nv_bfloat16* out, float* lse, WsHeader* hdr, cudaStream_t st);

}  // namespace dsa
