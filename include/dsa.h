/*
 * dsa.h — C ABI of libdsa: dynamic top-k block-sparse causal attention
 * (prefill) on NVIDIA B200 (sm_100a).
 *
 * The operation, as the pages describe it:
 *   1. Pool.   Each bs x bs tile of the attention matrix is decided as a unit
 *              (zblog.xzdbk.com/559 dynamic-sparse-attention post, section
 *              硬件友好的稀疏计算实现, 64x64 blocks; "DeepSeek NSA" article,
 *              section 2.1, 32x32 blocks with a light per-block estimate).
 *              The estimate used here: Qp[i] = mean of query block i,
 *              Kp[j] = mean of key block j (fp32).
 *   2. Score.  s(i, j) = Qp[i] . Kp[j] for j <= i, in fp32 ("DeepSeek NSA",
 *              section 2.2: the routing decision stays in FP32).
 *   3. Select. Per (batch, query head, query block i): the forced blocks
 *              F(i) = {i-w+1 .. i} U {0 .. n_sink-1} (causal part only) plus the
 *              k best remaining causal blocks, best = higher score, ties to
 *              the lower block index (zblog post, section
 *              基于Top-k选择的局部-全局混合: top-k with local window and global
 *              tokens).
 *   4. Attend. O = softmax(Q K^T * scale) V over the kept blocks only, causal
 *              inside the diagonal block, online softmax, query head h reading
 *              KV head h / (Hq/Hkv) ("稀疏注意力 vs Flash Attention v2",
 *              section 1 pseudocode; "DeepSeek NSA", section 2.2, bf16 matmul).
 *
 * Conventions for every entry point:
 *   - Tensors are DEVICE pointers to contiguous row-major arrays, d innermost:
 *     Q and O [B, Hq, N, d]; K and V [B, Hkv, N, d]; all bf16 (dsa_bf16 is the
 *     16-bit pattern of one bfloat16). Q, K, V, O and the workspace must be
 *     16-byte aligned.
 *   - Block index rows: idx int32 [B, Hq, nb, W] with nb = N / block and
 *     W = dsa_kmax(p); each row lists its kept key blocks in ascending order,
 *     padded with -1; cnt int32 [B, Hq, nb] holds each row's length. When
 *     W == 0 (no block can be kept) idx may be NULL.
 *   - The caller owns all memory. The library never allocates device or host
 *     memory; it uses the caller's workspace (dsa_workspace_size bytes), except
 *     dsa_select_blocks_static, whose scratch is the library's static device
 *     array.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) and do not synchronise the host, so a sequence of calls
 *     can be captured into a CUDA graph.
 *   - An argument error is reported synchronously by the return value and
 *     launches nothing. Errors found on the device (an index out of range, a
 *     bounded wait that gave up) set a flag in the workspace header; read it
 *     with dsa_check_status.
 *   - The device must be an sm_100a GPU (B200). The library holds no state
 *     except, per device, a cache of the kernels' shared-memory attributes
 *     and the static scratch array of dsa_select_blocks_static.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t dsa_bf16; /* bit pattern of one bfloat16 value */

typedef enum dsa_status {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1,    /* a null/misaligned pointer, a negative size, Hq % Hkv != 0, ... */
  DSA_ERR_UNSUPPORTED = 2,    /* valid but outside the supported shapes (see dsa_params) */
  DSA_ERR_WORKSPACE = 3,      /* workspace missing or smaller than dsa_workspace_size */
  DSA_ERR_CUDA = 4,           /* a CUDA runtime call or a kernel launch failed */
  DSA_ERR_DEVICE_TIMEOUT = 5, /* a bounded wait inside a kernel gave up (device flag) */
  DSA_ERR_DEVICE_BOUNDS = 6   /* a kernel met an index outside its valid range (device flag) */
} dsa_status;

/* Selection rule (dsa_params.select_mode). */
typedef enum dsa_select_mode {
  DSA_SELECT_TOPK = 0,       /* per (batch, query head, query block): forced + top-k (steps 1-3 above) */
  DSA_SELECT_GROUP_TOPK = 1, /* per (batch, KV head, query block): the same rule on the sum of the
                                group's query-head scores s_h (fp32, added in head order); every
                                query head of the group receives that list. The pages note that
                                GQA's shared KV cache makes one index per KV head natural
                                (zblog.xzdbk.com/559 post, section on speculative decoding) and
                                merge the lists of several index heads (DSA post, section 2.1). */
  DSA_SELECT_THRESHOLD = 2   /* per (batch, query head, query block): forced + the remaining causal
                                blocks j whose block probability softmax_j(scale * s(i, j)) over
                                j <= i is >= select_tau, at most k of them (the best first). The
                                DeepSeek NSA article, section 2.2, thresholds the fp32 scores
                                (0.1), section 4.2 starts the threshold at 0.05; the zblog post
                                adapts k or the threshold per input. */
} dsa_select_mode;

/* Attention kernel choice (dsa_params.attn_kernel). AUTO runs the tcgen05
 * kernel for every supported shape (block 32, 64 or 128, d 64 or 128) and the
 * warp-MMA kernel otherwise; dsa_attn_uses_tcgen05 reports the choice. */
typedef enum dsa_attn_kernel {
  DSA_ATTN_AUTO = 0,     /* the tcgen05 kernel where the shape has one, else warp-MMA */
  DSA_ATTN_TCGEN05 = 1,  /* tcgen05/TMEM tensor-core kernel with TMA tile loads */
  DSA_ATTN_MMA_SYNC = 2  /* warp-level mma.sync kernel (the legacy tensor-core path) */
} dsa_attn_kernel;

/*
 * Problem shape and selection settings.
 *   B, Hq, Hkv, N, d : batch, query heads, KV heads, tokens, head dim.
 *                      Hq % Hkv == 0; d is 64 or 128; B == 0 or N == 0 is an
 *                      empty problem (every call returns DSA_OK, launches nothing).
 *   block            : tile edge bs, one of 32, 64, 128; N % block == 0;
 *                      nb = N / block must be <= 1024.
 *   k_free           : top-k picks beyond the forced set, for every head
 *                      (used when k_per_head is NULL); >= 0.
 *   k_per_head       : optional HOST array of Hq budgets (>= 0), shared across
 *                      the batch; read during the call only. Hq <= 256 then.
 *   local_window     : w >= 0; forces blocks {i-w+1 .. i} (1 = diagonal only).
 *   n_sink           : >= 0; forces blocks {0 .. n_sink-1}.
 *   scale            : softmax scale; 0 means 1/sqrt(d); must be finite, >= 0.
 *   attn_kernel      : a dsa_attn_kernel value.
 *   select_mode      : a dsa_select_mode value. DSA_SELECT_GROUP_TOPK needs
 *                      k_per_head == NULL and Hq/Hkv <= 32.
 *   select_tau       : DSA_SELECT_THRESHOLD: the threshold tau, 0 < tau <= 1;
 *                      other modes: must be 0. The block probabilities are
 *                      computed in fp32 (exp2 of c2 * (s - max) over their
 *                      fp32 sum, c2 = scale * log2(e)), so a block j of query
 *                      block i whose exact probability p_j is within
 *                      delta_j * tau of tau may fall on either side, with
 *                        eps_j   = (block + d) 2^-24 sum_d mean|q_d| mean|k_jd|
 *                                  (fp32 error bound of the score s(i, j);
 *                                  mean|.| over the block's rows),
 *                        eta_j   = c2 (eps_j + max eps) + 2^-23 c2 |s_j - max s|,
 *                        delta_j = ln2 (eta_j + max eta) + (i + 5) 2^-24 + 2^-21.
 */
typedef struct dsa_params {
  int B, Hq, Hkv, N, d;
  int block;
  int k_free;
  const int32_t *k_per_head;
  int local_window;
  int n_sink;
  float scale;
  int attn_kernel;
  int select_mode;
  float select_tau;
} dsa_params;

/* Row width W of idx: min(nb, max_h k_h + local_window + n_sink). 0 for an
 * invalid or empty problem. */
size_t dsa_kmax(const dsa_params *p);

/* Which kernel the forward attention (step 4 of dsa_forward and
 * dsa_sparse_attn_fwd) runs for p: 1 the tcgen05 kernel, 0 the warp-MMA
 * kernel, -1 when p is invalid or asks for DSA_ATTN_TCGEN05 on a shape that
 * kernel does not support. No device work; safe to call without a GPU. */
int dsa_attn_uses_tcgen05(const dsa_params *p);

/* Bytes of device workspace the calls below need for this problem (*bytes is
 * set on success). The first 256 bytes are a header (device error flag, work
 * counters); zero them once after allocating (dsa_workspace_init). */
dsa_status dsa_workspace_size(const dsa_params *p, size_t *bytes);

/* Zero the workspace header on `stream` (asynchronous). */
dsa_status dsa_workspace_init(void *ws, size_t ws_bytes, void *stream);

/*
 * Set the time limit of the kernels' bounded waits for calls that use this
 * workspace (asynchronous on `stream`; stored in the workspace header, which
 * dsa_workspace_init resets to 0). ns = 0 selects the default (2 s for the
 * tensor-core kernels, 1 s for the decode kernel). Every wait inside the
 * pipelined kernels (a stage that has not arrived, a buffer not yet released)
 * is bounded: when one gives up, the kernel raises DSA_ERR_DEVICE_TIMEOUT,
 * stops issuing work, waits (with the default limit) for the copies and
 * tensor-core products it has in flight, frees its tensor memory and returns;
 * its outputs are then undefined. A tiny limit makes the waits give up on
 * purpose, which is how the failure path is tested. There is no counterpart
 * in the pages: the pages describe no failure handling.
 */
dsa_status dsa_workspace_set_wait_limit(void *ws, size_t ws_bytes, unsigned long long ns, void *stream);

/*
 * Steps 1-2. scores: device fp32 [B, Hq, nb, nb]; scores[b,h,i,j] =
 * Qp[b,h,i] . Kp[b,h/(Hq/Hkv),j] for j <= i and -inf for j > i.
 * Uses the workspace for the pooled blocks.
 */
dsa_status dsa_block_scores(const dsa_params *p, const dsa_bf16 *q, const dsa_bf16 *k,
                            float *scores, void *ws, size_t ws_bytes, void *stream);

/*
 * Step 3 on caller scores laid out as dsa_block_scores writes them (only the
 * entries j <= i are read). Writes idx [B,Hq,nb,W] and cnt [B,Hq,nb]. Given
 * the scores of dsa_block_scores, the result equals the selection inside
 * dsa_forward bit for bit.
 */
dsa_status dsa_topk_select(const dsa_params *p, const float *scores, int32_t *idx,
                           int32_t *cnt, void *stream);

/*
 * Steps 1-3 in one call (pool, score, select); the scores stay on chip and
 * only the selection is written: idx [B,Hq,nb,W], cnt [B,Hq,nb]. The result
 * equals dsa_block_scores followed by dsa_topk_select, bit for bit, and is the
 * selection dsa_forward uses.
 */
dsa_status dsa_select_blocks(const dsa_params *p, const dsa_bf16 *q, const dsa_bf16 *k,
                             int32_t *idx, int32_t *cnt, void *ws, size_t ws_bytes,
                             void *stream);

/*
 * Steps 1-3 like dsa_select_blocks, for callers that cannot give the library
 * a workspace (a host loop that may not call cudaMalloc, which can
 * synchronise the device; a runtime whose device memory is planned once at
 * start-up). The pages describe no such variant: it exists only so that the
 * selection can run with no caller memory besides q, k, idx and cnt.
 *   - Scratch: the pooled blocks live in a 16 MiB array in the library's own
 *     static device memory (one per device, placed there when the CUDA driver
 *     loads the library's module); nothing is allocated and nothing in it
 *     needs to start at zero. A problem whose pooled Qp and Kp (fp32,
 *     B*(Hq+Hkv)*nb*d*4 bytes, each part rounded up to 256) exceed 16 MiB gets
 *     DSA_ERR_WORKSPACE and launches nothing.
 *   - Set-up: the first call in a device's CUDA context looks the array's
 *     address up (cudaGetSymbolAddress, with that device current) and caches
 *     it per context; make that first call before any stream capture on the
 *     device. A context that is destroyed and created again (e.g. after
 *     cudaDeviceReset) gets a new lookup on its first call; the array's
 *     contents do not survive the reset.
 *   - Overlapping calls on one device (two streams, two host threads) share
 *     the array and race: order them (one stream, or events).
 *   - Arguments, outputs and argument errors as dsa_select_blocks; the result
 *     equals dsa_select_blocks bit for bit. There is no workspace header, so
 *     no device error flag is set (the selection kernel still skips any write
 *     past a row's W entries).
 */
dsa_status dsa_select_blocks_static(const dsa_params *p, const dsa_bf16 *q, const dsa_bf16 *k,
                                    int32_t *idx, int32_t *cnt, void *stream);

/*
 * Step 4 on a caller selection. idx/cnt as above, W = dsa_kmax(p); every
 * entry n < cnt must satisfy 0 <= idx <= i, and a row must be ascending
 * without repeats. The kernel skips, and flags with DSA_ERR_DEVICE_BOUNDS, an
 * entry out of range or not greater than the entry before it in the row (a
 * repeat or a step down), and attends over the rest. out: bf16
 * [B,Hq,N,d] (round to nearest even). lse: optional fp32 [B,Hq,N], natural-log
 * log-sum-exp of the scaled logits of each row. A row with no visible key
 * gets out = 0 and lse = -inf.
 */
dsa_status dsa_sparse_attn_fwd(const dsa_params *p, const dsa_bf16 *q, const dsa_bf16 *k,
                               const dsa_bf16 *v, const int32_t *idx, const int32_t *cnt,
                               dsa_bf16 *out, float *lse, void *ws, size_t ws_bytes,
                               void *stream);

/*
 * Backward of step 4: gradients of the attention over the kept blocks with
 * the kept lists held fixed (the selection is a discrete choice and passes no
 * gradient). The DeepSeek NSA article (section 2.2) trains with the sparse
 * pattern but states no backward rule; this is the exact gradient of
 * O = softmax(Q K^T * scale) V over the kept, causally visible keys:
 * P = exp(S * scale - lse), dP = dO V^T, D = rowsum(dO * O),
 * dS = P * (dP - D), dQ = scale * dS K, dK = scale * dS^T Q, dV = P^T dO,
 * with dK, dV of a KV head summed over its query heads.
 * q, out, dout, dq: bf16 [B, Hq, N, d]; k, v, dk, dv: bf16 [B, Hkv, N, d];
 * out and lse (fp32 [B, Hq, N], natural log, -inf for a row with no visible
 * key) are the forward's outputs for the same idx/cnt (int32 [B, Hq, nb, W]
 * and [B, Hq, nb]). dq, dk, dv are written in full (zero where nothing
 * contributes); all pointers 16-byte aligned and device-resident. ws: at
 * least dsa_workspace_size bytes. Entries outside 0 <= j <= i are skipped and
 * raise DSA_ERR_DEVICE_BOUNDS. The sums run in a fixed order: the results are
 * deterministic.
 */
dsa_status dsa_sparse_attn_bwd(const dsa_params *p, const dsa_bf16 *q, const dsa_bf16 *k,
                               const dsa_bf16 *v, const dsa_bf16 *out, const float *lse,
                               const dsa_bf16 *dout, const int32_t *idx, const int32_t *cnt,
                               dsa_bf16 *dq, dsa_bf16 *dk, dsa_bf16 *dv, void *ws,
                               size_t ws_bytes, void *stream);

/*
 * Steps 1-4 in one call; the scores never reach device memory. idx/cnt are
 * optional outputs (NULL keeps them in the workspace); lse is optional.
 */
dsa_status dsa_forward(const dsa_params *p, const dsa_bf16 *q, const dsa_bf16 *k,
                       const dsa_bf16 *v, dsa_bf16 *out, float *lse, int32_t *idx,
                       int32_t *cnt, void *ws, size_t ws_bytes, void *stream);

/*
 * Decode support: pooling of the key cache. kp[b, g, j, :] = mean of key rows
 * j*block .. j*block+block-1 of k[b, g] (fp32), for j_begin <= j < j_end.
 * k: bf16 [B, Hkv, N, d] key cache of capacity N = p->N tokens; kp: fp32
 * [B, Hkv, N/block, d], caller-owned. Call it for each block as it completes.
 */
dsa_status dsa_pool_keys(const dsa_params *p, const dsa_bf16 *k, float *kp, int j_begin,
                         int j_end, void *stream);

/*
 * Decode step: one new query token per (batch, query head) at position
 * length - 1 (1 <= length <= N), against the caches k, v bf16 [B, Hkv, N, d]
 * (rows >= length are not read) and the pooled cache kp (blocks
 * j < (length-1)/block must be pooled; the token's own block is pooled inside
 * the call from its present keys). q: bf16 [B, Hq, d]. The token's block row is
 * selected by p->select_mode exactly as in prefill (scores q . Kp[j]); out:
 * bf16 [B, Hq, d] = softmax(q K^T * scale) V over the present keys of the kept
 * blocks; lse: optional fp32 [B, Hq]; idx/cnt: optional int32 [B, Hq, W] /
 * [B, Hq] (both or neither), the kept blocks. ws: at least dsa_workspace_size
 * bytes (scores, partial softmax states of the splits, arrival counters). The zblog.xzdbk.com/559 post (section
 * 动态开销与计算收益的权衡) keeps the sparse index with the KV cache for
 * inference; here the pooled keys are kept and the index is re-derived per token.
 */
dsa_status dsa_decode_fwd(const dsa_params *p, const dsa_bf16 *q, const dsa_bf16 *k,
                          const dsa_bf16 *v, const float *kp, int length, dsa_bf16 *out,
                          float *lse, int32_t *idx, int32_t *cnt, void *ws, size_t ws_bytes,
                          void *stream);

/* Synchronise `stream`, read the device error flag in the workspace header,
 * clear it, and return it (DSA_OK if no kernel raised one). */
dsa_status dsa_check_status(void *ws, void *stream);

/* Static English text for a status value. */
const char *dsa_status_string(dsa_status s);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H */
