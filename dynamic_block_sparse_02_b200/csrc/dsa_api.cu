// C-ABI entry points of libdsa (declared in include/dsa.h): argument checks,
// workspace layout and kernel launches. No entry point allocates memory or
// synchronises the host, except dsa_check_status, which synchronises on
// purpose to read the device error flag.
#include <cmath>
#include <cuda.h>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "dsa_internal.cuh"

using dsa::Shape;

namespace {

// An NVTX range around one entry point (host side: the range covers the
// argument checks and the kernel launches, which profilers correlate with the
// kernels they issued). NVTX costs nothing unless a tool is attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

constexpr size_t kAlign = 256;

size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_empty(const dsa_params* p) { return p->B == 0 || p->N == 0; }

// Checks every field and derives the shape. Empty problems (B or N zero)
// are valid; their other fields must still be well formed.
dsa_status make_shape(const dsa_params* p, Shape* s) {
  if (p == nullptr) return DSA_ERR_INVALID_ARG;
  if (p->B < 0 || p->N < 0 || p->Hq < 1 || p->Hkv < 1 || p->d < 1 || p->block < 1)
    return DSA_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return DSA_ERR_INVALID_ARG;
  if (p->local_window < 0 || p->n_sink < 0) return DSA_ERR_INVALID_ARG;
  if (!std::isfinite(p->scale) || p->scale < 0.f) return DSA_ERR_INVALID_ARG;
  if (p->attn_kernel < DSA_ATTN_AUTO || p->attn_kernel > DSA_ATTN_MMA_SYNC)
    return DSA_ERR_INVALID_ARG;
  if (p->select_mode < DSA_SELECT_TOPK || p->select_mode > DSA_SELECT_THRESHOLD)
    return DSA_ERR_INVALID_ARG;
  if (p->select_mode == DSA_SELECT_THRESHOLD
          ? !(p->select_tau > 0.f && p->select_tau <= 1.f)
          : p->select_tau != 0.f)
    return DSA_ERR_INVALID_ARG;
  if (p->select_mode == DSA_SELECT_GROUP_TOPK && p->k_per_head != nullptr) return DSA_ERR_INVALID_ARG;
  long long kmax_head = 0;
  if (p->k_per_head != nullptr) {
    if (p->Hq > dsa::kMaxHeads) return DSA_ERR_UNSUPPORTED;
    for (int h = 0; h < p->Hq; ++h) {
      if (p->k_per_head[h] < 0) return DSA_ERR_INVALID_ARG;
      if (p->k_per_head[h] > kmax_head) kmax_head = p->k_per_head[h];
    }
  } else {
    if (p->k_free < 0) return DSA_ERR_INVALID_ARG;
    kmax_head = p->k_free;
  }
  if (p->d != 64 && p->d != 128) return DSA_ERR_UNSUPPORTED;
  if (p->block != 32 && p->block != 64 && p->block != 128) return DSA_ERR_UNSUPPORTED;
  if (p->N % p->block != 0) return DSA_ERR_UNSUPPORTED;
  if (p->select_mode == DSA_SELECT_GROUP_TOPK && p->Hq / p->Hkv > 32) return DSA_ERR_UNSUPPORTED;
  const int nb = p->N / p->block;
  if (nb > dsa::kMaxBlocks) return DSA_ERR_UNSUPPORTED;
  // element counts must stay well inside 64-bit and the grids inside 2^31
  const long long elems = (long long)p->B * p->Hq * p->N * p->d;
  if ((long long)p->B * p->Hq * nb > 0x7fffffffLL || elems > (1LL << 40))
    return DSA_ERR_UNSUPPORTED;
  s->B = p->B;
  s->Hq = p->Hq;
  s->Hkv = p->Hkv;
  s->N = p->N;
  s->d = p->d;
  s->bs = p->block;
  s->nb = nb;
  s->group = p->Hq / p->Hkv;
  s->lw = p->local_window;
  s->ns = p->n_sink;
  long long w = kmax_head + (long long)p->local_window + (long long)p->n_sink;
  s->W = (int)(w < nb ? w : nb);
  s->scale = p->scale == 0.f ? 1.0f / std::sqrt((float)p->d) : p->scale;
  s->kmax_head = (int)(kmax_head < nb ? kmax_head : nb);
  s->per_head = p->k_per_head != nullptr;
  s->group_select = p->select_mode == DSA_SELECT_GROUP_TOPK;
  s->tau = p->select_mode == DSA_SELECT_THRESHOLD ? p->select_tau : 0.f;
  s->c2 = s->scale * 1.4426950408889634f;
  return DSA_OK;
}

struct Layout {
  size_t qp, kp, idx, cnt, total;
};

Layout layout(const Shape& s) {
  Layout L;
  size_t off = dsa::kHeaderBytes;
  L.qp = off;
  off += round_up((size_t)s.B * s.Hq * s.nb * s.d * sizeof(float));
  L.kp = off;
  off += round_up((size_t)s.B * s.Hkv * s.nb * s.d * sizeof(float));
  L.idx = off;
  off += round_up((size_t)s.B * s.Hq * s.nb * s.W * sizeof(int32_t));
  L.cnt = off;
  off += round_up((size_t)s.B * s.Hq * s.nb * sizeof(int32_t));
  L.total = off;
  return L;
}

dsa_status check_ws(const Shape& s, const void* ws, size_t ws_bytes) {
  if (ws == nullptr || !aligned16(ws)) return DSA_ERR_WORKSPACE;
  if (ws_bytes < layout(s).total) return DSA_ERR_WORKSPACE;
  return DSA_OK;
}

// The device must be Blackwell sm_100; results are cached per device.
dsa_status check_device() {
  static int cached[64] = {0};  // 0 unknown, 1 ok, 2 unsupported
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  if (dev >= 0 && dev < 64 && cached[dev] != 0) return cached[dev] == 1 ? DSA_OK : DSA_ERR_UNSUPPORTED;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return DSA_ERR_CUDA;
  const bool ok = major == 10 && minor == 0;
  if (dev >= 0 && dev < 64) cached[dev] = ok ? 1 : 2;
  return ok ? DSA_OK : DSA_ERR_UNSUPPORTED;
}

dsa::KBudget budgets(const dsa_params* p) {
  dsa::KBudget kb;
  std::memset(&kb, 0, sizeof(kb));
  if (p->k_per_head != nullptr) {
    for (int h = 0; h < p->Hq; ++h) kb.k[h] = p->k_per_head[h];
  } else {
    kb.k[0] = p->k_free;
  }
  return kb;
}

dsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

dsa_status run_attention(const dsa_params* p, const Shape& s, const dsa_bf16* q, const dsa_bf16* k,
                         const dsa_bf16* v, const int32_t* idx, const int32_t* cnt, dsa_bf16* out,
                         float* lse, dsa::WsHeader* hdr, cudaStream_t st) {
  auto bq = reinterpret_cast<const __nv_bfloat16*>(q);
  auto bk = reinterpret_cast<const __nv_bfloat16*>(k);
  auto bv = reinterpret_cast<const __nv_bfloat16*>(v);
  auto bo = reinterpret_cast<__nv_bfloat16*>(out);
  const bool tc_ok = dsa::attn_tc_supported(s);
  if (p->attn_kernel == DSA_ATTN_TCGEN05 && !tc_ok) return DSA_ERR_UNSUPPORTED;
  if (dsa_attn_uses_tcgen05(p) == 1)
    return from_cuda(dsa::launch_attn_tc(s, bq, bk, bv, idx, cnt, bo, lse, hdr, st));
  return from_cuda(dsa::launch_attn_mma(s, bq, bk, bv, idx, cnt, bo, lse, hdr, st));
}

// Steps 1-3: pooling, then the fused score + select kernel.
dsa_status run_selection(const dsa_params* p, const Shape& s, const dsa_bf16* q, const dsa_bf16* k,
                         int32_t* idx, int32_t* cnt, void* ws, cudaStream_t st) {
  const Layout L = layout(s);
  char* base = static_cast<char*>(ws);
  auto hdr = reinterpret_cast<dsa::WsHeader*>(base);
  float* qp = reinterpret_cast<float*>(base + L.qp);
  float* kp = reinterpret_cast<float*>(base + L.kp);
  cudaError_t e = dsa::launch_pool(s, reinterpret_cast<const __nv_bfloat16*>(q),
                                   reinterpret_cast<const __nv_bfloat16*>(k), qp, kp, st);
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  return from_cuda(dsa::launch_score_select(s, budgets(p), qp, kp, idx, cnt, hdr, st));
}

}  // namespace

// ---------------------------------------------------------------------------
// Selection with its scratch in static device memory (dsa_select_blocks_static).
//
// Some callers cannot hand the library a workspace: a plain C host program
// that runs the selection step inside a loop where it may not allocate device
// memory, because cudaMalloc/cudaFree can synchronise the whole device and
// stall work queued by others, or a runtime that plans all device memory once
// at start-up and has no spare region for this step. For them the pooled
// blocks Qp and Kp live in this file-scope array instead of a workspace. The
// array belongs to this library's module: the CUDA driver places it in device
// memory when it loads the module on a device, and this code never allocates.
//
// Limit: Qp and Kp together (each rounded up to 256 bytes) must fit in
// kStaticScratchBytes = 16 MiB, which holds e.g. B=1, Hq=32, Hkv=8, N=32768,
// block=64, d=128 (8 MiB + 2 MiB). Larger problems get DSA_ERR_WORKSPACE.
//
// Nothing in the array has to start at zero: the pooling kernel writes every
// pooled value before the score/select kernel reads it. There is one array per
// device (per process), so two calls that overlap on one device (two streams,
// two host threads) race on it and must be ordered by the caller.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;

static __device__ __align__(256) unsigned char g_select_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
struct ScratchAddr {
  unsigned long long ctx_id;  // unique id of the CUDA context the address belongs to
  void* addr;
};
ScratchAddr g_scratch_addr[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current CUDA context (driver entry points
// through the runtime, so the library needs no link against libcuda).
// Returns false when there is no current context yet.
bool current_ctx_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  if (get_current == nullptr || get_id == nullptr) {
    void* f1 = nullptr;
    void* f2 = nullptr;
    cudaDriverEntryPointQueryResult q1, q2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &q1) != cudaSuccess ||
        q1 != cudaDriverEntryPointSuccess ||
        cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &q2) != cudaSuccess ||
        q2 != cudaDriverEntryPointSuccess)
      return false;
    get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    get_id = reinterpret_cast<CtxGetIdFn>(f2);
  }
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_select_scratch in the current device's context. The
// first call in a context looks it up with cudaGetSymbolAddress (which may
// load the module into that context); later calls in the same context return
// the cached address. The cache is keyed on the context's unique id, so a
// context that was destroyed and re-created (cudaDeviceReset, a primary
// context released and retained again) gets a fresh lookup, never the old
// context's address.
dsa_status select_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  unsigned long long id = 0;
  const bool have_id = current_ctx_id(&id);
  if (have_id && g_scratch_addr[dev].addr != nullptr && g_scratch_addr[dev].ctx_id == id) {
    *out = g_scratch_addr[dev].addr;
    return DSA_OK;
  }
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, g_select_scratch) != cudaSuccess || addr == nullptr)
    return DSA_ERR_CUDA;
  // the lookup has made a context current if none was
  if (!current_ctx_id(&id)) return DSA_ERR_CUDA;
  g_scratch_addr[dev].ctx_id = id;
  g_scratch_addr[dev].addr = addr;
  *out = addr;
  return DSA_OK;
}

// Bytes of g_select_scratch one problem needs: Qp then Kp.
size_t static_scratch_need(const Shape& s, size_t* kp_off) {
  *kp_off = round_up((size_t)s.B * s.Hq * s.nb * s.d * sizeof(float));
  return *kp_off + round_up((size_t)s.B * s.Hkv * s.nb * s.d * sizeof(float));
}

// Writes the wait limit into a workspace header (one thread).
__global__ void set_wait_limit_kernel(dsa::WsHeader* hdr, unsigned long long ns) { hdr->wait_limit_ns = ns; }

}  // namespace

extern "C" {

size_t dsa_kmax(const dsa_params* p) {
  Shape s;
  if (make_shape(p, &s) != DSA_OK || is_empty(p)) return 0;
  return (size_t)s.W;
}

int dsa_attn_uses_tcgen05(const dsa_params* p) {
  Shape s;
  if (make_shape(p, &s) != DSA_OK) return -1;
  const bool tc_ok = dsa::attn_tc_supported(s);
  switch (p->attn_kernel) {
    case DSA_ATTN_TCGEN05: return tc_ok ? 1 : -1;
    case DSA_ATTN_MMA_SYNC: return 0;
    default:
      return tc_ok ? 1 : 0;
  }
}

dsa_status dsa_workspace_size(const dsa_params* p, size_t* bytes) {
  if (bytes == nullptr) return DSA_ERR_INVALID_ARG;
  Shape s;
  dsa_status st = make_shape(p, &s);
  if (st != DSA_OK) return st;
  if (is_empty(p)) {
    *bytes = dsa::kHeaderBytes;
  } else {
    const size_t a = layout(s).total, b = dsa::decode_ws_layout(s).total;
    const size_t c = dsa::bwd_ws_layout(s).total;
    *bytes = a > b ? (a > c ? a : c) : (b > c ? b : c);
  }
  return DSA_OK;
}

dsa_status dsa_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr || !aligned16(ws) || ws_bytes < dsa::kHeaderBytes) return DSA_ERR_WORKSPACE;
  return from_cuda(cudaMemsetAsync(ws, 0, dsa::kHeaderBytes, (cudaStream_t)stream));
}

dsa_status dsa_workspace_set_wait_limit(void* ws, size_t ws_bytes, unsigned long long ns, void* stream) {
  if (ws == nullptr || !aligned16(ws) || ws_bytes < dsa::kHeaderBytes) return DSA_ERR_WORKSPACE;
  if (check_device() != DSA_OK) return DSA_ERR_UNSUPPORTED;
  set_wait_limit_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(static_cast<dsa::WsHeader*>(ws), ns);
  return from_cuda(cudaGetLastError());
}

dsa_status dsa_block_scores(const dsa_params* p, const dsa_bf16* q, const dsa_bf16* k,
                            float* scores, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("dsa_block_scores");
  Shape s;
  dsa_status st = make_shape(p, &s);
  if (st != DSA_OK) return st;
  if (is_empty(p)) return DSA_OK;
  if (q == nullptr || k == nullptr || scores == nullptr || !aligned16(q) || !aligned16(k) ||
      !aligned16(scores))
    return DSA_ERR_INVALID_ARG;
  if ((st = check_ws(s, ws, ws_bytes)) != DSA_OK) return st;
  if ((st = check_device()) != DSA_OK) return st;
  const Layout L = layout(s);
  char* base = static_cast<char*>(ws);
  float* qp = reinterpret_cast<float*>(base + L.qp);
  float* kp = reinterpret_cast<float*>(base + L.kp);
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = dsa::launch_pool(s, reinterpret_cast<const __nv_bfloat16*>(q),
                                   reinterpret_cast<const __nv_bfloat16*>(k), qp, kp, cs);
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  return from_cuda(dsa::launch_scores(s, qp, kp, scores, cs));
}

dsa_status dsa_topk_select(const dsa_params* p, const float* scores, int32_t* idx, int32_t* cnt,
                           void* stream) {
  NvtxRange nvtx("dsa_topk_select");
  Shape s;
  dsa_status st = make_shape(p, &s);
  if (st != DSA_OK) return st;
  if (is_empty(p)) return DSA_OK;
  if (scores == nullptr || (idx == nullptr && s.W > 0) || cnt == nullptr || !aligned16(scores))
    return DSA_ERR_INVALID_ARG;
  if ((st = check_device()) != DSA_OK) return st;
  return from_cuda(dsa::launch_select(s, budgets(p), scores, idx, cnt, nullptr, (cudaStream_t)stream));
}

dsa_status dsa_select_blocks(const dsa_params* p, const dsa_bf16* q, const dsa_bf16* k,
                             int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("dsa_select_blocks");
  Shape s;
  dsa_status st = make_shape(p, &s);
  if (st != DSA_OK) return st;
  if (is_empty(p)) return DSA_OK;
  if (q == nullptr || k == nullptr || (idx == nullptr && s.W > 0) || cnt == nullptr ||
      !aligned16(q) || !aligned16(k))
    return DSA_ERR_INVALID_ARG;
  if ((st = check_ws(s, ws, ws_bytes)) != DSA_OK) return st;
  if ((st = check_device()) != DSA_OK) return st;
  return run_selection(p, s, q, k, idx, cnt, ws, (cudaStream_t)stream);
}

dsa_status dsa_select_blocks_static(const dsa_params* p, const dsa_bf16* q, const dsa_bf16* k,
                                    int32_t* idx, int32_t* cnt, void* stream) {
  NvtxRange nvtx("dsa_select_blocks_static");
  Shape s;
  dsa_status st = make_shape(p, &s);
  if (st != DSA_OK) return st;
  if (is_empty(p)) return DSA_OK;
  if (q == nullptr || k == nullptr || (idx == nullptr && s.W > 0) || cnt == nullptr ||
      !aligned16(q) || !aligned16(k))
    return DSA_ERR_INVALID_ARG;
  size_t kp_off = 0;
  if (static_scratch_need(s, &kp_off) > kStaticScratchBytes) return DSA_ERR_WORKSPACE;
  if ((st = check_device()) != DSA_OK) return st;
  void* scratch = nullptr;
  if ((st = select_scratch(&scratch)) != DSA_OK) return st;
  char* base = static_cast<char*>(scratch);
  float* qp = reinterpret_cast<float*>(base);
  float* kp = reinterpret_cast<float*>(base + kp_off);
  cudaStream_t cs = (cudaStream_t)stream;
  cudaError_t e = dsa::launch_pool(s, reinterpret_cast<const __nv_bfloat16*>(q),
                                   reinterpret_cast<const __nv_bfloat16*>(k), qp, kp, cs);
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  // No workspace header here: the selection kernel's row-overflow guard still
  // skips an out-of-range write but has no flag to set.
  return from_cuda(dsa::launch_score_select(s, budgets(p), qp, kp, idx, cnt, nullptr, cs));
}

dsa_status dsa_sparse_attn_fwd(const dsa_params* p, const dsa_bf16* q, const dsa_bf16* k,
                               const dsa_bf16* v, const int32_t* idx, const int32_t* cnt,
                               dsa_bf16* out, float* lse, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("dsa_sparse_attn_fwd");
  Shape s;
  dsa_status st = make_shape(p, &s);
  if (st != DSA_OK) return st;
  if (is_empty(p)) return DSA_OK;
  if (q == nullptr || k == nullptr || v == nullptr || (idx == nullptr && s.W > 0) ||
      cnt == nullptr || out == nullptr || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      !aligned16(out))
    return DSA_ERR_INVALID_ARG;
  if ((st = check_ws(s, ws, ws_bytes)) != DSA_OK) return st;
  if ((st = check_device()) != DSA_OK) return st;
  auto hdr = static_cast<dsa::WsHeader*>(ws);
  return run_attention(p, s, q, k, v, idx, cnt, out, lse, hdr, (cudaStream_t)stream);
}

dsa_status dsa_sparse_attn_bwd(const dsa_params* p, const dsa_bf16* q, const dsa_bf16* k,
                               const dsa_bf16* v, const dsa_bf16* out, const float* lse,
                               const dsa_bf16* dout, const int32_t* idx, const int32_t* cnt,
                               dsa_bf16* dq, dsa_bf16* dk, dsa_bf16* dv, void* ws, size_t ws_bytes,
                               void* stream) {
  NvtxRange nvtx("dsa_sparse_attn_bwd");
  Shape s;
  dsa_status st = make_shape(p, &s);
  if (st != DSA_OK) return st;
  if (is_empty(p)) return DSA_OK;
  const void* need16[] = {q, k, v, out, dout, dq, dk, dv};
  for (const void* ptr : need16)
    if (ptr == nullptr || !aligned16(ptr)) return DSA_ERR_INVALID_ARG;
  if (lse == nullptr || !aligned16(lse) || cnt == nullptr || (idx == nullptr && s.W > 0))
    return DSA_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned16(ws) || ws_bytes < dsa::bwd_ws_layout(s).total) return DSA_ERR_WORKSPACE;
  if ((st = check_device()) != DSA_OK) return st;
  const bool tc_ok = dsa::attn_bwd_tc_supported(s);
  if (p->attn_kernel == DSA_ATTN_TCGEN05 && !tc_ok) return DSA_ERR_UNSUPPORTED;
  const bool use_tc = tc_ok && p->attn_kernel != DSA_ATTN_MMA_SYNC;
  return from_cuda(dsa::launch_attn_bwd(
      s, reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(k),
      reinterpret_cast<const __nv_bfloat16*>(v), reinterpret_cast<const __nv_bfloat16*>(out), lse,
      reinterpret_cast<const __nv_bfloat16*>(dout), idx, cnt, reinterpret_cast<__nv_bfloat16*>(dq),
      reinterpret_cast<__nv_bfloat16*>(dk), reinterpret_cast<__nv_bfloat16*>(dv), ws, use_tc,
      (cudaStream_t)stream));
}

dsa_status dsa_forward(const dsa_params* p, const dsa_bf16* q, const dsa_bf16* k, const dsa_bf16* v,
                       dsa_bf16* out, float* lse, int32_t* idx, int32_t* cnt, void* ws,
                       size_t ws_bytes, void* stream) {
  NvtxRange nvtx("dsa_forward");
  Shape s;
  dsa_status st = make_shape(p, &s);
  if (st != DSA_OK) return st;
  if (is_empty(p)) return DSA_OK;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || !aligned16(q) ||
      !aligned16(k) || !aligned16(v) || !aligned16(out))
    return DSA_ERR_INVALID_ARG;
  // idx may be NULL alongside a caller cnt only when rows hold no entries (W == 0)
  if (cnt == nullptr && idx != nullptr) return DSA_ERR_INVALID_ARG;
  if (cnt != nullptr && idx == nullptr && s.W > 0) return DSA_ERR_INVALID_ARG;
  if ((st = check_ws(s, ws, ws_bytes)) != DSA_OK) return st;
  if ((st = check_device()) != DSA_OK) return st;
  const Layout L = layout(s);
  char* base = static_cast<char*>(ws);
  auto hdr = reinterpret_cast<dsa::WsHeader*>(base);
  if (cnt == nullptr) {
    idx = reinterpret_cast<int32_t*>(base + L.idx);
    cnt = reinterpret_cast<int32_t*>(base + L.cnt);
  }
  cudaStream_t cs = (cudaStream_t)stream;
  if ((st = run_selection(p, s, q, k, idx, cnt, ws, cs)) != DSA_OK) return st;
  return run_attention(p, s, q, k, v, idx, cnt, out, lse, hdr, cs);
}

dsa_status dsa_pool_keys(const dsa_params* p, const dsa_bf16* k, float* kp, int j_begin, int j_end,
                         void* stream) {
  NvtxRange nvtx("dsa_pool_keys");
  Shape s;
  dsa_status st = make_shape(p, &s);
  if (st != DSA_OK) return st;
  if (is_empty(p)) return DSA_OK;
  if (j_begin < 0 || j_end < j_begin || j_end > s.nb) return DSA_ERR_INVALID_ARG;
  if (j_end == j_begin) return DSA_OK;
  if (k == nullptr || kp == nullptr || !aligned16(k) || !aligned16(kp)) return DSA_ERR_INVALID_ARG;
  if ((st = check_device()) != DSA_OK) return st;
  return from_cuda(dsa::launch_pool_range(s, reinterpret_cast<const __nv_bfloat16*>(k), kp, j_begin,
                                          j_end, (cudaStream_t)stream));
}

dsa_status dsa_decode_fwd(const dsa_params* p, const dsa_bf16* q, const dsa_bf16* k,
                          const dsa_bf16* v, const float* kp, int length, dsa_bf16* out, float* lse,
                          int32_t* idx, int32_t* cnt, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx("dsa_decode_fwd");
  Shape s;
  dsa_status st = make_shape(p, &s);
  if (st != DSA_OK) return st;
  if (is_empty(p)) return DSA_OK;
  if (length < 1 || length > s.N) return DSA_ERR_INVALID_ARG;
  if (q == nullptr || k == nullptr || v == nullptr || kp == nullptr || out == nullptr ||
      !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(kp))
    return DSA_ERR_INVALID_ARG;
  if ((idx == nullptr) != (cnt == nullptr) && !(idx == nullptr && s.W == 0)) return DSA_ERR_INVALID_ARG;
  if (ws == nullptr || !aligned16(ws) || ws_bytes < dsa::decode_ws_layout(s).total)
    return DSA_ERR_WORKSPACE;
  if ((st = check_device()) != DSA_OK) return st;
  return from_cuda(dsa::launch_decode(
      s, budgets(p), reinterpret_cast<const __nv_bfloat16*>(q),
      reinterpret_cast<const __nv_bfloat16*>(k), reinterpret_cast<const __nv_bfloat16*>(v), kp,
      length, reinterpret_cast<__nv_bfloat16*>(out), lse, idx, cnt,
      ws, (cudaStream_t)stream));
}

dsa_status dsa_check_status(void* ws, void* stream) {
  if (ws == nullptr || !aligned16(ws)) return DSA_ERR_WORKSPACE;
  cudaStream_t cs = (cudaStream_t)stream;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return DSA_ERR_CUDA;
  int flag = 0;
  if (cudaMemcpy(&flag, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (flag != 0) {
    if (cudaMemset(ws, 0, 4 * sizeof(int)) != cudaSuccess) return DSA_ERR_CUDA;
  }
  return (dsa_status)flag;
}

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARG: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape or device";
    case DSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case DSA_ERR_CUDA: return "CUDA runtime or launch error";
    case DSA_ERR_DEVICE_TIMEOUT: return "a bounded wait on the device gave up";
    case DSA_ERR_DEVICE_BOUNDS: return "a kernel met an index out of range";
  }
  return "unknown status";
}

}  // extern "C"
