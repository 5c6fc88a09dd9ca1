// api.cu -- the C ABI declared in include/infllmv2.h: argument validation,
// the per-device status word, and the order in which each entry point
// enqueues its kernels.
#include <math.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "sm100.cuh"

namespace infllmv2 {

// The library's only global device state: one status word per device (each
// device that loads the module gets its own copy of this variable).
__device__ int g_status_word;

namespace {

std::atomic<uint64_t> g_wait_ns{2000000000ull};  // 2 s

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_status_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

int current_device() {
  int d = 0;
  if (cudaGetDevice(&d) != cudaSuccess) return -1;
  return d;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

cudaError_t get_dev_ctx(DevCtx* ctx) {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[d]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_status_word);
    if (e != cudaSuccess) return e;
    g_status_ptr[d] = static_cast<int*>(p);
  }
  ctx->status = g_status_ptr[d];
  ctx->wait_ns = g_wait_ns.load();
  return cudaSuccess;
}

int sm_count() {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sm_count[d]) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d);
    g_sm_count[d] = n > 0 ? n : 148;
  }
  return g_sm_count[d];
}

namespace {

// Checks the configuration shared by every entry point; fills `g`.
int validate(const infllmv2_params* p, bool needs_topk, Geometry* g) {
  if (!p) return INFLLMV2_ERR_INVALID_ARG;
  if (p->B < 0 || p->T < 0 || p->Hq <= 0 || p->Hkv <= 0) return INFLLMV2_ERR_INVALID_ARG;
  if (p->Hq % p->Hkv != 0) return INFLLMV2_ERR_INVALID_ARG;
  if (p->head_dim != kHeadDim || p->block_size != kBlock || p->cmp_kernel != kCmpKernel ||
      p->cmp_stride != kCmpStride || p->causal != 1)
    return INFLLMV2_ERR_UNSUPPORTED;
  const int G = p->Hq / p->Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16) return INFLLMV2_ERR_UNSUPPORTED;
  if (!(p->scale >= 0.f) || isinf(p->scale)) return INFLLMV2_ERR_INVALID_ARG;
  if (needs_topk) {
    if (p->topk < 1 || p->topk > kMaxTopk || p->n_init < 0 || p->n_local < 0 ||
        p->n_init + p->n_local > p->topk)
      return INFLLMV2_ERR_INVALID_ARG;
  }
  if (static_cast<int64_t>(p->T) > (1 << 22)) return INFLLMV2_ERR_UNSUPPORTED;
  g->B = p->B;
  g->T = p->T;
  g->q0 = 0;
  g->Tq = p->T;
  g->Hq = p->Hq;
  g->Hkv = p->Hkv;
  g->G = G;
  g->n_c = num_compressed(p->T);
  g->topk = p->topk;
  g->n_init = p->n_init;
  g->n_local = p->n_local;
  g->scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf(static_cast<float>(kHeadDim));
  g->scale_log2 = g->scale * 1.4426950408889634f;
  return INFLLMV2_OK;
}

bool empty(const Geometry& g) { return g.B == 0 || g.T == 0; }

// One warp waits on an mbarrier that nothing arrives on; the bounded wait
// expires, reports INFLLMV2_STATUS_TIMEOUT and the kernel returns.
__global__ void selftest_wait_kernel(DevCtx ctx) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, ctx.wait_ns))
    report_status(ctx.status, INFLLMV2_STATUS_TIMEOUT);
}

int check_ptrs(std::initializer_list<const void*> ptrs) {
  for (const void* q : ptrs) {
    if (!q) return INFLLMV2_ERR_INVALID_ARG;
    if (!aligned16(q)) return INFLLMV2_ERR_UNSUPPORTED;
  }
  return INFLLMV2_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Block scores of the query rows q0 .. q0+Tq-1 (causally packed).
size_t select_ws_bytes(const Geometry& g) {
  return static_cast<size_t>(g.B) * g.Hkv *
         static_cast<size_t>(score_row_offset(g.q0 + g.Tq) - score_row_offset(g.q0)) *
         sizeof(float);
}

// Block selection holds a row's block scores in registers: sequences of at
// most INFLLMV2_MAX_SELECT_T tokens (4096 blocks); checked before any launch.
int check_select_size(const Geometry& g) {
  return g.T > INFLLMV2_MAX_SELECT_T ? INFLLMV2_ERR_UNSUPPORTED : INFLLMV2_OK;
}

// Workspace of the block-sparse attention: the union lists of the query-tile
// schedule (groups of 4, 8 or 16 heads), else the packed K/V tiles of the
// per-token schedule.
size_t attn_ws_bytes(const Geometry& g) {
  return union_supported(g) ? union_ws_bytes(g) : packed_kv_bytes(g);
}

// Enqueues the block-sparse attention: the query-tile schedule over each
// tile's union of selected blocks when the group allows it and the workspace
// holds its lists; else one work item per query token, gathering from packed
// K/V tiles when the workspace holds them, from K and V directly otherwise.
int enqueue_sparse(const Geometry& g, const void* Q, const void* K, const void* V,
                   const int32_t* idx, void* O, float* lse, void* ws, size_t ws_bytes,
                   bool per_token, const DevCtx& ctx, cudaStream_t st) {
  if (!per_token && union_supported(g) && ws && ws_bytes >= union_ws_bytes(g))
    return launch_union_tile(g, Q, K, V, idx, O, lse, ws, ctx, st);
  const bool pack = ws && ws_bytes >= packed_kv_bytes(g);
  if (pack)
    if (int e = launch_pack_kv(g, K, V, ws, st)) return e;
  return launch_sparse_attn(g, Q, K, V, idx, O, lse, pack ? ws : nullptr, ctx, st);
}

// validate() plus the query range of a prefill chunk.
int validate_chunk(const infllmv2_params* p, int32_t q_offset, int32_t q_len, Geometry* g) {
  if (int e = validate(p, true, g)) return e;
  if (q_offset < 0 || q_len < 0 || static_cast<int64_t>(q_offset) + q_len != p->T)
    return INFLLMV2_ERR_INVALID_ARG;
  g->q0 = q_offset;
  g->Tq = q_len;
  return INFLLMV2_OK;
}

int ctx_or_error(DevCtx* ctx) {
  return get_dev_ctx(ctx) == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

size_t chunk_ws_bytes(const Geometry& g, bool dense) {
  return dense ? 0 : align256(select_ws_bytes(g)) + attn_ws_bytes(g);
}

// The chunk's kernels: dense attention, or scoring -> top-k -> sparse
// attention.  Arguments already checked.
int enqueue_chunk(const Geometry& g, bool dense, const void* Q, const void* K, const void* V,
                  const void* Kc, void* O, float* lse, int32_t* idx, void* ws, size_t ws_bytes,
                  const DevCtx& ctx, cudaStream_t st) {
  if (dense) return launch_dense_tile(g, Q, K, V, O, lse, ctx, st);
  const size_t sel = align256(select_ws_bytes(g));
  if (ws_bytes < sel) return INFLLMV2_ERR_WORKSPACE;
  if (int e = launch_score_blocks(g, Q, Kc, static_cast<float*>(ws), ctx, st)) return e;
  if (int e = launch_topk(g, static_cast<float*>(ws), idx, st)) return e;
  return enqueue_sparse(g, Q, K, V, idx, O, lse, static_cast<uint8_t*>(ws) + sel, ws_bytes - sel,
                        false, ctx, st);
}

// A packed batch of sequences: cu_seqlens_q / _k (host) hold n_seqs + 1
// ascending offsets from 0; every sequence's query count is at most its key
// count.  *need: the largest workspace any one sequence needs (they run one
// after another on the stream and share it).
int check_varlen(const infllmv2_params* p, int32_t n_seqs, const int32_t* cu_q,
                 const int32_t* cu_k, size_t* need) {
  if (!p || n_seqs < 0) return INFLLMV2_ERR_INVALID_ARG;
  if (n_seqs > 0 && (!cu_q || !cu_k)) return INFLLMV2_ERR_INVALID_ARG;
  if (n_seqs > 0 && (cu_q[0] != 0 || cu_k[0] != 0)) return INFLLMV2_ERR_INVALID_ARG;
  *need = 0;
  for (int i = 0; i < n_seqs; ++i) {
    const int64_t ql = static_cast<int64_t>(cu_q[i + 1]) - cu_q[i];
    const int64_t kl = static_cast<int64_t>(cu_k[i + 1]) - cu_k[i];
    if (ql < 0 || kl < 0 || ql > kl) return INFLLMV2_ERR_INVALID_ARG;
    infllmv2_params pi = *p;
    pi.B = 1;
    pi.T = static_cast<int32_t>(kl);
    Geometry g;
    if (int e = validate_chunk(&pi, static_cast<int32_t>(kl - ql), static_cast<int32_t>(ql), &g))
      return e;
    const bool dense = kl <= p->switch_threshold;
    if (!dense && ql > 0)
      if (int e = check_select_size(g)) return e;
    const size_t w = ql > 0 ? chunk_ws_bytes(g, dense) : 0;
    if (w > *need) *need = w;
  }
  return INFLLMV2_OK;
}

}  // namespace
}  // namespace infllmv2

using namespace infllmv2;

extern "C" {

int infllmv2_version(void) { return 100; }

int32_t infllmv2_num_compressed(int32_t T) { return num_compressed(T); }

const char* infllmv2_strerror(int code) {
  switch (code) {
    case INFLLMV2_OK: return "ok";
    case INFLLMV2_ERR_INVALID_ARG: return "invalid argument";
    case INFLLMV2_ERR_UNSUPPORTED: return "unsupported configuration or misaligned pointer";
    case INFLLMV2_ERR_CUDA: return "CUDA call failed";
    case INFLLMV2_ERR_TIMEOUT: return "device wait limit exceeded";
    case INFLLMV2_ERR_WORKSPACE: return "workspace too small";
    case INFLLMV2_ERR_DEVICE_CHECK: return "device-side argument check failed";
    default: return "unknown error";
  }
}

void infllmv2_set_wait_limit(int64_t ns) {
  g_wait_ns.store(ns < 0 ? 0ull : static_cast<uint64_t>(ns));
}

size_t infllmv2_workspace_bytes(const infllmv2_params* p, int32_t op) {
  Geometry g;
  // the dense forward takes no top-k parameters (as infllmv2_dense_attn)
  const bool dense_fwd = (op == INFLLMV2_OP_FORWARD || op == INFLLMV2_OP_FORWARD_FP32) && p &&
                         p->T <= p->switch_threshold;
  if (validate(p, !dense_fwd, &g) != INFLLMV2_OK) return SIZE_MAX;
  switch (op) {
    case INFLLMV2_OP_SELECT:
      return check_select_size(g) ? SIZE_MAX : select_ws_bytes(g);
    case INFLLMV2_OP_FORWARD:
      if (dense_fwd) return 0;
      return check_select_size(g) ? SIZE_MAX : align256(select_ws_bytes(g)) + attn_ws_bytes(g);
    case INFLLMV2_OP_DECODE:
      return g.T > INFLLMV2_MAX_DECODE_T ? SIZE_MAX : decode_ws_bytes(g);
    case INFLLMV2_OP_ATTN: return attn_ws_bytes(g);
    case INFLLMV2_OP_ATTN_PER_TOKEN: return packed_kv_bytes(g);
    case INFLLMV2_OP_BACKWARD:
      return union_supported(g) && !check_select_size(g) ? bwd_ws_bytes(g) : SIZE_MAX;
    case INFLLMV2_OP_FORWARD_FP32:
      if (dense_fwd) return 0;
      return check_select_size(g) ? SIZE_MAX : select_ws_bytes(g);
    default: return SIZE_MAX;
  }
}

int infllmv2_compress_keys(const infllmv2_params* p, const void* K, void* Kc, void* stream) {
  Geometry g;
  if (int e = validate(p, false, &g)) return e;
  if (empty(g) || g.n_c == 0) return INFLLMV2_OK;
  if (int e = check_ptrs({K, Kc})) return e;
  return launch_compress_keys(g, K, Kc, 0, static_cast<cudaStream_t>(stream));
}

int infllmv2_select_blocks(const infllmv2_params* p, const void* Q, const void* Kc, int32_t* idx,
                           void* ws, size_t ws_bytes, void* stream) {
  Geometry g;
  if (int e = validate(p, true, &g)) return e;
  if (int e = check_select_size(g)) return e;
  if (empty(g)) return INFLLMV2_OK;
  if (int e = check_ptrs({Q, idx, ws})) return e;
  if (g.n_c > 0)
    if (int e = check_ptrs({Kc})) return e;
  if (ws_bytes < select_ws_bytes(g)) return INFLLMV2_ERR_WORKSPACE;
  DevCtx ctx;
  if (int e = ctx_or_error(&ctx)) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  float* scores = static_cast<float*>(ws);
  if (int e = launch_score_blocks(g, Q, Kc, scores, ctx, st)) return e;
  return launch_topk(g, scores, idx, st);
}

int infllmv2_sparse_attn(const infllmv2_params* p, const void* Q, const void* K, const void* V,
                         const int32_t* idx, void* O, float* lse, void* ws, size_t ws_bytes,
                         void* stream) {
  Geometry g;
  if (int e = validate(p, true, &g)) return e;
  if (empty(g)) return INFLLMV2_OK;
  if (int e = check_ptrs({Q, K, V, idx, O, lse})) return e;
  if (ws && !aligned16(ws)) return INFLLMV2_ERR_UNSUPPORTED;
  DevCtx ctx;
  if (int e = ctx_or_error(&ctx)) return e;
  return enqueue_sparse(g, Q, K, V, idx, O, lse, ws, ws_bytes, false, ctx,
                        static_cast<cudaStream_t>(stream));
}

int infllmv2_sparse_attn_per_token(const infllmv2_params* p, const void* Q, const void* K,
                                   const void* V, const int32_t* idx, void* O, float* lse,
                                   void* ws, size_t ws_bytes, void* stream) {
  Geometry g;
  if (int e = validate(p, true, &g)) return e;
  if (empty(g)) return INFLLMV2_OK;
  if (int e = check_ptrs({Q, K, V, idx, O, lse})) return e;
  if (ws && !aligned16(ws)) return INFLLMV2_ERR_UNSUPPORTED;
  DevCtx ctx;
  if (int e = ctx_or_error(&ctx)) return e;
  return enqueue_sparse(g, Q, K, V, idx, O, lse, ws, ws_bytes, true, ctx,
                        static_cast<cudaStream_t>(stream));
}

int infllmv2_sparse_attn_backward(const infllmv2_params* p, const void* Q, const void* K,
                                  const void* V, const int32_t* idx, const void* O,
                                  const float* lse, const void* dO, float* dQ, float* dK,
                                  float* dV, void* ws, size_t ws_bytes, void* stream) {
  Geometry g;
  if (int e = validate(p, true, &g)) return e;
  if (!union_supported(g)) return INFLLMV2_ERR_UNSUPPORTED;
  if (int e = check_select_size(g)) return e;
  if (empty(g)) return INFLLMV2_OK;
  if (int e = check_ptrs({Q, K, V, idx, O, lse, dO, dQ, dK, dV, ws})) return e;
  if (ws_bytes < bwd_ws_bytes(g)) return INFLLMV2_ERR_WORKSPACE;
  DevCtx ctx;
  if (int e = ctx_or_error(&ctx)) return e;
  return launch_sparse_bwd(g, Q, K, V, idx, O, lse, dO, dQ, dK, dV, ws, ctx,
                           static_cast<cudaStream_t>(stream));
}

int infllmv2_dense_attn(const infllmv2_params* p, const void* Q, const void* K, const void* V,
                        void* O, float* lse, void* ws, size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  Geometry g;
  if (int e = validate(p, false, &g)) return e;
  if (empty(g)) return INFLLMV2_OK;
  if (int e = check_ptrs({Q, K, V, O, lse})) return e;
  DevCtx ctx;
  if (int e = ctx_or_error(&ctx)) return e;
  return launch_dense_tile(g, Q, K, V, O, lse, ctx, static_cast<cudaStream_t>(stream));
}

int infllmv2_compressed_attn(const infllmv2_params* p, const void* Q, const void* Kc,
                             const void* Vc, void* O, float* lse, void* stream) {
  Geometry g;
  if (int e = validate(p, false, &g)) return e;
  if (empty(g)) return INFLLMV2_OK;
  if (int e = check_ptrs({Q, O, lse})) return e;
  if (g.n_c > 0)
    if (int e = check_ptrs({Kc, Vc})) return e;
  DevCtx ctx;
  if (int e = ctx_or_error(&ctx)) return e;
  return launch_compressed_tile(g, Q, Kc, Vc, O, lse, ctx, static_cast<cudaStream_t>(stream));
}

int infllmv2_forward(const infllmv2_params* p, const void* Q, const void* K, const void* V,
                     void* O, float* lse, void* Kc_ws, int32_t* idx_ws, int32_t* path_used,
                     void* ws, size_t ws_bytes, void* stream) {
  if (!p) return INFLLMV2_ERR_INVALID_ARG;
  const bool dense = p->T <= p->switch_threshold;
  if (path_used) *path_used = dense ? INFLLMV2_PATH_DENSE : INFLLMV2_PATH_SPARSE;
  if (dense) return infllmv2_dense_attn(p, Q, K, V, O, lse, ws, ws_bytes, stream);
  Geometry g;
  if (int e = validate(p, true, &g)) return e;
  if (int e = check_select_size(g)) return e;
  if (empty(g)) return INFLLMV2_OK;
  // workspace: block scores of the selection, then the attention's
  const size_t sel = align256(select_ws_bytes(g));
  if (ws_bytes < sel) return INFLLMV2_ERR_WORKSPACE;
  if (g.n_c > 0)
    if (int e = infllmv2_compress_keys(p, K, Kc_ws, stream)) return e;
  if (int e = infllmv2_select_blocks(p, Q, Kc_ws, idx_ws, ws, ws_bytes, stream)) return e;
  return infllmv2_sparse_attn(p, Q, K, V, idx_ws, O, lse, static_cast<uint8_t*>(ws) + sel,
                              ws_bytes - sel, stream);
}

int infllmv2_forward_fp32(const infllmv2_params* p, const void* Q, const void* K, const void* V,
                          float* O, float* lse, float* Kc32_ws, int32_t* idx_ws,
                          int32_t* path_used, void* ws, size_t ws_bytes, void* stream) {
  if (!p) return INFLLMV2_ERR_INVALID_ARG;
  const bool dense = p->T <= p->switch_threshold;
  Geometry g;
  if (int e = validate(p, !dense, &g)) return e;
  if (!dense)
    if (int e = check_select_size(g)) return e;
  if (path_used) *path_used = dense ? INFLLMV2_PATH_DENSE : INFLLMV2_PATH_SPARSE;
  if (empty(g)) return INFLLMV2_OK;
  if (int e = check_ptrs({Q, K, V, O, lse})) return e;
  if (!dense) {
    if (int e = check_ptrs({idx_ws, ws})) return e;
    if (g.n_c > 0)
      if (int e = check_ptrs({Kc32_ws})) return e;
    if (ws_bytes < select_ws_bytes(g)) return INFLLMV2_ERR_WORKSPACE;
  }
  return launch_forward_f32(g, Q, K, V, O, lse, Kc32_ws, idx_ws, static_cast<float*>(ws), dense,
                            static_cast<cudaStream_t>(stream));
}

size_t infllmv2_prefill_chunk_workspace_bytes(const infllmv2_params* p, int32_t q_offset,
                                              int32_t q_len) {
  Geometry g;
  if (validate_chunk(p, q_offset, q_len, &g) != INFLLMV2_OK) return SIZE_MAX;
  if (p->T <= p->switch_threshold) return 0;
  return check_select_size(g) ? SIZE_MAX : chunk_ws_bytes(g, false);
}

int infllmv2_prefill_chunk(const infllmv2_params* p, int32_t q_offset, int32_t q_len,
                           const void* Q, const void* K, const void* V, const void* Kc, void* O,
                           float* lse, int32_t* idx, int32_t* path_used, void* ws,
                           size_t ws_bytes, void* stream) {
  Geometry g;
  if (int e = validate_chunk(p, q_offset, q_len, &g)) return e;
  const bool dense = p->T <= p->switch_threshold;
  if (!dense)
    if (int e = check_select_size(g)) return e;
  if (path_used) *path_used = dense ? INFLLMV2_PATH_DENSE : INFLLMV2_PATH_SPARSE;
  if (g.B == 0 || g.Tq == 0) return INFLLMV2_OK;
  if (int e = check_ptrs({Q, K, V, O, lse})) return e;
  if (!dense) {
    if (int e = check_ptrs({idx, ws})) return e;
    if (g.n_c > 0)
      if (int e = check_ptrs({Kc})) return e;
  }
  DevCtx ctx;
  if (int e = ctx_or_error(&ctx)) return e;
  return enqueue_chunk(g, dense, Q, K, V, Kc, O, lse, idx, ws, ws_bytes, ctx,
                       static_cast<cudaStream_t>(stream));
}

size_t infllmv2_prefill_varlen_workspace_bytes(const infllmv2_params* p, int32_t n_seqs,
                                               const int32_t* cu_seqlens_q,
                                               const int32_t* cu_seqlens_k) {
  size_t need = 0;
  if (check_varlen(p, n_seqs, cu_seqlens_q, cu_seqlens_k, &need) != INFLLMV2_OK) return SIZE_MAX;
  return need;
}

int infllmv2_prefill_varlen(const infllmv2_params* p, int32_t n_seqs,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                            const void* Q, const void* K, const void* V, const void* Kc, void* O,
                            float* lse, int32_t* idx, int32_t* path_used, void* ws,
                            size_t ws_bytes, void* stream) {
  size_t need = 0;
  if (int e = check_varlen(p, n_seqs, cu_seqlens_q, cu_seqlens_k, &need)) return e;
  if (n_seqs == 0 || cu_seqlens_q[n_seqs] == 0) return INFLLMV2_OK;
  if (int e = check_ptrs({Q, K, V, O, lse})) return e;
  bool any_sparse = false, any_cmp = false;
  for (int i = 0; i < n_seqs; ++i) {
    const int kl = cu_seqlens_k[i + 1] - cu_seqlens_k[i];
    if (kl > p->switch_threshold && cu_seqlens_q[i + 1] > cu_seqlens_q[i]) {
      any_sparse = true;
      any_cmp |= num_compressed(kl) > 0;
    }
  }
  if (any_sparse)
    if (int e = check_ptrs({idx, ws})) return e;
  if (any_cmp)
    if (int e = check_ptrs({Kc})) return e;
  if (ws_bytes < need) return INFLLMV2_ERR_WORKSPACE;
  DevCtx ctx;
  if (int e = ctx_or_error(&ctx)) return e;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int Hq = p->Hq, Hkv = p->Hkv;
  int64_t cmp_off = 0;  // compressed rows before sequence i
  for (int i = 0; i < n_seqs; ++i) {
    const int q_start = cu_seqlens_q[i], q_len = cu_seqlens_q[i + 1] - q_start;
    const int k_start = cu_seqlens_k[i], k_len = cu_seqlens_k[i + 1] - k_start;
    const bool dense = k_len <= p->switch_threshold;
    if (path_used) path_used[i] = dense ? INFLLMV2_PATH_DENSE : INFLLMV2_PATH_SPARSE;
    infllmv2_params pi = *p;
    pi.B = 1;
    pi.T = k_len;
    Geometry g;
    if (int e = validate_chunk(&pi, k_len - q_len, q_len, &g)) return e;
    if (q_len > 0) {
      const size_t row = static_cast<size_t>(kHeadDim) * sizeof(__nv_bfloat16);
      const uint8_t* Qi = static_cast<const uint8_t*>(Q) + static_cast<size_t>(q_start) * Hq * row;
      uint8_t* Oi = static_cast<uint8_t*>(O) + static_cast<size_t>(q_start) * Hq * row;
      const uint8_t* Ki = static_cast<const uint8_t*>(K) + static_cast<size_t>(k_start) * Hkv * row;
      const uint8_t* Vi = static_cast<const uint8_t*>(V) + static_cast<size_t>(k_start) * Hkv * row;
      const uint8_t* Kci =
          Kc ? static_cast<const uint8_t*>(Kc) + static_cast<size_t>(cmp_off) * Hkv * 2 * row
             : nullptr;
      float* lsei = lse + static_cast<int64_t>(q_start) * Hq;
      int32_t* idxi = idx ? idx + static_cast<int64_t>(q_start) * Hkv * p->topk : nullptr;
      if (int e = enqueue_chunk(g, dense, Qi, Ki, Vi, Kci, Oi, lsei, idxi, ws, ws_bytes, ctx, st))
        return e;
    }
    cmp_off += num_compressed(k_len);
  }
  return INFLLMV2_OK;
}

int infllmv2_decode_step(const infllmv2_params* p, const void* q, const void* k_new,
                         const void* v_new, void* K_cache, void* V_cache, void* Kc_cache,
                         int32_t* seqlens, void* O, float* lse, int32_t* idx_out, void* ws,
                         size_t ws_bytes, void* stream) {
  Geometry g;
  if (int e = validate(p, true, &g)) return e;
  if (g.T > INFLLMV2_MAX_DECODE_T) return INFLLMV2_ERR_UNSUPPORTED;
  if (g.B == 0) return INFLLMV2_OK;
  if (g.T < 1) return INFLLMV2_ERR_INVALID_ARG;
  if (int e = check_ptrs({q, k_new, v_new, K_cache, V_cache, seqlens, O, lse, ws})) return e;
  if (g.n_c > 0)
    if (int e = check_ptrs({Kc_cache})) return e;
  if (idx_out && !aligned16(idx_out)) return INFLLMV2_ERR_UNSUPPORTED;
  if (ws_bytes < decode_ws_bytes(g)) return INFLLMV2_ERR_WORKSPACE;
  DevCtx ctx;
  if (int e = ctx_or_error(&ctx)) return e;
  return launch_decode_step(g, q, k_new, v_new, K_cache, V_cache, Kc_cache, seqlens, O, lse,
                            idx_out, ws, ctx, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

namespace infllmv2 {
namespace {

// Scratch of infllmv2_decode_step_noalloc: a fixed array in every device's
// copy of this module, so neither the caller nor the library allocates.
static __device__ __align__(256) uint8_t g_noalloc_scratch[INFLLMV2_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address must be looked
// up, once per device, with that device current.
int noalloc_scratch(void** out) {
  const int d = current_device();
  if (d < 0 || d >= kMaxDevices) return INFLLMV2_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_ptr[d]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr)
      return INFLLMV2_ERR_CUDA;
    g_noalloc_ptr[d] = ptr;
  }
  *out = g_noalloc_ptr[d];
  return INFLLMV2_OK;
}

}  // namespace
}  // namespace infllmv2

extern "C" {

int infllmv2_decode_step_noalloc(const infllmv2_params* p, const void* q, const void* k_new,
                                 const void* v_new, void* K_cache, void* V_cache,
                                 void* Kc_cache, int32_t* seqlens, void* O, float* lse,
                                 int32_t* idx_out, void* stream) {
  Geometry g;
  if (int e = validate(p, true, &g)) return e;
  if (g.T > INFLLMV2_MAX_DECODE_T) return INFLLMV2_ERR_UNSUPPORTED;
  if (g.B == 0) return INFLLMV2_OK;
  if (g.T < 1) return INFLLMV2_ERR_INVALID_ARG;
  if (int e = check_ptrs({q, k_new, v_new, K_cache, V_cache, seqlens, O, lse})) return e;
  if (g.n_c > 0)
    if (int e = check_ptrs({Kc_cache})) return e;
  if (idx_out && !aligned16(idx_out)) return INFLLMV2_ERR_UNSUPPORTED;
  if (decode_ws_bytes(g) > INFLLMV2_NOALLOC_SCRATCH_BYTES) return INFLLMV2_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (int e = noalloc_scratch(&scratch)) return e;
  DevCtx ctx;
  if (int e = ctx_or_error(&ctx)) return e;
  return launch_decode_step(g, q, k_new, v_new, K_cache, V_cache, Kc_cache, seqlens, O, lse,
                            idx_out, scratch, ctx, static_cast<cudaStream_t>(stream));
}

int infllmv2_selftest_timeout(void* stream) {
  DevCtx ctx;
  if (int e = ctx_or_error(&ctx)) return e;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ctx);
  return cudaGetLastError() == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

int infllmv2_get_status(void* stream, int32_t* status_out) {
  if (!status_out) return INFLLMV2_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return INFLLMV2_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status_word, sizeof(int)) != cudaSuccess) return INFLLMV2_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int)) != cudaSuccess)
    return INFLLMV2_ERR_CUDA;
  *status_out = v;
  return INFLLMV2_OK;
}

}  // extern "C"
