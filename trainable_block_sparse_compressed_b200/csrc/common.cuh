// common.cuh -- shared definitions of the InfLLM-V2 CUDA library: problem
// geometry, the device status word, launch plumbing and the kernel launchers
// that api.cu calls.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "../../include/infllmv2.h"

namespace infllmv2 {

constexpr int kHeadDim = 128;     // d
constexpr int kBlock = 64;        // key block size
constexpr int kCmpKernel = 32;    // compression window
constexpr int kCmpStride = 16;    // compression stride
constexpr int kMaxTopk = 256;
// A compressed key is stored as an unevaluated pair of bf16 planes,
// Kc = hi + lo with hi = RNE(mean), lo = RNE(mean - hi) (about 17 significant
// bits), laid out [B, n_c, Hkv, 2, d]: a single bf16 rounding of the mean
// moves block scores by up to ~1e-2 relative, far more than the selection
// tolerates.
constexpr int kKcRow = 2 * kHeadDim;  // elements per (window, kv head)

// Everything a kernel needs about one call, resolved on the host.
struct Geometry {
  int B, T, Hq, Hkv, G;   // G = Hq / Hkv; T: tokens of the sequence (keys)
  int q0, Tq;             // the queries are tokens q0 .. q0+Tq-1 (prefill: 0, T)
  int n_c;                // compressed rows of T tokens
  int topk, n_init, n_local;
  float scale;            // softmax scale
  float scale_log2;       // scale * log2(e)
};

__host__ __device__ inline int num_compressed(int T) {
  return T < kCmpKernel ? 0 : (T - kCmpKernel) / kCmpStride + 1;
}

// Windows j with 16j + 31 <= t.
__host__ __device__ inline int visible_windows(int t) {
  return t < kCmpKernel - 1 ? 0 : (t - (kCmpKernel - 1)) / kCmpStride + 1;
}

// Offset (in floats) of query row t's block scores inside one (b, g) slab of
// the selection workspace: rows are packed causally, row t holds t/64 + 1
// scores.  sum_{t'<t} (t'/64 + 1) = 32 c (c + 1) + r (c + 1), c = t/64, r = t%64.
__host__ __device__ inline int64_t score_row_offset(int64_t t) {
  const int64_t c = t / kBlock, r = t % kBlock;
  return 32 * c * (c + 1) + r * (c + 1);
}

// Per-call device context: status word and wait limit.
struct DevCtx {
  int* status;          // device pointer to the status word of this device
  uint64_t wait_ns;     // bounded-wait limit
};

__device__ __forceinline__ void report_status(int* status, int bit) {
  atomicOr(status, bit);
}

// Index checks of the bounds-checked build (compiled with -DINFLLMV2_CHECKS,
// libinfllmv2_checks.so): a failed check sets INFLLMV2_STATUS_CHECK and the
// caller skips the access.  In the regular build the check is the constant
// true and generates no code.
#ifdef INFLLMV2_CHECKS
#define INFLLMV2_CHECK(status, cond) \
  ((cond) ? true : (report_status((status), INFLLMV2_STATUS_CHECK), false))
#else
#define INFLLMV2_CHECK(status, cond) true
#endif

// Stores 8 channels of a compressed key (fp32 means) as the (hi, lo) pair:
// hi at dst[0..7], lo at dst[kHeadDim .. kHeadDim+7].
__device__ __forceinline__ void store_kc_pair(const float (&m)[8], __nv_bfloat16* dst) {
  uint4 hi, lo;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&hi);
  __nv_bfloat162* l = reinterpret_cast<__nv_bfloat162*>(&lo);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    h[k] = __floats2bfloat162_rn(m[2 * k], m[2 * k + 1]);
    const float2 f = __bfloat1622float2(h[k]);
    l[k] = __floats2bfloat162_rn(m[2 * k] - f.x, m[2 * k + 1] - f.y);
  }
  *reinterpret_cast<uint4*>(dst) = hi;
  *reinterpret_cast<uint4*>(dst + kHeadDim) = lo;
}

// Host helpers (api.cu).
cudaError_t get_dev_ctx(DevCtx* ctx);
int sm_count();

// Raises a kernel's dynamic shared memory limit to `bytes` on the current
// device, once per device (`done` holds one bit per device id < 64; others
// are set on every call, which is harmless).
template <typename F>
inline int set_smem_limit(F* func, size_t bytes, std::atomic<uint64_t>& done) {
  int d = -1;
  if (cudaGetDevice(&d) != cudaSuccess) return INFLLMV2_ERR_CUDA;
  const uint64_t bit = (d >= 0 && d < 64) ? (uint64_t{1} << d) : 0;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return INFLLMV2_OK;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes)) != cudaSuccess)
    return INFLLMV2_ERR_CUDA;
  done.fetch_or(bit, std::memory_order_release);
  return INFLLMV2_OK;
}

// Tensor maps (tma.cpp).
int make_tmap_bf16_4d(CUtensorMap* map, const void* base, const uint64_t dims[4],
                      const uint64_t strides_bytes[3], const uint32_t box[4]);

// Kernel launchers (one per .cu file); each returns an INFLLMV2_* code.
int launch_compress_keys(const Geometry& g, const void* K, void* Kc, int kv_rows_total,
                         cudaStream_t st);
int launch_score_blocks(const Geometry& g, const void* Q, const void* Kc, float* scores,
                        const DevCtx& ctx, cudaStream_t st);
int launch_topk(const Geometry& g, const float* scores, int32_t* idx, cudaStream_t st);
// K/V block tiles (pack.cu): bytes for both tensors, and the repacking launch.
size_t packed_kv_bytes(const Geometry& g);
int launch_pack_kv(const Geometry& g, const void* K, const void* V, void* packed,
                   cudaStream_t st);
// Sparse attention over selected blocks, one work item per query token.
// packed: K/V tiles from launch_pack_kv, or null to gather from K and V.
int launch_sparse_attn(const Geometry& g, const void* Q, const void* K, const void* V,
                       const int32_t* idx, void* O, float* lse, const void* packed,
                       const DevCtx& ctx, cudaStream_t st);
// Query-tile attention (tile_attn.cu): dense causal, the union of the tile's
// selected blocks, or the compressed windows.
bool union_supported(const Geometry& g);
size_t union_lists_ws_bytes(const Geometry& g);  // the union lists and their counts
size_t union_ws_bytes(const Geometry& g);        // the lists, then packed K/V tiles
// Union lists of the query tiles of g (in ws, union_ws_bytes(g) bytes):
// per tile, `stride` slots of (block, token mask) ascending, and the counts.
int launch_union_build(const Geometry& g, const int32_t* idx, void* ws, const uint2** ulist,
                       const int32_t** ucount, int* stride, cudaStream_t st);
int launch_dense_tile(const Geometry& g, const void* Q, const void* K, const void* V, void* O,
                      float* lse, const DevCtx& ctx, cudaStream_t st);
int launch_union_tile(const Geometry& g, const void* Q, const void* K, const void* V,
                      const int32_t* idx, void* O, float* lse, void* ws, const DevCtx& ctx,
                      cudaStream_t st);
int launch_compressed_tile(const Geometry& g, const void* Q, const void* Kc, const void* Vc,
                           void* O, float* lse, const DevCtx& ctx, cudaStream_t st);
// The fp32 validation build of the forward (fp32_path.cu): dense, or compress
// into Kc32 -> block scores into `scores` -> top-k into idx -> attention.
int launch_forward_f32(const Geometry& g, const void* Q, const void* K, const void* V, void* O,
                       float* lse, float* Kc32, int32_t* idx, float* scores, bool dense,
                       cudaStream_t st);
// Backward of the block-sparse attention with the selection fixed (attn_bwd.cu).
size_t bwd_ws_bytes(const Geometry& g);
int launch_sparse_bwd(const Geometry& g, const void* Q, const void* K, const void* V,
                      const int32_t* idx, const void* O, const float* lse, const void* dO, float* dQ,
                      float* dK, float* dV, void* ws, const DevCtx& ctx, cudaStream_t st);
// Decode (decode.cu); g.T is the cache capacity.
size_t decode_ws_bytes(const Geometry& g);
int launch_decode_step(const Geometry& g, const void* q, const void* k_new, const void* v_new,
                       void* K_cache, void* V_cache, void* Kc_cache, int32_t* seqlens, void* O,
                       float* lse, int32_t* idx_out, void* ws, const DevCtx& ctx,
                       cudaStream_t st);

}  // namespace infllmv2
