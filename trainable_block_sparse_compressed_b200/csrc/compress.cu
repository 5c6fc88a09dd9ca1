// compress.cu -- compressed keys: the mean of every 32-token key window, one
// window every 16 tokens (InfLLM-V2 skill write-up, Core Concept: the
// compressed pattern aggregates tokens hierarchically; window 32, stride 16
// are the method's settings).
//
// HBM-bound.  One thread owns 8 consecutive channels (16 bytes) of one
// (batch, window, kv head): it issues the window's 32 row loads as 128-bit
// read-only loads, sums them in fp32 in token order and stores the mean as
// the bf16 pair hi + lo (see common.cuh).  The 32 threads of a warp cover the 16
// channel chunks of Hkv = 2 heads, i.e. one contiguous 512-byte token row, so
// every load instruction is fully coalesced.  A key row is read by two
// windows; the second read hits L2.
#include "common.cuh"

namespace infllmv2 {
namespace {

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4& v) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __bfloat1622float2(h[k]);
    acc[2 * k] += f.x;
    acc[2 * k + 1] += f.y;
  }
}

// K: [B, T, Hkv, 128]  ->  Kc: [B, n_c, Hkv, 2, 128] (hi, lo planes).
__global__ void __launch_bounds__(256) compress_keys_kernel(const __nv_bfloat16* __restrict__ K,
                                                            __nv_bfloat16* __restrict__ Kc,
                                                            int B, int T, int Hkv, int n_c) {
  const int64_t total = static_cast<int64_t>(B) * n_c * Hkv * 16;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx & 15);
    int64_t rest = idx >> 4;
    const int g = static_cast<int>(rest % Hkv);
    rest /= Hkv;
    const int j = static_cast<int>(rest % n_c);
    const int b = static_cast<int>(rest / n_c);
    const int64_t row_stride = static_cast<int64_t>(Hkv) * kHeadDim;  // elements per token
    const __nv_bfloat16* src =
        K + (static_cast<int64_t>(b) * T + static_cast<int64_t>(j) * kCmpStride) * row_stride +
        static_cast<int64_t>(g) * kHeadDim + 8 * c;
    uint4 v[kCmpKernel];
#pragma unroll
    for (int i = 0; i < kCmpKernel; ++i)
      v[i] = __ldg(reinterpret_cast<const uint4*>(src + i * row_stride));
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < kCmpKernel; ++i) add_bf16x8(acc, v[i]);
    const float inv = 1.0f / kCmpKernel;  // exact power of two
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] *= inv;
    store_kc_pair(acc, Kc + ((static_cast<int64_t>(b) * n_c + j) * Hkv + g) * kKcRow + 8 * c);
  }
}

}  // namespace

int launch_compress_keys(const Geometry& g, const void* K, void* Kc, int /*kv_rows_total*/,
                         cudaStream_t st) {
  if (g.n_c == 0 || g.B == 0) return INFLLMV2_OK;
  const int64_t total = static_cast<int64_t>(g.B) * g.n_c * g.Hkv * 16;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sm_count()) * 16;
  if (blocks > cap) blocks = cap;
  compress_keys_kernel<<<static_cast<unsigned>(blocks), threads, 0, st>>>(
      static_cast<const __nv_bfloat16*>(K), static_cast<__nv_bfloat16*>(Kc), g.B, g.T, g.Hkv,
      g.n_c);
  return cudaGetLastError() == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

}  // namespace infllmv2
