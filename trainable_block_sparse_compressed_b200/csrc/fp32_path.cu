// fp32_path.cu -- the fp32 validation build of the forward path: the same
// steps as the tensor-core path (compressed keys, per-head softmax scores
// summed over the GQA group and max-pooled to 64-token blocks, top-k block
// selection, block-sparse or dense causal attention), every product and sum
// in fp32 on the CUDA cores, compressed keys kept in fp32 and P and O never
// rounded to bf16.  It exists to check the method's arithmetic to ~1e-6
// rather than to bf16 rounding; its speed is not a goal.
//
//   compress_f32 : Kc32[b, j, g, :] = fp32 mean of K[b, 16j .. 16j+31, g, :],
//                  summed in token order (skill write-up, Core Concept:
//                  hierarchical token aggregation; window 32, stride 16);
//   score_f32    : one warp per query row (b, g, t): each head's log-sum-exp
//                  over the visible windows (pass 1), then the group sum of
//                  the heads' probabilities per window, max-pooled onto the
//                  blocks whose tokens the window overlaps (pass 2), into the
//                  same causally packed block-score rows the top-k reads
//                  (skill write-up, Architecture Overview, Hardware Kernel
//                  bullet: scores summed over the heads of a group);
//   attn_f32     : one warp per query row, lane = 4 channels of every head of
//                  the group, exact online softmax over the row's keys (its
//                  selected blocks, or every key 0..t) with fp32 P and O.
#include <math.h>

#include "common.cuh"

namespace infllmv2 {
namespace {

constexpr float kLn2d = 0.6931471805599453f;

__global__ void __launch_bounds__(256) compress_f32_kernel(const __nv_bfloat16* __restrict__ K,
                                                           float* __restrict__ Kc, int B, int T,
                                                           int Hkv, int n_c) {
  const int64_t total = static_cast<int64_t>(B) * n_c * Hkv * kHeadDim;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(i % kHeadDim);
    int64_t rest = i / kHeadDim;
    const int g = static_cast<int>(rest % Hkv);
    rest /= Hkv;
    const int j = static_cast<int>(rest % n_c);
    const int b = static_cast<int>(rest / n_c);
    const __nv_bfloat16* src =
        K + ((static_cast<int64_t>(b) * T + static_cast<int64_t>(j) * kCmpStride) * Hkv + g) *
                kHeadDim + c;
    float acc = 0.f;
    for (int k = 0; k < kCmpKernel; ++k)
      acc += __bfloat162float(src[static_cast<int64_t>(k) * Hkv * kHeadDim]);
    Kc[i] = acc * (1.0f / kCmpKernel);
  }
}

constexpr int kRowsPerCta = 4;  // warps (query rows) per CTA of the scoring kernel

// Dynamic shared memory per warp: the group's G query rows (fp32) and the
// row's block scores (as ordered int bits, for atomicMax).
template <int G>
__global__ void __launch_bounds__(32 * kRowsPerCta) score_f32_kernel(
    const __nv_bfloat16* __restrict__ Q, const float* __restrict__ Kc, float* __restrict__ scores,
    int B, int q0, int Tq, int Hq, int Hkv, int n_c, int nb_cap, float scale_log2) {
  extern __shared__ float fsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* q = fsm + warp * (G * kHeadDim);
  int* bs = reinterpret_cast<int*>(fsm + kRowsPerCta * G * kHeadDim) + warp * nb_cap;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + warp;
  const int64_t n_rows = static_cast<int64_t>(B) * Hkv * Tq;
  if (row >= n_rows) return;
  const int qtok = static_cast<int>(row % Tq);
  const int64_t bg = row / Tq;
  const int b = static_cast<int>(bg / Hkv), g = static_cast<int>(bg % Hkv);
  const int t = q0 + qtok;
  const int v = min(n_c, visible_windows(t));
  const int cur = t / kBlock;
  for (int i = lane; i < G * kHeadDim; i += 32)
    q[i] = __bfloat162float(
        Q[((static_cast<int64_t>(b) * Tq + qtok) * Hq + g * G) * kHeadDim + i]);
  const int neg_inf_bits = __float_as_int(-INFINITY);
  for (int i = lane; i <= cur; i += 32) bs[i] = neg_inf_bits;
  __syncwarp();
  const float* kc = Kc + static_cast<int64_t>(b) * n_c * Hkv * kHeadDim + g * kHeadDim;
  auto dots = [&](int j, float (&s)[G]) {
    const float4* kr = reinterpret_cast<const float4*>(kc + static_cast<int64_t>(j) * Hkv * kHeadDim);
#pragma unroll
    for (int h = 0; h < G; ++h) s[h] = 0.f;
    for (int c4 = 0; c4 < kHeadDim / 4; ++c4) {
      const float4 k4 = __ldg(kr + c4);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float4 q4 = reinterpret_cast<const float4*>(q + h * kHeadDim)[c4];
        s[h] = fmaf(q4.x, k4.x, s[h]);
        s[h] = fmaf(q4.y, k4.y, s[h]);
        s[h] = fmaf(q4.z, k4.z, s[h]);
        s[h] = fmaf(q4.w, k4.w, s[h]);
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) s[h] *= scale_log2;
  };
  // pass 1: each head's log2-sum-exp over the visible windows
  float m[G], l[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
  }
  for (int j = lane; j < v; j += 32) {
    float s[G];
    dots(j, s);
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float mn = fmaxf(m[h], s[h]);
      l[h] = l[h] * exp2f(m[h] - mn) + exp2f(s[h] - mn);
      m[h] = mn;
    }
  }
  float lse2[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float M = m[h], L = l[h];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float M2 = __shfl_xor_sync(0xffffffffu, M, o);
      const float L2 = __shfl_xor_sync(0xffffffffu, L, o);
      const float mn = fmaxf(M, M2);
      L = (mn == -INFINITY) ? 0.f
                            : (M > -INFINITY ? L * exp2f(M - mn) : 0.f) +
                                  (M2 > -INFINITY ? L2 * exp2f(M2 - mn) : 0.f);
      M = mn;
    }
    lse2[h] = M + log2f(L);
  }
  // pass 2: group sum of the probabilities, max-pooled onto blocks j/4 and,
  // for the window 4b-1 shared by blocks b-1 and b, also (j+1)/4
  for (int j = lane; j < v; j += 32) {
    float s[G];
    dots(j, s);
    float S = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) S += exp2f(s[h] - lse2[h]);
    const int bits = __float_as_int(S);  // S >= 0: int order is float order
    const int b0 = j / 4;
    if (b0 <= cur) atomicMax(bs + b0, bits);
    if ((j & 3) == 3 && b0 + 1 <= cur) atomicMax(bs + b0 + 1, bits);
  }
  __syncwarp();
  const int64_t row0 = score_row_offset(q0);
  const int64_t slab = score_row_offset(q0 + Tq) - row0;
  float* out = scores + bg * slab + score_row_offset(t) - row0;
  for (int i = lane; i <= cur; i += 32) out[i] = __int_as_float(bs[i]);
}

// One warp per query row; idx == null: dense (every key 0..t).
template <int G>
__global__ void __launch_bounds__(128) attn_f32_kernel(
    const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ idx, float* __restrict__ O,
    float* __restrict__ lse, int B, int q0, int Tq, int T, int Hq, int Hkv, int topk,
    float scale_log2) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 4 + warp;
  const int64_t n_rows = static_cast<int64_t>(B) * Hkv * Tq;
  if (row >= n_rows) return;
  const int qtok = static_cast<int>(row % Tq);
  const int64_t bg = row / Tq;
  const int b = static_cast<int>(bg / Hkv), g = static_cast<int>(bg % Hkv);
  const int t = q0 + qtok, cur = t / kBlock;
  const int c0 = 4 * lane;
  float q[G][4], o[G][4], m[G], l[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const __nv_bfloat16* qs = Q + ((static_cast<int64_t>(b) * Tq + qtok) * Hq + g * G + h) * kHeadDim + c0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      q[h][c] = __bfloat162float(qs[c]);
      o[h][c] = 0.f;
    }
    m[h] = -INFINITY;
    l[h] = 0.f;
  }
  const int32_t* irow = idx ? idx + row * topk : nullptr;
  const int n_blocks = irow ? topk : cur + 1;
  for (int e = 0; e < n_blocks; ++e) {
    const int blk = irow ? __ldg(irow + e) : e;
    if (blk < 0 || blk > cur) {
      if (irow) break;  // valid entries come first, ascending
      continue;
    }
    const int k_end = min(blk * kBlock + kBlock - 1, t);
    for (int k = blk * kBlock; k <= k_end; ++k) {
      const int64_t off = ((static_cast<int64_t>(b) * T + k) * Hkv + g) * kHeadDim + c0;
      float kv[4], vv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        kv[c] = __bfloat162float(K[off + c]);
        vv[c] = __bfloat162float(V[off + c]);
      }
      float s[G];
#pragma unroll
      for (int h = 0; h < G; ++h)
        s[h] = q[h][0] * kv[0] + q[h][1] * kv[1] + q[h][2] * kv[2] + q[h][3] * kv[3];
#pragma unroll
      for (int w = 16; w > 0; w >>= 1) {
#pragma unroll
        for (int h = 0; h < G; ++h) s[h] += __shfl_xor_sync(0xffffffffu, s[h], w);
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float x = s[h] * scale_log2;
        const float mn = fmaxf(m[h], x);
        const float alpha = exp2f(m[h] - mn);  // 0 for the row's first key
        const float p = exp2f(x - mn);
        l[h] = l[h] * alpha + p;
#pragma unroll
        for (int c = 0; c < 4; ++c) o[h][c] = o[h][c] * alpha + p * vv[c];
        m[h] = mn;
      }
    }
  }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float* os = O + ((static_cast<int64_t>(b) * Tq + qtok) * Hq + g * G + h) * kHeadDim + c0;
    const float inv = l[h] > 0.f ? 1.f / l[h] : 0.f;
    *reinterpret_cast<float4*>(os) =
        make_float4(o[h][0] * inv, o[h][1] * inv, o[h][2] * inv, o[h][3] * inv);
    if (lane == 0)
      lse[(static_cast<int64_t>(b) * Hq + g * G + h) * Tq + qtok] =
          l[h] > 0.f ? (m[h] + log2f(l[h])) * kLn2d : -INFINITY;
  }
}

template <int G>
int launch_f32_g(const Geometry& g, const void* Q, const void* K, const void* V, void* O,
                 float* lse, float* Kc32, int32_t* idx, float* scores, bool dense,
                 cudaStream_t st) {
  const int64_t rows = static_cast<int64_t>(g.B) * g.Hkv * g.Tq;
  if (!dense) {
    if (g.n_c > 0) {
      const int64_t total = static_cast<int64_t>(g.B) * g.n_c * g.Hkv * kHeadDim;
      const int64_t blocks = (total + 255) / 256;
      compress_f32_kernel<<<static_cast<unsigned>(blocks < 65535 * 16 ? blocks : 65535 * 16), 256,
                            0, st>>>(static_cast<const __nv_bfloat16*>(K), Kc32, g.B, g.T, g.Hkv,
                                     g.n_c);
      if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
    }
    const int nb_cap = (g.q0 + g.Tq - 1) / kBlock + 1;
    const size_t smem = (static_cast<size_t>(kRowsPerCta) * G * kHeadDim +
                         static_cast<size_t>(kRowsPerCta) * nb_cap) * sizeof(float);
    if (smem > 227 * 1024) return INFLLMV2_ERR_UNSUPPORTED;
    static std::atomic<uint64_t> smem_set{0};
    if (int e = set_smem_limit(score_f32_kernel<G>, 227 * 1024, smem_set)) return e;
    score_f32_kernel<G><<<static_cast<unsigned>((rows + kRowsPerCta - 1) / kRowsPerCta),
                          32 * kRowsPerCta, smem, st>>>(
        static_cast<const __nv_bfloat16*>(Q), Kc32, scores, g.B, g.q0, g.Tq, g.Hq, g.Hkv, g.n_c,
        nb_cap, g.scale_log2);
    if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
    if (int e = launch_topk(g, scores, idx, st)) return e;
  }
  attn_f32_kernel<G><<<static_cast<unsigned>((rows + 3) / 4), 128, 0, st>>>(
      static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K),
      static_cast<const __nv_bfloat16*>(V), dense ? nullptr : idx, static_cast<float*>(O), lse,
      g.B, g.q0, g.Tq, g.T, g.Hq, g.Hkv, g.topk, g.scale_log2);
  return cudaGetLastError() == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

}  // namespace

int launch_forward_f32(const Geometry& g, const void* Q, const void* K, const void* V, void* O,
                       float* lse, float* Kc32, int32_t* idx, float* scores, bool dense,
                       cudaStream_t st) {
  if (g.B == 0 || g.Tq == 0) return INFLLMV2_OK;
  switch (g.G) {
    case 1: return launch_f32_g<1>(g, Q, K, V, O, lse, Kc32, idx, scores, dense, st);
    case 2: return launch_f32_g<2>(g, Q, K, V, O, lse, Kc32, idx, scores, dense, st);
    case 4: return launch_f32_g<4>(g, Q, K, V, O, lse, Kc32, idx, scores, dense, st);
    case 8: return launch_f32_g<8>(g, Q, K, V, O, lse, Kc32, idx, scores, dense, st);
    case 16: return launch_f32_g<16>(g, Q, K, V, O, lse, Kc32, idx, scores, dense, st);
    default: return INFLLMV2_ERR_UNSUPPORTED;
  }
}

}  // namespace infllmv2
