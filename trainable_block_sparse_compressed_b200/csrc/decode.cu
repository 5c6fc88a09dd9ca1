// decode.cu -- one decode step for B sequences with caches (reportify digest,
// Performance Evaluation: the operator speed-up is reported for decode as
// well as prefill).
//
// Kernel sequence on the caller's stream:
//   1. append      : K/V of the new token at pos = seqlens[b]; when window
//                    (pos-31)/16 completes, its compressed key (mean of the 32
//                    rows, summed in token order and stored as the bf16 pair
//                    hi + lo exactly as compress.cu does, so incremental and
//                    batch compressed keys are bit-identical);
//   2. score       : x[j, h] = scale*log2(e) * q_h . Kc[j] for the visible
//                    windows, split over many CTAs (HBM-bound stream of the
//                    compressed-key cache), plus each split's per-head max and
//                    sum of exp2 for the softmax;
//   3. select      : per (sequence, kv head), split over CTAs of 128 blocks
//                    each: merge the splits into each head's log-sum-exp,
//                    group-sum the probabilities, max-pool onto 64-token
//                    blocks; the last CTA of the row runs the warp top-k with
//                    the forced blocks;
//   4. attention   : sparse_attn.cu in decode mode, the selected blocks split
//                    into chunks, unnormalised partials;
//   5. combine     : merge the chunk partials into O and LSE (one CTA per
//                    head); seqlens += 1.
#include "common.cuh"
#include "sm100.cuh"
#include "topk.cuh"

namespace infllmv2 {

int launch_decode_attn(const Geometry& g, const void* q, const void* Kcache, const void* Vcache,
                       const int32_t* idx, const int32_t* seqlens, float* part, int n_chunks,
                       int chunk_blocks, const DevCtx& ctx, cudaStream_t st);

namespace {

constexpr int kScoreRows = 512;     // compressed rows per scoring CTA
constexpr int kChunkBlocks = 8;     // selected blocks per attention item
constexpr float kLn2 = 0.6931471805599453f;

constexpr int kPoolBlocks = 128;    // blocks max-pooled per pooling CTA

struct DecodeLayout {
  int NC, NB, n_split, n_chunks, n_pool;
  size_t off_active, off_x, off_ml, off_idx, off_part, off_bs, off_cnt, total;
};

DecodeLayout decode_layout(const Geometry& g) {
  DecodeLayout L;
  L.NC = num_compressed(g.T);
  L.NB = g.T > 0 ? (g.T - 1) / kBlock + 1 : 0;
  L.n_split = L.NC > 0 ? (L.NC + kScoreRows - 1) / kScoreRows : 1;
  L.n_chunks = (g.topk + kChunkBlocks - 1) / kChunkBlocks;
  L.n_pool = L.NB > 0 ? (L.NB + kPoolBlocks - 1) / kPoolBlocks : 1;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t bg = static_cast<size_t>(g.B) * g.Hkv;
  size_t o = 0;
  L.off_active = o;
  o = up(o + static_cast<size_t>(g.B) * sizeof(int32_t));
  L.off_x = o;
  o = up(o + bg * L.NC * g.G * sizeof(float));
  L.off_ml = o;
  o = up(o + bg * L.n_split * g.G * 2 * sizeof(float));
  L.off_idx = o;
  o = up(o + bg * g.topk * sizeof(int32_t));
  L.off_part = o;
  o = up(o + bg * L.n_chunks * g.G * (kHeadDim + 2) * sizeof(float));
  L.off_bs = o;
  o = up(o + bg * static_cast<size_t>(L.NB) * sizeof(float));
  L.off_cnt = o;
  o = up(o + bg * sizeof(uint32_t));
  L.total = o;
  return L;
}

// ---- 1. append ------------------------------------------------------------
__global__ void __launch_bounds__(32) decode_append_kernel(
    const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new,
    __nv_bfloat16* __restrict__ Kc_, __nv_bfloat16* __restrict__ Vc_,
    __nv_bfloat16* __restrict__ Kcmp, const int32_t* __restrict__ seqlens,
    int32_t* __restrict__ active, uint32_t* __restrict__ pool_count, int Hkv, int Lmax, int NC,
    int* status) {
  const int b = blockIdx.x / Hkv, g = blockIdx.x % Hkv;
  const int tid = threadIdx.x;
  if (tid == 0) pool_count[blockIdx.x] = 0;  // arrivals of this step's pooling CTAs
  const int pos = seqlens[b];
  const bool act = pos >= 0 && pos < Lmax;
  if (g == 0 && tid == 0) {
    active[b] = act ? 1 : 0;
    if (!act) report_status(status, INFLLMV2_STATUS_SEQ_FULL);
  }
  if (!act) return;
  const int c = tid & 15;
  const int64_t row_stride = static_cast<int64_t>(Hkv) * kHeadDim;
  const int64_t src = (static_cast<int64_t>(b) * Hkv + g) * kHeadDim + 8 * c;
  const int64_t dst = (static_cast<int64_t>(b) * Lmax + pos) * row_stride + g * kHeadDim + 8 * c;
  const uint4 kv = *reinterpret_cast<const uint4*>((tid < 16 ? k_new : v_new) + src);
  *reinterpret_cast<uint4*>((tid < 16 ? Kc_ : Vc_) + dst) = kv;
  if (tid < 16 && pos >= kCmpKernel - 1 && (pos - (kCmpKernel - 1)) % kCmpStride == 0) {
    const int j = (pos - (kCmpKernel - 1)) / kCmpStride;
    if (j < NC) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i < kCmpKernel; ++i) {
        const int tok = j * kCmpStride + i;
        const uint4 v = tok == pos ? kv
                                   : *reinterpret_cast<const uint4*>(
                                         Kc_ + (static_cast<int64_t>(b) * Lmax + tok) * row_stride +
                                         g * kHeadDim + 8 * c);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __bfloat1622float2(h[k]);
          acc[2 * k] += f.x;
          acc[2 * k + 1] += f.y;
        }
      }
      const float inv = 1.0f / kCmpKernel;
#pragma unroll
      for (int k = 0; k < 8; ++k) acc[k] *= inv;
      store_kc_pair(acc, Kcmp + ((static_cast<int64_t>(b) * NC + j) * Hkv + g) * kKcRow + 8 * c);
    }
  }
}

// ---- 2. score --------------------------------------------------------------
template <int G>
__global__ void __launch_bounds__(256) decode_score_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ Kcmp,
    const int32_t* __restrict__ seqlens, float* __restrict__ x_out, float* __restrict__ ml,
    int Hq, int Hkv, int NC, int Lmax, int n_split, float scale_log2) {
  __shared__ float sq[G][kHeadDim];
  __shared__ float red_m[8][G], red_l[8][G];
  const int split = blockIdx.x % n_split;
  const int bg = blockIdx.x / n_split;
  const int b = bg / Hkv, g = bg % Hkv;
  const int t = seqlens[b];
  const int v = (t >= 0 && t < Lmax) ? min(NC, visible_windows(t)) : 0;
  for (int i = threadIdx.x; i < G * kHeadDim; i += blockDim.x) {
    const int h = i / kHeadDim, d = i % kHeadDim;
    sq[h][d] = __bfloat162float(q[(static_cast<int64_t>(b) * Hq + g * G + h) * kHeadDim + d]) *
               scale_log2;
  }
  __syncthreads();
  float m[G], l[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
  }
  const int j_end = min(v, (split + 1) * kScoreRows);
  for (int j = split * kScoreRows + threadIdx.x; j < j_end; j += blockDim.x) {
    const __nv_bfloat16* row = Kcmp + ((static_cast<int64_t>(b) * NC + j) * Hkv + g) * kKcRow;
    float acc[G];
#pragma unroll
    for (int h = 0; h < G; ++h) acc[h] = 0.f;
#pragma unroll 4
    for (int d0 = 0; d0 < kHeadDim; d0 += 8) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(row + d0));
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(row + kHeadDim + d0));
      const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&u);
      const __nv_bfloat162* lv = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 fh = __bfloat1622float2(hv[k]);
        const float2 fl = __bfloat1622float2(lv[k]);
        const float2 f = make_float2(fh.x + fl.x, fh.y + fl.y);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          acc[h] = fmaf(f.x, sq[h][d0 + 2 * k], acc[h]);
          acc[h] = fmaf(f.y, sq[h][d0 + 2 * k + 1], acc[h]);
        }
      }
    }
    float* xo = x_out + (static_cast<int64_t>(bg) * NC + j) * G;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      xo[h] = acc[h];
      const float mn = fmaxf(m[h], acc[h]);
      l[h] = l[h] * fast_exp2(m[h] - mn) + fast_exp2(acc[h] - mn);
      m[h] = mn;
    }
  }
  // CTA reduction of (m, l) per head
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float mw = warp_max(m[h]);
    float lw = mw > -INFINITY ? warp_sum(l[h] * fast_exp2(m[h] - mw)) : 0.f;
    if (lane == 0) {
      red_m[warp][h] = mw;
      red_l[warp][h] = lw;
    }
  }
  __syncthreads();
  if (threadIdx.x < G) {
    const int h = threadIdx.x;
    float M = -INFINITY;
    for (int w = 0; w < 8; ++w) M = fmaxf(M, red_m[w][h]);
    float L = 0.f;
    if (M > -INFINITY)
      for (int w = 0; w < 8; ++w) L += red_l[w][h] * fast_exp2(red_m[w][h] - M);
    float* o = ml + (static_cast<int64_t>(bg) * n_split + split) * G * 2;
    o[2 * h] = M;
    o[2 * h + 1] = L;
  }
}

// ---- 3. select ---------------------------------------------------------------
// Pooling CTA (bg, part) owns blocks [part*128, part*128 + 128) of row bg:
// merges the score splits into each head's log2-sum-exp, sums the G heads'
// probabilities over the windows overlapping its blocks, max-pools them, and
// writes the block scores.  The last CTA of the row to finish (an arrival
// counter that the append kernel zeroed) runs the CTA top-k over the row,
// PER blocks per thread.
template <int G, int PER>
__global__ void __launch_bounds__(256) decode_select_kernel(
    const float* __restrict__ x, const float* __restrict__ ml, const int32_t* __restrict__ seqlens,
    float* bs_all, uint32_t* pool_count, int32_t* __restrict__ idx, int Hkv, int NC, int NB,
    int Lmax, int n_split, int n_pool, int topk, int n_init, int n_local) {
  constexpr int kWin = 4 * kPoolBlocks + 4;  // windows 4*blk0-1 .. 4*blk1+3 (clipped)
  __shared__ float S[kWin];
  __shared__ float lse2[G];
  __shared__ bool last;
  const int bg = blockIdx.x / n_pool;
  const int part = blockIdx.x % n_pool;
  const int b = bg / Hkv;
  const int t = seqlens[b];
  int32_t* orow = idx + static_cast<int64_t>(bg) * topk;
  if (!(t >= 0 && t < Lmax)) {
    if (part == 0)
      for (int k = threadIdx.x; k < topk; k += blockDim.x) orow[k] = -1;
    return;
  }
  const int v = min(NC, visible_windows(t));
  const int cur = t / kBlock;
  const int blk0 = part * kPoolBlocks;
  const int blk1 = min(cur + 1, blk0 + kPoolBlocks);
  float* bs = bs_all + static_cast<int64_t>(bg) * NB;
  if (blk0 < blk1) {
    if (threadIdx.x < G) {
      const int h = threadIdx.x;
      const float* p = ml + static_cast<int64_t>(bg) * n_split * G * 2;
      float M = -INFINITY;
      for (int s2 = 0; s2 < n_split; ++s2) M = fmaxf(M, p[s2 * G * 2 + 2 * h]);
      float L = 0.f;
      if (M > -INFINITY)
        for (int s2 = 0; s2 < n_split; ++s2)
          L += p[s2 * G * 2 + 2 * h + 1] * fast_exp2(p[s2 * G * 2 + 2 * h] - M);
      lse2[h] = M > -INFINITY ? M + __log2f(L) : INFINITY;
    }
    __syncthreads();
    const int j0 = max(0, 4 * blk0 - 1);
    const int j1 = min(v, 4 * blk1 + 3);  // exclusive
    for (int j = j0 + threadIdx.x; j < j1; j += blockDim.x) {
      const float4* xr = reinterpret_cast<const float4*>(x + (static_cast<int64_t>(bg) * NC + j) * G);
      float acc = 0.f;
      if constexpr (G % 4 == 0) {
#pragma unroll
        for (int h4 = 0; h4 < G / 4; ++h4) {
          const float4 u = __ldg(xr + h4);
          acc += fast_exp2(u.x - lse2[4 * h4]) + fast_exp2(u.y - lse2[4 * h4 + 1]) +
                 fast_exp2(u.z - lse2[4 * h4 + 2]) + fast_exp2(u.w - lse2[4 * h4 + 3]);
        }
      } else {
        const float* xs = x + (static_cast<int64_t>(bg) * NC + j) * G;
#pragma unroll
        for (int h = 0; h < G; ++h) acc += fast_exp2(__ldg(xs + h) - lse2[h]);
      }
      S[j - j0] = acc;
    }
    __syncthreads();
    for (int blk = blk0 + threadIdx.x; blk < blk1; blk += blockDim.x) {
      const int j_lo = max(0, 4 * blk - 1), j_hi = min(v - 1, 4 * blk + 3);
      float mx = -INFINITY;
      for (int j = j_lo; j <= j_hi; ++j) mx = fmaxf(mx, S[j - j0]);
      bs[blk] = mx;
    }
  }
  // the last pooling CTA of the row selects
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(pool_count + bg, 1u) == static_cast<uint32_t>(n_pool - 1);
  __syncthreads();
  if (!last) return;
  __threadfence();
  cta_select_row<256, PER>(bs, cur, topk, n_init, n_local, orow);
}

// Blocks per thread of the 256-thread CTA top-k for rows of up to nb blocks
// (0 if too many).
inline int select_per(int nb) {
  for (int per = 1; per <= 32; per *= 2)
    if (256 * per >= nb) return per;
  return 0;
}

// ---- 5. combine --------------------------------------------------------------
// One CTA per (sequence, kv head, head), one thread per channel.
template <int G>
__global__ void __launch_bounds__(128) decode_combine_kernel(
    const float* __restrict__ part, const int32_t* __restrict__ active, int32_t* seqlens,
    __nv_bfloat16* __restrict__ O, float* __restrict__ lse, int Hq, int Hkv, int n_chunks,
    int64_t n_items) {
  const int bg = blockIdx.x / G, h = blockIdx.x % G;
  const int b = bg / Hkv, g = bg % Hkv;
  const int d = threadIdx.x;
  const bool act = active[b] != 0;
  const float* po = part;
  const float* pml = part + n_items * (G * kHeadDim);
  float M = -INFINITY;
  for (int c = 0; c < n_chunks; ++c)
    M = fmaxf(M, pml[(static_cast<int64_t>(bg) * n_chunks + c) * 2 * G + 2 * h]);
  float acc = 0.f, wsum = 0.f;
  if (act && M > -INFINITY) {
    for (int c = 0; c < n_chunks; ++c) {
      const int64_t itm = static_cast<int64_t>(bg) * n_chunks + c;
      const float mc = pml[itm * 2 * G + 2 * h];
      if (mc == -INFINITY) continue;
      const float w = fast_exp2(mc - M);
      acc += w * po[itm * G * kHeadDim + h * kHeadDim + d];
      wsum += w * pml[itm * 2 * G + 2 * h + 1];
    }
  }
  const bool ok = act && wsum > 0.f;
  O[(static_cast<int64_t>(b) * Hq + g * G + h) * kHeadDim + d] =
      __float2bfloat16_rn(ok ? acc / wsum : 0.f);
  if (d == 0) lse[static_cast<int64_t>(b) * Hq + g * G + h] = ok ? (M + __log2f(wsum)) * kLn2 : 0.f;
  if (g == 0 && h == 0 && d == 0 && act) seqlens[b] += 1;
}

template <int G>
int launch_decode_g(const Geometry& g, const DecodeLayout& L, const void* q, const void* k_new,
                    const void* v_new, void* Kc_, void* Vc_, void* Kcmp, int32_t* seqlens, void* O,
                    float* lse, int32_t* idx, uint8_t* ws, const DevCtx& ctx, cudaStream_t st) {
  int32_t* active = reinterpret_cast<int32_t*>(ws + L.off_active);
  float* x = reinterpret_cast<float*>(ws + L.off_x);
  float* ml = reinterpret_cast<float*>(ws + L.off_ml);
  float* part = reinterpret_cast<float*>(ws + L.off_part);
  float* bs = reinterpret_cast<float*>(ws + L.off_bs);
  uint32_t* pool_count = reinterpret_cast<uint32_t*>(ws + L.off_cnt);
  const int bgn = g.B * g.Hkv;
  decode_append_kernel<<<bgn, 32, 0, st>>>(
      static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new),
      static_cast<__nv_bfloat16*>(Kc_), static_cast<__nv_bfloat16*>(Vc_),
      static_cast<__nv_bfloat16*>(Kcmp), seqlens, active, pool_count, g.Hkv, g.T, L.NC,
      ctx.status);
  if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
  decode_score_kernel<G><<<bgn * L.n_split, 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(Kcmp), seqlens, x, ml,
      g.Hq, g.Hkv, L.NC, g.T, L.n_split, g.scale_log2);
  if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
  const int per = select_per(L.NB);
#define INFLLMV2_SEL(V)                                                                        \
  decode_select_kernel<G, V><<<bgn * L.n_pool, 256, 0, st>>>(                                  \
      x, ml, seqlens, bs, pool_count, idx, g.Hkv, L.NC, L.NB, g.T, L.n_split, L.n_pool, g.topk, \
      g.n_init, g.n_local)
  switch (per) {
    case 1: INFLLMV2_SEL(1); break;
    case 2: INFLLMV2_SEL(2); break;
    case 4: INFLLMV2_SEL(4); break;
    case 8: INFLLMV2_SEL(8); break;
    case 16: INFLLMV2_SEL(16); break;
    case 32: INFLLMV2_SEL(32); break;
    default: return INFLLMV2_ERR_UNSUPPORTED;
  }
#undef INFLLMV2_SEL
  if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
  if (int e = launch_decode_attn(g, q, Kc_, Vc_, idx, seqlens, part, L.n_chunks, kChunkBlocks, ctx,
                                 st))
    return e;
  const int64_t n_items = static_cast<int64_t>(bgn) * L.n_chunks;
  decode_combine_kernel<G><<<bgn * G, 128, 0, st>>>(part, active, seqlens,
                                                static_cast<__nv_bfloat16*>(O), lse, g.Hq, g.Hkv,
                                                L.n_chunks, n_items);
  return cudaGetLastError() == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

}  // namespace

size_t decode_ws_bytes(const Geometry& g) { return decode_layout(g).total; }

int launch_decode_step(const Geometry& g, const void* q, const void* k_new, const void* v_new,
                       void* K_cache, void* V_cache, void* Kc_cache, int32_t* seqlens, void* O,
                       float* lse, int32_t* idx_out, void* ws, const DevCtx& ctx,
                       cudaStream_t st) {
  const DecodeLayout L = decode_layout(g);
  if (select_per(L.NB) == 0) return INFLLMV2_ERR_UNSUPPORTED;
  uint8_t* w = static_cast<uint8_t*>(ws);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(w + L.off_idx);
  switch (g.G) {
    case 1: return launch_decode_g<1>(g, L, q, k_new, v_new, K_cache, V_cache, Kc_cache, seqlens, O, lse, idx, w, ctx, st);
    case 2: return launch_decode_g<2>(g, L, q, k_new, v_new, K_cache, V_cache, Kc_cache, seqlens, O, lse, idx, w, ctx, st);
    case 4: return launch_decode_g<4>(g, L, q, k_new, v_new, K_cache, V_cache, Kc_cache, seqlens, O, lse, idx, w, ctx, st);
    case 8: return launch_decode_g<8>(g, L, q, k_new, v_new, K_cache, V_cache, Kc_cache, seqlens, O, lse, idx, w, ctx, st);
    case 16: return launch_decode_g<16>(g, L, q, k_new, v_new, K_cache, V_cache, Kc_cache, seqlens, O, lse, idx, w, ctx, st);
    default: return INFLLMV2_ERR_UNSUPPORTED;
  }
}

}  // namespace infllmv2
