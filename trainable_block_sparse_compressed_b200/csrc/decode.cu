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
//                    windows, tiles of 128 compressed keys on tcgen05 (an
//                    HBM-bound stream of the compressed-key cache), plus each
//                    tile's per-head max and sum of exp2 for the softmax;
//   3. select      : per (sequence, kv head), split over CTAs of 128 blocks
//                    each: merge the splits into each head's log-sum-exp,
//                    group-sum the probabilities, max-pool onto 64-token
//                    blocks; then one CTA per row runs the exact top-k with
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

constexpr int kScoreTile = 128;     // compressed keys per scoring tile
constexpr int kChunkBlocks = 8;     // selected blocks per attention item
constexpr float kLn2 = 0.6931471805599453f;

constexpr int kPoolBlocks = 128;    // blocks max-pooled per pooling CTA

struct DecodeLayout {
  int NC, NB, n_split, n_chunks, n_pool;
  size_t off_active, off_x, off_ml, off_idx, off_part, off_bs, total;
};

DecodeLayout decode_layout(const Geometry& g) {
  DecodeLayout L;
  L.NC = num_compressed(g.T);
  L.NB = g.T > 0 ? (g.T - 1) / kBlock + 1 : 0;
  L.n_split = L.NC > 0 ? (L.NC + kScoreTile - 1) / kScoreTile : 1;  // score tiles per row
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
  L.total = o;
  return L;
}

// ---- 1. append ------------------------------------------------------------
__global__ void __launch_bounds__(32) decode_append_kernel(
    const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new,
    __nv_bfloat16* __restrict__ Kc_, __nv_bfloat16* __restrict__ Vc_,
    __nv_bfloat16* __restrict__ Kcmp, const int32_t* __restrict__ seqlens,
    int32_t* __restrict__ active, int Hkv, int Lmax, int NC, int* status) {
  const int b = blockIdx.x / Hkv, g = blockIdx.x % Hkv;
  const int tid = threadIdx.x;
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
// Unit = one tile of 128 compressed keys of one (sequence, kv head).  A
// persistent CTA walks units blockIdx.x, +gridDim.x, ...: warp 0 loads the
// tile's hi and lo planes (4 boxes of 128 rows x 64 channels, 128-byte
// swizzle) and the G query heads of the group into a 2-stage ring; warp 1
// issues D[128 keys x 16 heads] = Kc . q^T with tcgen05.mma over K = 256
// (q . hi + q . lo: the query tile is the B operand of both halves) into a
// TMEM accumulator (4 buffers); warps 2-9, two warpgroups taking alternate
// tiles (thread = key), write the scaled scores x[j, h] and each tile's
// per-head max and sum of exp2, which the
// select kernel merges into the head's log-sum-exp.  Units past the visible
// keys of their sequence are skipped by all roles alike.
constexpr int kDStages = 3;
constexpr int kDHalf = kScoreTile * 64 * 2;       // 128 rows x 64 channels: 16 KB
constexpr int kDKcBytes = 4 * kDHalf;             // hi and lo planes: 64 KB
constexpr int kDQBytes = 2 * 16 * 128;            // 16 head rows x 2 halves of 64 channels
constexpr int kDStageBytes = kDKcBytes + kDQBytes;  // 68 KB (a multiple of 1 KB)
constexpr int kDAcc = 4;                          // TMEM accumulators (16 columns each)
constexpr int kDThreads = 64 + 256;               // producer, MMA, two epilogue warpgroups

struct DScoreSmem {
  uint64_t full[kDStages], empty[kDStages];
  uint64_t acc_full[kDAcc], acc_empty[kDAcc];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  // per epilogue warpgroup: the tile's scaled scores, transposed for the
  // per-head reductions
  float xs[2][kScoreTile][17];
};

struct DUnit {
  int bg, tile, b, g, v;
  bool active;
};

__device__ __forceinline__ DUnit decode_unit(int64_t u, const int32_t* seqlens, int Hkv, int NC,
                                             int n_tpb, int Lmax) {
  // seqlens: the sequences' positions (shared memory copy when B is small)
  DUnit r;
  r.bg = static_cast<int>(u / n_tpb);
  r.tile = static_cast<int>(u % n_tpb);
  r.b = r.bg / Hkv;
  r.g = r.bg % Hkv;
  const int t = seqlens[r.b];
  r.v = (t >= 0 && t < Lmax) ? min(NC, visible_windows(t)) : 0;
  r.active = r.tile * kScoreTile < r.v;
  return r;
}

__device__ __forceinline__ bool dwait(uint64_t* bar, uint32_t parity, const DevCtx& ctx,
                                      volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort_flag) return false;
  if (mbar_wait(bar, parity, ctx.wait_ns)) return true;
  report_status(ctx.status, INFLLMV2_STATUS_TIMEOUT);
  *abort_flag = 1;
  return false;
}

template <int G>
__global__ void __launch_bounds__(kDThreads, 1) decode_score_kernel(
    const __grid_constant__ CUtensorMap tmKc, const __grid_constant__ CUtensorMap tmQ,
    const int32_t* __restrict__ seqlens, float* __restrict__ x_out, float* __restrict__ ml, int B,
    int Hkv, int NC, int n_tpb, int Lmax, float scale_log2, DevCtx ctx) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  DScoreSmem& sm = *reinterpret_cast<DScoreSmem*>(base + kDStages * kDStageBytes);
  __shared__ int32_t s_seq[256];
  const int warp = warp_id(), lane = lane_id();
  const int64_t n_units = static_cast<int64_t>(B) * Hkv * n_tpb;
  for (int i = threadIdx.x; i < B && i < 256; i += blockDim.x) s_seq[i] = seqlens[i];
  const int32_t* seq = B <= 256 ? s_seq : seqlens;

  // query rows past G stay zero (padding columns of the product)
  for (int s = 0; s < kDStages; ++s)
    for (int i = threadIdx.x; i < kDQBytes / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(base + s * kDStageBytes + kDKcBytes)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int a = 0; a < kDAcc; ++a) {
      mbar_init(&sm.acc_full[a], 1);
      mbar_init(&sm.acc_empty[a], 4);  // one arrival per warp of the owning warpgroup
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kDAcc * 16);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmKc);
      tma_prefetch_desc(&tmQ);
      int n = 0;
      for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
        const DUnit d = decode_unit(u, seq, Hkv, NC, n_tpb, Lmax);
        if (!d.active) continue;
        const int s = n % kDStages;
        if (n >= kDStages && !dwait(&sm.empty[s], ((n / kDStages) & 1) ^ 1, ctx, abort_flag)) break;
        uint8_t* dst = base + s * kDStageBytes;
        mbar_arrive_expect_tx(&sm.full[s], kDKcBytes + 2 * G * 128);
#pragma unroll
        for (int x = 0; x < 4; ++x)  // hi d[0:64], hi d[64:128], lo d[0:64], lo d[64:128]
          tma_load_4d(dst + x * kDHalf, &tmKc, &sm.full[s], 64 * x, d.g, d.tile * kScoreTile, d.b);
        tma_load_4d(dst + kDKcBytes, &tmQ, &sm.full[s], 0, d.g * G, 0, d.b);
        tma_load_4d(dst + kDKcBytes + 2048, &tmQ, &sm.full[s], 64, d.g * G, 0, d.b);
        ++n;
      }
      // drain: never leave with copies of this CTA in flight
      for (int q = n - 1; q >= 0 && q >= n - kDStages; --q)
        mbar_wait(&sm.full[q % kDStages], (q / kDStages) & 1, ctx.wait_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc_bf16(128, 16, 0, 0);
      int n = 0;
      for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x) {
        const DUnit d = decode_unit(u, seq, Hkv, NC, n_tpb, Lmax);
        if (!d.active) continue;
        const int s = n % kDStages, a = n % kDAcc;
        if (!dwait(&sm.full[s], (n / kDStages) & 1, ctx, abort_flag)) break;
        if (n >= kDAcc && !dwait(&sm.acc_empty[a], ((n / kDAcc) & 1) ^ 1, ctx, abort_flag)) break;
        tc_fence_after();
        const uint32_t kc_addr = smem_u32(base + s * kDStageBytes);
        const uint32_t q_addr = kc_addr + kDKcBytes;
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          // k < 8: hi plane, k >= 8: lo plane; both against the same q
          const uint32_t off = ((k >> 2) & 1) * kDHalf + (k & 3) * 32;
          const uint64_t ad = smem_desc(kc_addr + (k >> 3) * 2 * kDHalf + off, 16, 1024, 2);
          const uint64_t bd = smem_desc(q_addr + ((k >> 2) & 1) * 2048 + (k & 3) * 32, 16, 1024, 2);
          umma_bf16(tmem + a * 16, ad, bd, idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&sm.empty[s]);
        umma_commit(&sm.acc_full[a]);
        ++n;
      }
      umma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, ctx.wait_ns);
    }
  } else {
    // two warpgroups take the active tiles alternately (tile n -> warpgroup
    // n & 1, accumulator n % 4); each synchronises only within itself
    const int wg = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int ew = warp & 3;            // warp within the warpgroup (heads ew, ew+4, ...)
    const int r = quad * 32 + lane;     // TMEM lane = key within the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t bar_sync = 1 + 2 * wg, bar_or = 2 + 2 * wg;
    float (*xs)[17] = sm.xs[wg];
    int n = 0, k = 0;  // active tiles seen, units seen
    for (int64_t u = blockIdx.x; u < n_units; u += gridDim.x, ++k) {
      const DUnit d = decode_unit(u, seq, Hkv, NC, n_tpb, Lmax);
      float* mlo = ml + (static_cast<int64_t>(d.bg) * n_tpb + d.tile) * G * 2;
      if (!d.active) {
        if (wg == (k & 1) && r < G) {
          mlo[2 * r] = -INFINITY;
          mlo[2 * r + 1] = 0.f;
        }
        continue;
      }
      const int mine = (n & 1) == wg;
      const int a = n % kDAcc;
      const int use = n / kDAcc;  // earlier uses of accumulator a
      ++n;
      if (!mine) continue;
      const bool ok = !*abort_flag && mbar_wait(&sm.acc_full[a], use & 1, ctx.wait_ns);
      if (named_bar_or(bar_or, 128, !ok)) {
        if (!ok) report_status(ctx.status, INFLLMV2_STATUS_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      float x[16];
      tmem_ld16(lane_addr + a * 16, x);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[a]);
      const int j = d.tile * kScoreTile + r;
      const bool valid = j < d.v;
#pragma unroll
      for (int h = 0; h < G; ++h) x[h] = valid ? x[h] * scale_log2 : -INFINITY;
      if (valid && INFLLMV2_CHECK(ctx.status, j < NC && d.bg < B * Hkv)) {
        float* xo = x_out + (static_cast<int64_t>(d.bg) * NC + j) * G;
        if constexpr (G % 4 == 0) {
#pragma unroll
          for (int h4 = 0; h4 < G / 4; ++h4)
            reinterpret_cast<float4*>(xo)[h4] =
                make_float4(x[4 * h4], x[4 * h4 + 1], x[4 * h4 + 2], x[4 * h4 + 3]);
        } else {
#pragma unroll
          for (int h = 0; h < G; ++h) xo[h] = x[h];
        }
      }
      // per-head max and sum of exp2 over the tile's keys: transpose through
      // shared memory, then warp ew reduces heads ew, ew+4, ... (4 keys per
      // lane), all of its heads' shuffle chains interleaved
#pragma unroll
      for (int h = 0; h < G; ++h) xs[r][h] = x[h];
      named_bar_sync(bar_sync, 128);
      constexpr int kHW = (G + 3) / 4;  // heads per warp
      float v[kHW][4], M[kHW], L[kHW];
#pragma unroll
      for (int i = 0; i < kHW; ++i) {
        const int h = ew + 4 * i;
#pragma unroll
        for (int c = 0; c < 4; ++c) v[i][c] = h < G ? xs[lane + 32 * c][h] : -INFINITY;
        M[i] = fmaxf(fmaxf(v[i][0], v[i][1]), fmaxf(v[i][2], v[i][3]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int i = 0; i < kHW; ++i) M[i] = fmaxf(M[i], __shfl_xor_sync(0xffffffffu, M[i], o));
      }
#pragma unroll
      for (int i = 0; i < kHW; ++i)
        L[i] = M[i] > -INFINITY ? fast_exp2(v[i][0] - M[i]) + fast_exp2(v[i][1] - M[i]) +
                                      fast_exp2(v[i][2] - M[i]) + fast_exp2(v[i][3] - M[i])
                                : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
        for (int i = 0; i < kHW; ++i) L[i] += __shfl_xor_sync(0xffffffffu, L[i], o);
      }
      if (lane == 0) {
#pragma unroll
        for (int i = 0; i < kHW; ++i) {
          const int h = ew + 4 * i;
          if (h < G) {
            mlo[2 * h] = M[i];
            mlo[2 * h + 1] = L[i];
          }
        }
      }
      named_bar_sync(bar_sync, 128);  // xs is rewritten by this warpgroup's next tile
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kDAcc * 16);
  }
}

// ---- 3. select ---------------------------------------------------------------
// Pooling CTA (bg, part) owns blocks [part*128, part*128 + 128) of row bg:
// merges the score splits into each head's log2-sum-exp, sums the G heads'
// probabilities over the windows overlapping its blocks, max-pools them, and
// writes the block scores; decode_topk_kernel then selects per row.
template <int G>
__global__ void __launch_bounds__(256) decode_pool_kernel(
    const float* __restrict__ x, const float* __restrict__ ml, const int32_t* __restrict__ seqlens,
    float* __restrict__ bs_all, int Hkv, int NC, int NB, int Lmax, int n_split, int n_pool,
    int* status) {
  constexpr int kWin = 4 * kPoolBlocks + 4;  // windows 4*blk0-1 .. 4*blk1+3 (clipped)
  __shared__ float S[kWin];
  __shared__ float lse2[G];
  const int bg = blockIdx.x / n_pool;
  const int part = blockIdx.x % n_pool;
  const int b = bg / Hkv;
  const int t = seqlens[b];
  if (!(t >= 0 && t < Lmax)) return;
  const int v = min(NC, visible_windows(t));
  const int cur = t / kBlock;
  const int blk0 = part * kPoolBlocks;
  const int blk1 = min(cur + 1, blk0 + kPoolBlocks);
  float* bs = bs_all + static_cast<int64_t>(bg) * NB;
  if (blk0 < blk1) {
    {
      // 16 threads per head merge the score tiles' (max, sum) pairs
      const int h = threadIdx.x >> 4, sub = threadIdx.x & 15;
      const float* p = ml + static_cast<int64_t>(bg) * n_split * G * 2;
      float M = -INFINITY, L = 0.f;
      if (h < G) {
#pragma unroll 4
        for (int s2 = sub; s2 < n_split; s2 += 16) {
          const float2 e = *reinterpret_cast<const float2*>(p + (s2 * G + h) * 2);
          const float mn = fmaxf(M, e.x);
          if (mn > -INFINITY) {
            L = L * fast_exp2(M - mn) + e.y * fast_exp2(e.x - mn);
            M = mn;
          }
        }
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        const float M2 = __shfl_xor_sync(0xffffffffu, M, o);
        const float L2 = __shfl_xor_sync(0xffffffffu, L, o);
        const float mn = fmaxf(M, M2);
        if (mn > -INFINITY) {
          L = (M > -INFINITY ? L * fast_exp2(M - mn) : 0.f) +
              (M2 > -INFINITY ? L2 * fast_exp2(M2 - mn) : 0.f);
          M = mn;
        }
      }
      if (h < G && sub == 0) lse2[h] = M > -INFINITY ? M + __log2f(L) : INFINITY;
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
      if (INFLLMV2_CHECK(status, j - j0 >= 0 && j - j0 < kWin)) S[j - j0] = acc;
    }
    __syncthreads();
    for (int blk = blk0 + threadIdx.x; blk < blk1; blk += blockDim.x) {
      const int j_lo = max(0, 4 * blk - 1), j_hi = min(v - 1, 4 * blk + 3);
      float mx = -INFINITY;
      for (int j = j_lo; j <= j_hi; ++j) mx = fmaxf(mx, S[j - j0]);
      if (INFLLMV2_CHECK(status, blk < NB)) bs[blk] = mx;
    }
  }
}

// One CTA of 256 threads per (sequence, kv head): the exact top-k over the
// row's block scores, PER blocks per thread.
template <int PER>
__global__ void __launch_bounds__(256) decode_topk_kernel(
    const float* __restrict__ bs_all, const int32_t* __restrict__ seqlens, int32_t* __restrict__ idx,
    int Hkv, int NB, int Lmax, int topk, int n_init, int n_local) {
  const int bg = blockIdx.x;
  const int t = seqlens[bg / Hkv];
  int32_t* orow = idx + static_cast<int64_t>(bg) * topk;
  if (!(t >= 0 && t < Lmax)) {
    for (int k = threadIdx.x; k < topk; k += blockDim.x) orow[k] = -1;
    return;
  }
  cta_select_row<256, PER>(bs_all + static_cast<int64_t>(bg) * NB, t / kBlock, topk, n_init,
                           n_local, orow);
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
  const int bgn = g.B * g.Hkv;
  decode_append_kernel<<<bgn, 32, 0, st>>>(
      static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new),
      static_cast<__nv_bfloat16*>(Kc_), static_cast<__nv_bfloat16*>(Vc_),
      static_cast<__nv_bfloat16*>(Kcmp), seqlens, active, g.Hkv, g.T, L.NC,
      ctx.status);
  if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
  if (L.NC > 0) {
    CUtensorMap tk, tq;
    {
      const uint64_t dims[4] = {static_cast<uint64_t>(kKcRow), static_cast<uint64_t>(g.Hkv),
                                static_cast<uint64_t>(L.NC), static_cast<uint64_t>(g.B)};
      const uint64_t strides[3] = {static_cast<uint64_t>(kKcRow) * 2,
                                   static_cast<uint64_t>(g.Hkv) * kKcRow * 2,
                                   static_cast<uint64_t>(L.NC) * g.Hkv * kKcRow * 2};
      const uint32_t box[4] = {64u, 1u, static_cast<uint32_t>(kScoreTile), 1u};
      if (int e = make_tmap_bf16_4d(&tk, Kcmp, dims, strides, box)) return e;
    }
    {
      const uint64_t dims[4] = {static_cast<uint64_t>(kHeadDim), static_cast<uint64_t>(g.Hq), 1u,
                                static_cast<uint64_t>(g.B)};
      const uint64_t strides[3] = {static_cast<uint64_t>(kHeadDim) * 2,
                                   static_cast<uint64_t>(g.Hq) * kHeadDim * 2,
                                   static_cast<uint64_t>(g.Hq) * kHeadDim * 2};
      const uint32_t box[4] = {64u, static_cast<uint32_t>(G), 1u, 1u};
      if (int e = make_tmap_bf16_4d(&tq, q, dims, strides, box)) return e;
    }
    const size_t smem = 1024 + kDStages * kDStageBytes + sizeof(DScoreSmem);
    static std::atomic<uint64_t> smem_set{0};
    if (int e = set_smem_limit(decode_score_kernel<G>, smem, smem_set)) return e;
    const int64_t n_units = static_cast<int64_t>(bgn) * L.n_split;
    const int grid = static_cast<int>(n_units < sm_count() ? n_units : sm_count());
    decode_score_kernel<G><<<grid, kDThreads, smem, st>>>(tk, tq, seqlens, x, ml, g.B, g.Hkv, L.NC,
                                                          L.n_split, g.T, g.scale_log2, ctx);
    if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
  }
  const int per = select_per(L.NB);
  decode_pool_kernel<G><<<bgn * L.n_pool, 256, 0, st>>>(x, ml, seqlens, bs, g.Hkv, L.NC, L.NB, g.T,
                                                       L.n_split, L.n_pool, ctx.status);
  if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
#define INFLLMV2_SEL(V)                                                                     \
  decode_topk_kernel<V><<<bgn, 256, 0, st>>>(bs, seqlens, idx, g.Hkv, L.NB, g.T, g.topk, \
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
