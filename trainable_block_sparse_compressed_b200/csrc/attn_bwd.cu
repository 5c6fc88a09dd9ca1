// attn_bwd.cu -- gradients of the block-sparse attention with the block
// selection held fixed: the method is a trainable sparse attention (paper
// page, Abstract), and the selection is a discrete choice, so training
// propagates through the attention over the chosen blocks.  For one query
// row (token t, head h) over its keys,
//
//   P = softmax(scale q K^T),  O = P V,  D = rowsum(dO * O),
//   dP = dO V^T,  dS = P * (dP - D),
//   dq = scale dS K,  dK += scale dS^T q,  dV += P^T dO,
//
// with P recomputed from the forward's log-sum-exp (no online softmax).
// Three passes, all on the tensor cores (tcgen05.mma, bf16 in, fp32 out):
//
//   delta : D per query row (a row-sum of dO * O);
//   dQ    : the forward's query tiles (128 rows: 128/G tokens x G heads)
//           over the union of their tokens' blocks, each row masked to its
//           own blocks: S = Q K^T and dP = dO V^T per 128-key tile, dS in
//           tensor memory, dQ += dS K accumulated in tensor memory;
//   dK dV : key-block-major.  An inverted index lists, for every block, the
//           query tokens that selected it (ascending); a work item is one
//           block and up to kSeg of its tokens, in chunks of 128 gathered
//           rows: S = Q K_blk^T, dP = dO V_blk^T, then dV^T += dO^T P and
//           dK^T += Q^T dS accumulate in tensor memory (keys on the N side).
//           Items of one block write partials that a last pass sums in list
//           order, so the result does not depend on scheduling.
#include "common.cuh"
#include "sm100.cuh"
#include "topk.cuh"

namespace infllmv2 {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kIdxChunk = 256;  // query tokens per inverted-index chunk
constexpr int kSeg = 1024;      // query tokens of one block per dK/dV work item (at most)

__device__ __forceinline__ bool bwd_wait(uint64_t* bar, uint32_t parity, const DevCtx& ctx,
                                         volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort_flag) return false;
  if (mbar_wait(bar, parity, ctx.wait_ns)) return true;
  report_status(ctx.status, INFLLMV2_STATUS_TIMEOUT);
  *abort_flag = 1;
  return false;
}

// ---------------------------------------------------------------------------
// workspace
// ---------------------------------------------------------------------------
struct BwdLayout {
  int nb, n_ch, mi;         // key blocks, index chunks, item slots per (b, g)
  int64_t list_len;         // list slots per (b, g): Tq * topk
  size_t off_D, off_union, off_H, off_cnt, off_off, off_ioff, off_icnt, off_items, off_list,
      off_part, total;
};

BwdLayout bwd_layout(const Geometry& g) {
  BwdLayout L;
  auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
  const size_t bg = static_cast<size_t>(g.B) * g.Hkv;
  L.nb = g.Tq > 0 ? (g.q0 + g.Tq - 1) / kBlock + 1 : 0;
  L.n_ch = (g.Tq + kIdxChunk - 1) / kIdxChunk;
  L.list_len = static_cast<int64_t>(g.Tq) * g.topk;
  L.mi = static_cast<int>(L.list_len / kSeg) + L.nb + 1;
  size_t o = 0;
  L.off_D = o;
  o = up(o + static_cast<size_t>(g.B) * g.Hq * g.Tq * sizeof(float));
  L.off_union = o;
  o = up(o + union_lists_ws_bytes(g));
  L.off_H = o;
  o = up(o + bg * L.n_ch * L.nb * sizeof(int32_t));
  L.off_cnt = o;
  o = up(o + bg * L.nb * sizeof(int32_t));
  L.off_off = o;
  o = up(o + bg * L.nb * sizeof(int32_t));
  L.off_ioff = o;
  o = up(o + bg * L.nb * sizeof(int32_t));
  L.off_icnt = o;
  o = up(o + bg * sizeof(int32_t));
  L.off_items = o;
  o = up(o + bg * L.mi * sizeof(int4));
  L.off_list = o;
  o = up(o + bg * L.list_len * sizeof(int32_t));
  L.off_part = o;
  o = up(o + bg * L.mi * 2 * kBlock * kHeadDim * sizeof(float));
  L.total = o;
  return L;
}

// ---------------------------------------------------------------------------
// delta: D[b, h, t] = sum_d dO[b,t,h,d] O[b,t,h,d]; one warp per row
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_delta_kernel(const __nv_bfloat16* __restrict__ O,
                                                        const __nv_bfloat16* __restrict__ dO,
                                                        float* __restrict__ D, int B, int Tq,
                                                        int Hq) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<int64_t>(B) * Tq * Hq) return;
  const int h = static_cast<int>(row % Hq);
  const int64_t bt = row / Hq;
  const int t = static_cast<int>(bt % Tq), b = static_cast<int>(bt / Tq);
  const uint2 o = *reinterpret_cast<const uint2*>(O + row * kHeadDim + 4 * lane);
  const uint2 d = *reinterpret_cast<const uint2*>(dO + row * kHeadDim + 4 * lane);
  const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o);
  const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&d);
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float2 a = __bfloat1622float2(o2[k]), c = __bfloat1622float2(d2[k]);
    acc = fmaf(a.x, c.x, fmaf(a.y, c.y, acc));
  }
  acc = warp_sum(acc);
  if (lane == 0) D[(static_cast<int64_t>(b) * Hq + h) * Tq + t] = acc;
}

// ---------------------------------------------------------------------------
// dQ over the query tiles' union lists
// ---------------------------------------------------------------------------
struct DqArgs {
  float* dQ;                // [B, Tq, Hq, 128] fp32
  const float* lse;         // [B, Hq, Tq] natural log
  const float* D;           // [B, Hq, Tq]
  const uint2* ulist;
  const int32_t* ucount;
  int ustride;
  int B, Hq, Hkv, q0, Tq;
  float scale, scale_log2;
};

constexpr int kDqThreads = 64 + 256;
constexpr int kDqQ = 128 * 256;        // Q (or dO) tile: 128 rows x 128 channels bf16
constexpr int kDqStage = 2 * 128 * 256;  // K and V of a 128-key tile
// tensor memory: S (0..127), dP (128..255), dQ (256..383), dS (384..447, bf16 pairs)
constexpr uint32_t kDqS = 0, kDqP = 128, kDqAcc = 256, kDqDs = 384;

struct DqSmem {
  uint64_t q_full, q_empty, kv_full[2], kv_empty[2];
  uint64_t s_full, s_free, ds_full, ds_done, o_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int G>
__global__ void __launch_bounds__(kDqThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DqArgs a, DevCtx ctx) {
  constexpr int TPT = 128 / G;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = base;
  uint8_t* sdO = sQ + kDqQ;
  uint8_t* sKV = sdO + kDqQ;
  DqSmem& sm = *reinterpret_cast<DqSmem*>(sKV + 2 * kDqStage);
  const int warp = warp_id(), lane = lane_id();
  const int n_qt = (a.Tq + TPT - 1) / TPT;
  const int bgn = a.B * a.Hkv;
  const int64_t n_items = static_cast<int64_t>(bgn) * n_qt;

  // stale V/K rows of a one-block tile meet dS = 0 and P = 0: keep them finite
  for (int i = threadIdx.x; i < 2 * kDqStage / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sKV)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, 8);
    mbar_init(&sm.ds_full, 8);
    mbar_init(&sm.ds_done, 1);
    mbar_init(&sm.o_free, 8);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  // item k: query tile qt (latest first) of (b, g)
  auto item = [&](int64_t k, int& b, int& g, int& qtok0, int64_t& list, int& n_u) {
    const int qt = n_qt - 1 - static_cast<int>(k / bgn);
    const int bg = static_cast<int>(k % bgn);
    b = bg / a.Hkv;
    g = bg % a.Hkv;
    qtok0 = qt * TPT;
    list = static_cast<int64_t>(bg) * n_qt + qt;
    n_u = a.ucount[list];
  };

  if (warp == 0) {
    if (lane == 0) {
      int qk = 0;
      int64_t gt = 0;
      bool ok = true;
      for (int64_t k = blockIdx.x; ok && k < n_items; k += gridDim.x) {
        int b, g, qtok0, n_u;
        int64_t list;
        item(k, b, g, qtok0, list, n_u);
        const int n_kt = (n_u + 1) >> 1;
        if (n_kt == 0) continue;
        if (qk >= 1 && !(ok = bwd_wait(&sm.q_empty, (qk - 1) & 1, ctx, abort_flag))) break;
        mbar_arrive_expect_tx(&sm.q_full, 2 * kDqQ);
        for (int h = 0; h < 2; ++h) {
          tma_load_4d(sQ + h * (kDqQ / 2), &tmQ, &sm.q_full, 64 * h, g * G, qtok0, b);
          tma_load_4d(sdO + h * (kDqQ / 2), &tmdO, &sm.q_full, 64 * h, g * G, qtok0, b);
        }
        ++qk;
        const uint2* L = a.ulist + list * a.ustride;
        for (int i = 0; i < n_kt; ++i, ++gt) {
          const int s = static_cast<int>(gt & 1);
          if (gt >= 2 && !(ok = bwd_wait(&sm.kv_empty[s], ((gt >> 1) & 1) ^ 1, ctx, abort_flag)))
            break;
          const int nblk = 2 * i + 1 < n_u ? 2 : 1;
          mbar_arrive_expect_tx(&sm.kv_full[s], nblk * 4 * 8192);
          uint8_t* stK = sKV + s * kDqStage;
          uint8_t* stV = stK + kDqStage / 2;
          for (int e = 0; e < nblk; ++e) {
            const int blk = static_cast<int>(__ldg(L + 2 * i + e).x);
            for (int h = 0; h < 2; ++h) {
              tma_load_4d(stK + h * 16384 + e * 8192, &tmK, &sm.kv_full[s], 64 * h, g, blk * kBlock, b);
              tma_load_4d(stV + h * 16384 + e * 8192, &tmV, &sm.kv_full[s], 64 * h, g, blk * kBlock, b);
            }
          }
        }
      }
      if (qk > 0) mbar_wait(&sm.q_full, (qk - 1) & 1, ctx.wait_ns);
      for (int64_t q = gt - 1; q >= 0 && q >= gt - 2; --q)
        mbar_wait(&sm.kv_full[q & 1], (q >> 1) & 1, ctx.wait_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = instr_desc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_dq = instr_desc_bf16(128, 128, 0, 1);
      const uint32_t q_addr = smem_u32(sQ), do_addr = smem_u32(sdO);
      int qk = 0, ik = 0;
      int64_t gt = 0;
      bool ok = true;
      // dQ += dS(q) K(q): A = dS in tensor memory, B = the K tile as
      // MN-major (channels contiguous), 16 keys = 2 KB, halves 16 KB apart
      auto issue_dq = [&](int64_t q, bool first) -> bool {
        if (!bwd_wait(&sm.ds_full, static_cast<uint32_t>(q & 1), ctx, abort_flag)) return false;
        if (first && ik > 0 && !bwd_wait(&sm.o_free, (ik - 1) & 1, ctx, abort_flag)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sKV + (q & 1) * kDqStage);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_bf16_ts(tmem + kDqAcc, tmem + kDqDs + 8 * kk, smem_desc(k_addr + kk * 2048, 16384, 1024, 2),
                       idesc_dq, (first && kk == 0) ? 0u : 1u);
        umma_commit(&sm.kv_empty[q & 1]);
        umma_commit(&sm.ds_done);
        return true;
      };
      for (int64_t k = blockIdx.x; ok && k < n_items; k += gridDim.x) {
        int b, g, qtok0, n_u;
        int64_t list;
        item(k, b, g, qtok0, list, n_u);
        const int n_kt = (n_u + 1) >> 1;
        if (n_kt == 0) continue;
        if (!(ok = bwd_wait(&sm.q_full, qk & 1, ctx, abort_flag))) break;
        for (int i = 0; ok && i < n_kt; ++i, ++gt) {
          const int s = static_cast<int>(gt & 1);
          if (!(ok = bwd_wait(&sm.kv_full[s], (gt >> 1) & 1, ctx, abort_flag))) break;
          // S and dP are single buffers: the softmax has loaded those of gt-1
          if (gt > 0 && !(ok = bwd_wait(&sm.s_free, static_cast<uint32_t>((gt - 1) & 1), ctx, abort_flag)))
            break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sKV + s * kDqStage);
          const uint32_t v_addr = k_addr + kDqStage / 2;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16(tmem + kDqS, smem_desc(q_addr + off, 16, 1024, 2),
                      smem_desc(k_addr + off, 16, 1024, 2), idesc_s, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16(tmem + kDqP, smem_desc(do_addr + off, 16, 1024, 2),
                      smem_desc(v_addr + off, 16, 1024, 2), idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(&sm.s_full);
          if (i == n_kt - 1) umma_commit(&sm.q_empty);
          if (i > 0) ok = issue_dq(gt - 1, i == 1);
        }
        if (ok) ok = issue_dq(gt - 1, n_kt == 1);
        ++qk;
        ++ik;
      }
      umma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, ctx.wait_ns);
    }
  } else {
    // softmax warps: warpgroup hf owns key columns 64 hf .. 64 hf + 63 (block hf of the pair)
    const int hf = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int tok = r / G, h = r % G;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    int64_t gt = 0;
    bool ok = true;
    for (int64_t k = blockIdx.x; ok && k < n_items; k += gridDim.x) {
      int b, g, qtok0, n_u;
      int64_t list;
      item(k, b, g, qtok0, list, n_u);
      const int n_kt = (n_u + 1) >> 1;
      if (n_kt == 0) continue;
      const int qtok = qtok0 + tok;
      const bool row_ok = qtok < a.Tq;
      const int t = a.q0 + qtok;
      const int64_t lrow = (static_cast<int64_t>(b) * a.Hq + g * G + h) * a.Tq + qtok;
      const float lse2 = row_ok ? __ldg(a.lse + lrow) * kLog2e : 0.f;
      const float Dr = row_ok ? __ldg(a.D + lrow) : 0.f;
      const uint2* L = a.ulist + list * a.ustride;
      for (int i = 0; i < n_kt; ++i, ++gt) {
        ok = __all_sync(0xffffffffu, bwd_wait(&sm.s_full, static_cast<uint32_t>(gt & 1), ctx, abort_flag));
        if (!ok) break;
        const uint2 e = 2 * i + hf < n_u ? __ldg(L + 2 * i + hf) : make_uint2(0u, 0u);
        const bool sel = row_ok && ((e.y >> tok) & 1u) != 0u;
        const int lo = static_cast<int>(e.x) * kBlock;
        tc_fence_after();
        float x[64], y[64];
        tmem_ld32(lane_addr + kDqS + 64 * hf, *reinterpret_cast<float(*)[32]>(x));
        tmem_ld32(lane_addr + kDqS + 64 * hf + 32, *reinterpret_cast<float(*)[32]>(x + 32));
        tmem_ld32(lane_addr + kDqP + 64 * hf, *reinterpret_cast<float(*)[32]>(y));
        tmem_ld32(lane_addr + kDqP + 64 * hf + 32, *reinterpret_cast<float(*)[32]>(y + 32));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_free);
        // dS is a single buffer: dQ of the previous tile must have read it
        if (gt > 0) {
          ok = __all_sync(0xffffffffu, bwd_wait(&sm.ds_done, static_cast<uint32_t>((gt - 1) & 1), ctx,
                                                abort_flag));
          if (!ok) break;
        }
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            float v2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int col = 32 * q + 2 * c + u;
              const bool valid = sel && lo + col <= t;
              const float p = valid ? fast_exp2(fmaf(x[col], a.scale_log2, -lse2)) : 0.f;
              v2[u] = p * (y[col] - Dr);
            }
            __nv_bfloat162 b2 = __floats2bfloat162_rn(v2[0], v2[1]);
            pk[c] = *reinterpret_cast<uint32_t*>(&b2);
          }
          tmem_st16(lane_addr + kDqDs + 32 * hf + 16 * q, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.ds_full);
      }
      if (!ok) break;
      // epilogue: dQ (this half's 64 channels) times the softmax scale
      ok = __all_sync(0xffffffffu, bwd_wait(&sm.ds_done, static_cast<uint32_t>((gt - 1) & 1), ctx,
                                            abort_flag));
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float o[32];
        tmem_ld32(lane_addr + kDqAcc + 64 * hf + 32 * c, o);
        tmem_ld_wait();
        if (row_ok) {
          float4* dst = reinterpret_cast<float4*>(
              a.dQ + ((static_cast<int64_t>(b) * a.Tq + qtok) * a.Hq + g * G + h) * kHeadDim + 64 * hf +
              32 * c);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            dst[j] = make_float4(o[4 * j] * a.scale, o[4 * j + 1] * a.scale, o[4 * j + 2] * a.scale,
                                 o[4 * j + 3] * a.scale);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_free);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// inverted index: for every (b, g, block), the query rows that selected it,
// ascending.  hist: per chunk of 256 rows, the count per block; scan: per
// block, the chunks' exclusive prefix and the total, the lists' starts, and
// the work items (at most kSeg rows each); fill: each chunk places its rows,
// row after row, after the earlier chunks' ones.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) bwd_hist_kernel(const int32_t* __restrict__ idx,
                                                       int32_t* __restrict__ H, int q0, int Tq,
                                                       int topk, int nb, int n_ch) {
  extern __shared__ int hist[];
  const int64_t bg = blockIdx.x / n_ch;
  const int c = blockIdx.x % n_ch;
  for (int i = threadIdx.x; i < nb; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int n = kIdxChunk * topk;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int qtok = c * kIdxChunk + e / topk;
    if (qtok >= Tq) break;
    const int v = __ldg(idx + (bg * Tq + qtok) * topk + e % topk);
    if (v >= 0 && v <= (q0 + qtok) / kBlock) atomicAdd(&hist[v], 1);
  }
  __syncthreads();
  int32_t* out = H + (bg * n_ch + c) * nb;
  for (int i = threadIdx.x; i < nb; i += blockDim.x) out[i] = hist[i];
}

constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads) bwd_scan_kernel(
    int32_t* __restrict__ H, int32_t* __restrict__ cnt, int32_t* __restrict__ off,
    int32_t* __restrict__ ioff, int32_t* __restrict__ icnt, int4* __restrict__ items, int nb,
    int n_ch, int mi) {
  __shared__ int scan_buf[kScanThreads / 32 + 1];
  const int64_t bg = blockIdx.x;
  int32_t* Hb = H + bg * n_ch * nb;
  // per block: exclusive prefix over the chunks, and the total
  for (int kb = threadIdx.x; kb < nb; kb += blockDim.x) {
    int run = 0;
    for (int c = 0; c < n_ch; ++c) {
      const int h = Hb[static_cast<int64_t>(c) * nb + kb];
      Hb[static_cast<int64_t>(c) * nb + kb] = run;
      run += h;
    }
    cnt[bg * nb + kb] = run;
  }
  __syncthreads();
  // list starts and item starts: exclusive scans over the blocks
  int base = 0, ibase = 0;
  for (int k0 = 0; k0 < nb; k0 += kScanThreads) {
    const int kb = k0 + threadIdx.x;
    const int c = kb < nb ? cnt[bg * nb + kb] : 0;
    const int ni = (c + kSeg - 1) / kSeg;
    int tot, itot;
    const int o = cta_exclusive_scan<kScanThreads>(c, scan_buf, &tot);
    const int io = cta_exclusive_scan<kScanThreads>(ni, scan_buf, &itot);
    if (kb < nb) {
      off[bg * nb + kb] = base + o;
      ioff[bg * nb + kb] = ibase + io;
      for (int s = 0; s < ni && ibase + io + s < mi; ++s)
        items[bg * mi + ibase + io + s] =
            make_int4(kb, base + o + s * kSeg, base + o + min((s + 1) * kSeg, c), 0);
    }
    base += tot;
    ibase += itot;
  }
  if (threadIdx.x == 0) icnt[bg] = min(ibase, mi);
}

__global__ void __launch_bounds__(256) bwd_fill_kernel(const int32_t* __restrict__ idx,
                                                       const int32_t* __restrict__ H,
                                                       const int32_t* __restrict__ off,
                                                       int32_t* __restrict__ list, int64_t list_len,
                                                       int q0, int Tq, int topk, int nb, int n_ch) {
  extern __shared__ int pos[];
  const int64_t bg = blockIdx.x / n_ch;
  const int c = blockIdx.x % n_ch;
  for (int i = threadIdx.x; i < nb; i += blockDim.x)
    pos[i] = off[bg * nb + i] + H[(bg * n_ch + c) * nb + i];
  __syncthreads();
  int32_t* out = list + bg * list_len;
  for (int tl = 0; tl < kIdxChunk; ++tl) {
    const int qtok = c * kIdxChunk + tl;
    if (qtok >= Tq) break;
    // a row's entries are distinct blocks: no two threads move the same slot
    for (int j = threadIdx.x; j < topk; j += blockDim.x) {
      const int v = __ldg(idx + (bg * Tq + qtok) * topk + j);
      if (v >= 0 && v <= (q0 + qtok) / kBlock) {
        const int p = pos[v]++;
        if (p >= 0 && p < list_len) out[p] = qtok;
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// dK, dV: key-block-major over the inverted index
// ---------------------------------------------------------------------------
struct KvArgs {
  const int4* items;        // [B*Hkv][mi]: (block, list begin, list end, -)
  const int32_t* icnt;      // items per (b, g)
  int mi;
  const int32_t* list;      // [B*Hkv][list_len] query rows
  int64_t list_len;
  float* part;              // [B*Hkv*mi][2][64][128]: dV, dK partials of each item
  const float* lse;
  const float* D;
  int B, Hq, Hkv, q0, Tq;
  float scale_log2;
};

constexpr int kKvThreads = 64 + 256;
constexpr int kKvBlk = 64 * 256;            // K or V of one block: 64 keys x 128 channels
constexpr int kKvChunk = 2 * 128 * 256;     // Q and dO rows of one chunk
constexpr int kKvPd = 2 * 128 * 64 * 2;     // P and dS of one chunk: 128 rows x 64 keys bf16 each
// tensor memory: S (0..63), dP (64..127), dV^T (128..191), dK^T (192..255)
constexpr uint32_t kKvS = 0, kKvP = 64, kKvDv = 128, kKvDk = 192;

struct KvSmem {
  uint64_t kv_full, kv_empty, ch_full[2], ch_empty[2];
  uint64_t s_full, s_free, pd_full[2], pd_free[2], acc_free, drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int G>
__global__ void __launch_bounds__(kKvThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const KvArgs a, DevCtx ctx) {
  constexpr int TPT = 128 / G;  // query tokens (of G rows each) per chunk
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sK = base;
  uint8_t* sV = sK + kKvBlk;
  uint8_t* sCh = sV + kKvBlk;                 // 2 stages: Q rows, then dO rows
  uint8_t* sPd = sCh + 2 * kKvChunk;          // 2 buffers: P, then dS
  KvSmem& sm = *reinterpret_cast<KvSmem*>(sPd + 2 * kKvPd);
  const int warp = warp_id(), lane = lane_id();
  const int bgn = a.B * a.Hkv;
  const int64_t n_slots = static_cast<int64_t>(bgn) * a.mi;

  if (threadIdx.x == 0) {
    mbar_init(&sm.kv_full, 1);
    mbar_init(&sm.kv_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.ch_full[s], 1);
      mbar_init(&sm.ch_empty[s], 1);
      mbar_init(&sm.pd_full[s], 8);
      mbar_init(&sm.pd_free[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.s_free, 8);
    mbar_init(&sm.acc_free, 8);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  // slot k: item k % mi of (b, g) = k / mi, if that (b, g) has so many
  auto slot = [&](int64_t k, int& bg, int4& it) -> bool {
    bg = static_cast<int>(k / a.mi);
    const int local = static_cast<int>(k % a.mi);
    if (local >= __ldg(a.icnt + bg)) return false;
    it = __ldg(a.items + k);
    return it.z > it.y;
  };

  if (warp == 0) {
    if (lane == 0) {
      int ik = 0;
      int64_t gc = 0;
      bool ok = true;
      for (int64_t k = blockIdx.x; ok && k < n_slots; k += gridDim.x) {
        int bg;
        int4 it;
        if (!slot(k, bg, it)) continue;
        const int b = bg / a.Hkv, g = bg % a.Hkv;
        if (ik >= 1 && !(ok = bwd_wait(&sm.kv_empty, (ik - 1) & 1, ctx, abort_flag))) break;
        mbar_arrive_expect_tx(&sm.kv_full, 2 * kKvBlk);
        for (int h = 0; h < 2; ++h) {
          tma_load_4d(sK + h * 8192, &tmK, &sm.kv_full, 64 * h, g, it.x * kBlock, b);
          tma_load_4d(sV + h * 8192, &tmV, &sm.kv_full, 64 * h, g, it.x * kBlock, b);
        }
        ++ik;
        const int32_t* L = a.list + bg * a.list_len;
        const int n_ch = (it.z - it.y + TPT - 1) / TPT;
        for (int c = 0; c < n_ch; ++c, ++gc) {
          const int s = static_cast<int>(gc & 1);
          if (gc >= 2 && !(ok = bwd_wait(&sm.ch_empty[s], ((gc >> 1) & 1) ^ 1, ctx, abort_flag)))
            break;
          mbar_arrive_expect_tx(&sm.ch_full[s], kKvChunk);
          uint8_t* q = sCh + s * kKvChunk;
          for (int i = 0; i < TPT; ++i) {
            // padding slots repeat the item's last row (masked by the softmax)
            const int p = min(it.y + c * TPT + i, it.z - 1);
            const int qtok = __ldg(L + p);
            for (int h = 0; h < 2; ++h) {
              tma_load_4d(q + h * 16384 + i * G * 128, &tmQ, &sm.ch_full[s], 64 * h, g * G, qtok, b);
              tma_load_4d(q + kKvChunk / 2 + h * 16384 + i * G * 128, &tmdO, &sm.ch_full[s], 64 * h,
                          g * G, qtok, b);
            }
          }
        }
      }
      if (ik > 0) mbar_wait(&sm.kv_full, (ik - 1) & 1, ctx.wait_ns);
      for (int64_t q = gc - 1; q >= 0 && q >= gc - 2; --q)
        mbar_wait(&sm.ch_full[q & 1], (q >> 1) & 1, ctx.wait_ns);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = instr_desc_bf16(128, 64, 0, 0);
      constexpr uint32_t idesc_acc = instr_desc_bf16(128, 64, 1, 1);
      const uint32_t k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      int ik = 0;
      int64_t gc = 0;
      bool ok = true;
      // dV^T += dO^T P and dK^T += Q^T dS of chunk q: A = dO^T / Q^T
      // (MN-major, 128-byte swizzle: 16 rows = 2 KB, channel halves 16 KB
      // apart); B = P / dS (MN-major, no swizzle: 8-row groups 128 B apart,
      // 8-key groups 2 KB apart)
      auto issue_acc = [&](int64_t q, bool first) -> bool {
        if (!bwd_wait(&sm.pd_full[q & 1], static_cast<uint32_t>((q >> 1) & 1), ctx, abort_flag))
          return false;
        if (first && ik > 1 && !bwd_wait(&sm.acc_free, (ik - 2) & 1, ctx, abort_flag)) return false;
        tc_fence_after();
        const uint32_t ch = smem_u32(sCh + (q & 1) * kKvChunk);
        const uint32_t pd = smem_u32(sPd + (q & 1) * kKvPd);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bp = smem_desc(pd + kk * 256, 128, 2048, 0);
          umma_bf16(tmem + kKvDv, smem_desc(ch + kKvChunk / 2 + kk * 2048, 16384, 1024, 2), bp,
                    idesc_acc, (first && kk == 0) ? 0u : 1u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t bs = smem_desc(pd + kKvPd / 2 + kk * 256, 128, 2048, 0);
          umma_bf16(tmem + kKvDk, smem_desc(ch + kk * 2048, 16384, 1024, 2), bs, idesc_acc,
                    (first && kk == 0) ? 0u : 1u);
        }
        umma_commit(&sm.ch_empty[q & 1]);
        umma_commit(&sm.pd_free[q & 1]);
        return true;
      };
      for (int64_t k = blockIdx.x; ok && k < n_slots; k += gridDim.x) {
        int bg;
        int4 it;
        if (!slot(k, bg, it)) continue;
        if (!(ok = bwd_wait(&sm.kv_full, ik & 1, ctx, abort_flag))) break;
        ++ik;
        const int n_ch = (it.z - it.y + TPT - 1) / TPT;
        for (int c = 0; ok && c < n_ch; ++c, ++gc) {
          if (!(ok = bwd_wait(&sm.ch_full[gc & 1], (gc >> 1) & 1, ctx, abort_flag))) break;
          if (gc > 0 && !(ok = bwd_wait(&sm.s_free, static_cast<uint32_t>((gc - 1) & 1), ctx, abort_flag)))
            break;
          tc_fence_after();
          const uint32_t ch = smem_u32(sCh + (gc & 1) * kKvChunk);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
            umma_bf16(tmem + kKvS, smem_desc(ch + off, 16, 1024, 2),
                      smem_desc(k_addr + koff, 16, 1024, 2), idesc_s, kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t koff = (kk >> 2) * 8192 + (kk & 3) * 32;
            umma_bf16(tmem + kKvP, smem_desc(ch + kKvChunk / 2 + off, 16, 1024, 2),
                      smem_desc(v_addr + koff, 16, 1024, 2), idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(&sm.s_full);
          if (c == n_ch - 1) umma_commit(&sm.kv_empty);
          if (c > 0) ok = issue_acc(gc - 1, c == 1);
        }
        if (ok) ok = issue_acc(gc - 1, n_ch == 1);
      }
      umma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, ctx.wait_ns);
    }
  } else {
    // softmax warps: warpgroup hf owns keys 32 hf .. 32 hf + 31 of the block;
    // thread = TMEM lane = gathered row (token slot r / G, head r % G); in
    // the accumulators a lane is a channel d
    const int hf = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int slot_i = r / G, h = r % G;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    // P / dS image (MN-major, no swizzle): row r, key n at
    // (n/8)*2048 + (r/8)*128 + (r%8)*16 + (n%8)*2
    const int row_off = (r >> 3) * 128 + (r & 7) * 16;
    int64_t gc = 0;
    bool ok = true;
    for (int64_t k = blockIdx.x; ok && k < n_slots; k += gridDim.x) {
      int bg;
      int4 it;
      if (!slot(k, bg, it)) continue;
      const int b = bg / a.Hkv, g = bg % a.Hkv;
      const int32_t* L = a.list + bg * a.list_len;
      const int key0 = it.x * kBlock + 32 * hf;
      const int n_ch = (it.z - it.y + TPT - 1) / TPT;
      for (int c = 0; c < n_ch; ++c, ++gc) {
        const int p = it.y + c * TPT + slot_i;
        const bool row_ok = p < it.z;
        const int qtok = row_ok ? __ldg(L + p) : 0;
        const int t = a.q0 + qtok;
        const int64_t lrow = (static_cast<int64_t>(b) * a.Hq + g * G + h) * a.Tq + qtok;
        const float lse2 = row_ok ? __ldg(a.lse + lrow) * kLog2e : 0.f;
        const float Dr = row_ok ? __ldg(a.D + lrow) : 0.f;
        ok = __all_sync(0xffffffffu, bwd_wait(&sm.s_full, static_cast<uint32_t>(gc & 1), ctx, abort_flag));
        if (!ok) break;
        tc_fence_after();
        float x[32], y[32];
        tmem_ld32(lane_addr + kKvS + 32 * hf, x);
        tmem_ld32(lane_addr + kKvP + 32 * hf, y);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.s_free);
        uint32_t pp[16], dd[16];
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) {
          float pv[2], dv[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int n = 2 * cc + u;
            const bool valid = row_ok && key0 + n <= t;
            pv[u] = valid ? fast_exp2(fmaf(x[n], a.scale_log2, -lse2)) : 0.f;
            dv[u] = pv[u] * (y[n] - Dr);
          }
          __nv_bfloat162 p2 = __floats2bfloat162_rn(pv[0], pv[1]);
          __nv_bfloat162 d2 = __floats2bfloat162_rn(dv[0], dv[1]);
          pp[cc] = *reinterpret_cast<uint32_t*>(&p2);
          dd[cc] = *reinterpret_cast<uint32_t*>(&d2);
        }
        // the buffer of chunk gc-2 must have been read by its MMAs
        if (gc >= 2) {
          ok = __all_sync(0xffffffffu, bwd_wait(&sm.pd_free[gc & 1],
                                                static_cast<uint32_t>(((gc >> 1) & 1) ^ 1), ctx, abort_flag));
          if (!ok) break;
        }
        uint8_t* buf = sPd + (gc & 1) * kKvPd;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int n8 = 4 * hf + j;  // 8-key group of the block
          *reinterpret_cast<uint4*>(buf + n8 * 2048 + row_off) =
              make_uint4(pp[4 * j], pp[4 * j + 1], pp[4 * j + 2], pp[4 * j + 3]);
          *reinterpret_cast<uint4*>(buf + kKvPd / 2 + n8 * 2048 + row_off) =
              make_uint4(dd[4 * j], dd[4 * j + 1], dd[4 * j + 2], dd[4 * j + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.pd_full[gc & 1]);
      }
      if (!ok) break;
      // epilogue: the item's dV and dK partials (lane = channel d)
      ok = __all_sync(0xffffffffu, bwd_wait(&sm.pd_free[(gc - 1) & 1],
                                            static_cast<uint32_t>(((gc - 1) >> 1) & 1), ctx, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float* part = a.part + static_cast<int64_t>(k) * 2 * kBlock * kHeadDim;
#pragma unroll
      for (int m = 0; m < 2; ++m) {
        float v[32];
        tmem_ld32(lane_addr + (m ? kKvDk : kKvDv) + 32 * hf, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          part[(static_cast<int64_t>(m) * kBlock + 32 * hf + j) * kHeadDim + r] = v[j];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_free);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// Sums each block's item partials in list order into dK (times the scale)
// and dV; blocks no row selected get zeros.  One CTA per (b, g, block).
__global__ void __launch_bounds__(256) bwd_reduce_kernel(
    const float* __restrict__ part, const int32_t* __restrict__ cnt,
    const int32_t* __restrict__ ioff, float* __restrict__ dK, float* __restrict__ dV, int Hkv,
    int T, int nb, int nb_all, int mi, float scale) {
  const int64_t bg = blockIdx.x / nb_all;
  const int kb = static_cast<int>(blockIdx.x % nb_all);
  const int b = static_cast<int>(bg / Hkv), g = static_cast<int>(bg % Hkv);
  const int c = kb < nb ? cnt[bg * nb + kb] : 0;
  const int ni = (c + kSeg - 1) / kSeg;
  const int i0 = kb < nb ? ioff[bg * nb + kb] : 0;
  for (int e = threadIdx.x; e < kBlock * kHeadDim; e += blockDim.x) {
    const int key = kb * kBlock + e / kHeadDim, d = e % kHeadDim;
    if (key >= T) break;
    float sv = 0.f, sk = 0.f;
    for (int s = 0; s < ni && i0 + s < mi; ++s) {
      const float* pp = part + (bg * mi + i0 + s) * 2 * kBlock * kHeadDim;
      sv += pp[e];
      sk += pp[kBlock * kHeadDim + e];
    }
    const int64_t o = ((static_cast<int64_t>(b) * T + key) * Hkv + g) * kHeadDim + d;
    dV[o] = sv;
    dK[o] = sk * scale;
  }
}

template <int G>
int launch_bwd_g(const Geometry& g, const BwdLayout& L, const void* Q, const void* K, const void* V,
                 const int32_t* idx, const float* lse, const void* dO, float* dQ, float* dK,
                 float* dV, uint8_t* ws, const DevCtx& ctx, cudaStream_t st) {
  // tensor maps: Q / dO rows, one token's G heads or a tile's 128/G tokens
  CUtensorMap tq, tdo, tqr, tdor, tk, tv;
  const uint64_t qd[4] = {static_cast<uint64_t>(kHeadDim), static_cast<uint64_t>(g.Hq),
                          static_cast<uint64_t>(g.Tq), static_cast<uint64_t>(g.B)};
  const uint64_t qs[3] = {static_cast<uint64_t>(kHeadDim) * 2,
                          static_cast<uint64_t>(g.Hq) * kHeadDim * 2,
                          static_cast<uint64_t>(g.Tq) * g.Hq * kHeadDim * 2};
  const uint32_t tile_box[4] = {64u, static_cast<uint32_t>(G), static_cast<uint32_t>(128 / G), 1u};
  const uint32_t row_box[4] = {64u, static_cast<uint32_t>(G), 1u, 1u};
  if (int e = make_tmap_bf16_4d(&tq, Q, qd, qs, tile_box)) return e;
  if (int e = make_tmap_bf16_4d(&tdo, dO, qd, qs, tile_box)) return e;
  if (int e = make_tmap_bf16_4d(&tqr, Q, qd, qs, row_box)) return e;
  if (int e = make_tmap_bf16_4d(&tdor, dO, qd, qs, row_box)) return e;
  const uint64_t kd[4] = {static_cast<uint64_t>(kHeadDim), static_cast<uint64_t>(g.Hkv),
                          static_cast<uint64_t>(g.T), static_cast<uint64_t>(g.B)};
  const uint64_t ks[3] = {static_cast<uint64_t>(kHeadDim) * 2,
                          static_cast<uint64_t>(g.Hkv) * kHeadDim * 2,
                          static_cast<uint64_t>(g.T) * g.Hkv * kHeadDim * 2};
  const uint32_t kbox[4] = {64u, 1u, static_cast<uint32_t>(kBlock), 1u};
  if (int e = make_tmap_bf16_4d(&tk, K, kd, ks, kbox)) return e;
  if (int e = make_tmap_bf16_4d(&tv, V, kd, ks, kbox)) return e;
  const int grid = sm_count();
  float* D = reinterpret_cast<float*>(ws + L.off_D);
  // dQ
  {
    DqArgs a{};
    a.dQ = dQ;
    a.lse = lse;
    a.D = D;
    if (int e = launch_union_build(g, idx, ws + L.off_union, &a.ulist, &a.ucount, &a.ustride, st))
      return e;
    a.B = g.B;
    a.Hq = g.Hq;
    a.Hkv = g.Hkv;
    a.q0 = g.q0;
    a.Tq = g.Tq;
    a.scale = g.scale;
    a.scale_log2 = g.scale_log2;
    const size_t smem = 1024 + 2 * kDqQ + 2 * kDqStage + sizeof(DqSmem);
    static std::atomic<uint64_t> smem_set{0};
    if (int e = set_smem_limit(bwd_dq_kernel<G>, smem, smem_set)) return e;
    bwd_dq_kernel<G><<<grid, kDqThreads, smem, st>>>(tq, tdo, tk, tv, a, ctx);
    if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
  }
  // inverted index
  const int bgn = g.B * g.Hkv;
  int32_t* H = reinterpret_cast<int32_t*>(ws + L.off_H);
  int32_t* cnt = reinterpret_cast<int32_t*>(ws + L.off_cnt);
  int32_t* off = reinterpret_cast<int32_t*>(ws + L.off_off);
  int32_t* ioff = reinterpret_cast<int32_t*>(ws + L.off_ioff);
  int32_t* icnt = reinterpret_cast<int32_t*>(ws + L.off_icnt);
  int4* items = reinterpret_cast<int4*>(ws + L.off_items);
  int32_t* list = reinterpret_cast<int32_t*>(ws + L.off_list);
  float* part = reinterpret_cast<float*>(ws + L.off_part);
  const size_t nb_smem = static_cast<size_t>(L.nb) * sizeof(int);
  bwd_hist_kernel<<<bgn * L.n_ch, 256, nb_smem, st>>>(idx, H, g.q0, g.Tq, g.topk, L.nb, L.n_ch);
  bwd_scan_kernel<<<bgn, kScanThreads, 0, st>>>(H, cnt, off, ioff, icnt, items, L.nb, L.n_ch, L.mi);
  bwd_fill_kernel<<<bgn * L.n_ch, 256, nb_smem, st>>>(idx, H, off, list, L.list_len, g.q0, g.Tq,
                                                      g.topk, L.nb, L.n_ch);
  if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
  // dK, dV partials, then the in-order sum
  {
    KvArgs a{};
    a.items = items;
    a.icnt = icnt;
    a.mi = L.mi;
    a.list = list;
    a.list_len = L.list_len;
    a.part = part;
    a.lse = lse;
    a.D = D;
    a.B = g.B;
    a.Hq = g.Hq;
    a.Hkv = g.Hkv;
    a.q0 = g.q0;
    a.Tq = g.Tq;
    a.scale_log2 = g.scale_log2;
    const size_t smem = 1024 + 2 * kKvBlk + 2 * kKvChunk + 2 * kKvPd + sizeof(KvSmem);
    static std::atomic<uint64_t> smem_set{0};
    if (int e = set_smem_limit(bwd_dkdv_kernel<G>, smem, smem_set)) return e;
    bwd_dkdv_kernel<G><<<grid, kKvThreads, smem, st>>>(tqr, tdor, tk, tv, a, ctx);
    if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
  }
  const int nb_all = (g.T + kBlock - 1) / kBlock;
  bwd_reduce_kernel<<<bgn * nb_all, 256, 0, st>>>(part, cnt, ioff, dK, dV, g.Hkv, g.T, L.nb, nb_all,
                                                 L.mi, g.scale);
  return cudaGetLastError() == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

}  // namespace

size_t bwd_ws_bytes(const Geometry& g) { return bwd_layout(g).total; }

int launch_sparse_bwd(const Geometry& g, const void* Q, const void* K, const void* V,
                      const int32_t* idx, const void* O, const float* lse, const void* dO, float* dQ,
                      float* dK, float* dV, void* ws, const DevCtx& ctx, cudaStream_t st) {
  if (g.B == 0 || g.Tq == 0) return INFLLMV2_OK;
  const BwdLayout L = bwd_layout(g);
  uint8_t* w = static_cast<uint8_t*>(ws);
  const int64_t rows = static_cast<int64_t>(g.B) * g.Tq * g.Hq;
  bwd_delta_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(O), static_cast<const __nv_bfloat16*>(dO),
      reinterpret_cast<float*>(w + L.off_D), g.B, g.Tq, g.Hq);
  if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
  switch (g.G) {
    case 4: return launch_bwd_g<4>(g, L, Q, K, V, idx, lse, dO, dQ, dK, dV, w, ctx, st);
    case 8: return launch_bwd_g<8>(g, L, Q, K, V, idx, lse, dO, dQ, dK, dV, w, ctx, st);
    case 16: return launch_bwd_g<16>(g, L, Q, K, V, idx, lse, dO, dQ, dK, dV, w, ctx, st);
    default: return INFLLMV2_ERR_UNSUPPORTED;
  }
}

}  // namespace infllmv2
