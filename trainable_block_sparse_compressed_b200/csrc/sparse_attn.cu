// sparse_attn.cu -- block-sparse causal attention over selected key blocks
// (reportify digest, Technical Mechanism: after block selection, attention is
// computed only over the selected key/value subsets), and the dense causal
// path (every block <= t/64; InfLLM-V2 skill write-up, Architecture
// Overview, dense pathway bullet).
//
// Work item = one query token t of one (batch, kv head): its G query heads
// share the item's selected blocks.  On i.i.d. data neighbouring tokens share
// almost no blocks, so a query tile of several tokens would multiply tensor
// work by the union size; the kernel therefore runs each token on its own and
// swaps the operands so that the 128-row side of tcgen05.mma is keys:
//
//   S^T[128 keys x 16 heads]  = K_pair (A, K-major) x Q^T (B, K-major)
//   O^T[128 d    x 16 heads] += V_pair^T (A, MN-major) x P^T (B, K-major)
//
// A "pair" is two selected 64-key blocks gathered by TMA into one 128-row
// operand (K and V: 4 x 8 KB boxes each).  Heads beyond G are padding.
// Persistent CTAs (one per SM) stream pairs of consecutive items through a
// 3-stage ring without draining between items.
//
// Warp roles: warp 0 = TMA producer, warp 1 = MMA issuer / TMEM owner, warps
// 2-5 = softmax (thread = TMEM lane = key row for S^T, = channel d for O^T).
// Each pair's P V product lands in a fresh TMEM buffer and is folded into an
// fp32 register accumulator with the usual online-softmax rescale, so the
// accumulator never has to be rescaled inside tensor memory.
//
// Decode mode: one query token per sequence at t = seqlens[b]; the selected
// blocks of each (sequence, kv head) are split into chunks so that enough
// items exist to occupy every SM, and each item writes an unnormalised
// partial (o, m, l) that decode.cu merges.
#include "common.cuh"
#include "sm100.cuh"

namespace infllmv2 {
namespace {

constexpr int kStages = 3;
constexpr int kSlotBytes = 64 * 128;                 // 64 rows x 128 B (one box)
constexpr int kHalf = 2 * kSlotBytes;                // 128 rows x 64 channels
constexpr int kStageBytes = 4 * kHalf;               // K (2 halves) + V (2 halves) = 64 KB
constexpr int kQBytes = 16 * 256;                    // 16 rows x 128 channels
constexpr int kPBytes = 16 * 256;                    // 16 heads x 128 keys
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 64;                   // S^T x2, PV x2 (16 columns each)
constexpr float kLn2 = 0.6931471805599453f;

struct AttnSmem {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2];
  uint64_t pv_full[2], pv_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  float red[2][4][16];   // per-warp partial head maxima, double-buffered by pair
  float lsum[4][16];     // per-warp partial row sums at item end
};

struct AttnArgs {
  const int32_t* idx;       // selected blocks (null when dense)
  __nv_bfloat16* O;         // final output (prefill / dense)
  float* lse;
  float* part;              // decode partials: [items][G][128] o, then [items][G][2] (m, l)
  const int32_t* seqlens;   // decode: query position of each sequence
  int B, T, Hq, Hkv, topk;  // T: tokens (prefill) or cache capacity (decode)
  int mode;                 // 0 sparse prefill, 1 dense prefill, 2 decode
  int n_chunks, chunk_blocks;
  float scale_log2;
};

struct Item {
  int b, g, t, qtok, cur, e0, n, n_pairs;
  const int32_t* row;  // index row (null when dense)
};

// Length of the prefix of entries in [0, cur] (warp-collective).
__device__ __forceinline__ int count_valid(const int32_t* __restrict__ row, int topk, int cur,
                                           int lane) {
  int n = 0;
  for (int base = 0; base < topk; base += 32) {
    const int i = base + lane;
    const int v = i < topk ? __ldg(row + i) : -1;
    const bool ok = i < topk && v >= 0 && v <= cur;
    const uint32_t bad = __ballot_sync(0xffffffffu, !ok);
    if (bad) return n + __ffs(bad) - 1;
    n += 32;
  }
  return n;
}

// Resolves work item `it` (warp-collective: every lane gets the same answer).
__device__ __forceinline__ Item resolve_item(int64_t it, const AttnArgs& a, int lane) {
  Item r;
  if (a.mode == 2) {
    const int c = static_cast<int>(it % a.n_chunks);
    const int64_t bg = it / a.n_chunks;
    r.b = static_cast<int>(bg / a.Hkv);
    r.g = static_cast<int>(bg % a.Hkv);
    r.t = a.seqlens[r.b];
    r.qtok = 0;
    r.cur = r.t / kBlock;
    r.row = a.idx + bg * a.topk;
    const int nv = (r.t >= 0 && r.t < a.T) ? count_valid(r.row, a.topk, r.cur, lane) : 0;
    r.e0 = c * a.chunk_blocks;
    r.n = max(0, min(a.chunk_blocks, nv - r.e0));
  } else {
    const int64_t per_g = static_cast<int64_t>(a.B) * a.T;
    r.g = static_cast<int>(it / per_g);
    const int64_t rem = it % per_g;
    r.b = static_cast<int>(rem / a.T);
    r.t = static_cast<int>(rem % a.T);
    r.qtok = r.t;
    r.cur = r.t / kBlock;
    r.e0 = 0;
    if (a.mode == 1) {
      r.row = nullptr;
      r.n = r.cur + 1;
    } else {
      r.row = a.idx + ((static_cast<int64_t>(r.b) * a.Hkv + r.g) * a.T + r.t) * a.topk;
      r.n = count_valid(r.row, a.topk, r.cur, lane);
    }
  }
  r.n_pairs = (r.n + 1) >> 1;
  return r;
}

// Block of entry e (0 <= e < n) of an item.
__device__ __forceinline__ int item_block(const Item& it, int e) {
  return it.row ? __ldg(it.row + it.e0 + e) : it.e0 + e;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, const DevCtx& ctx,
                                              volatile int* abort_flag) {
  if (*abort_flag) return false;
  if (mbar_wait(bar, parity, ctx.wait_ns)) return true;
  report_status(ctx.status, INFLLMV2_STATUS_TIMEOUT);
  *abort_flag = 1;
  return false;
}

template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                       const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnArgs args, DevCtx ctx) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sKV = base;                                   // kStages x 64 KB
  uint8_t* sQ = sKV + kStages * kStageBytes;             // 2 x 4 KB
  uint8_t* sP = sQ + 2 * kQBytes;                        // 2 x 4 KB
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(sP + 2 * kPBytes);

  const int warp = warp_id(), lane = lane_id();
  const int64_t n_items = args.mode == 2
                              ? static_cast<int64_t>(args.B) * args.Hkv * args.n_chunks
                              : static_cast<int64_t>(args.Hkv) * args.B * args.T;
  const float scale_log2 = args.scale_log2;

  // zero the operand buffers once: a pair with a single block leaves its
  // second slot stale, and stale data must be finite (it is multiplied by 0)
  {
    uint4* p = reinterpret_cast<uint4*>(base);
    const int n16 = (kStages * kStageBytes + 2 * kQBytes + 2 * kPBytes) / 16;
    for (int i = threadIdx.x; i < n16; i += blockDim.x) p[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.q_full[a], 1);
      mbar_init(&sm.q_empty[a], 1);
      mbar_init(&sm.s_full[a], 1);
      mbar_init(&sm.s_empty[a], 128);
      mbar_init(&sm.p_full[a], 128);
      mbar_init(&sm.pv_full[a], 1);
      mbar_init(&sm.pv_empty[a], 128);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0) {
    // ------------------------------ producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    int64_t gp = 0;  // global pair counter of this CTA
    int qk = 0;      // items with at least one pair
    int q_issued = 0;
    int64_t kv_issued = 0;
    bool ok = true;
    for (int64_t it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
      const Item item = resolve_item(it, args, lane);
      if (item.n_pairs == 0) continue;
      const int qb = qk & 1;
      if (lane == 0) {
        if (qk >= 2) ok = wait_or_abort(&sm.q_empty[qb], ((qk >> 1) & 1) ^ 1, ctx, abort_flag);
        if (ok) {
          uint8_t* qdst = sQ + qb * kQBytes;
          mbar_arrive_expect_tx(&sm.q_full[qb], G * 256);
          tma_load_4d(qdst, &tmQ, &sm.q_full[qb], 0, item.g * G, item.qtok, item.b);
          tma_load_4d(qdst + 2048, &tmQ, &sm.q_full[qb], 64, item.g * G, item.qtok, item.b);
          ++q_issued;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ++qk;
      for (int p = 0; ok && p < item.n_pairs; ++p, ++gp) {
        const int blk0 = item_block(item, 2 * p);
        const bool two = 2 * p + 1 < item.n;
        const int blk1 = two ? item_block(item, 2 * p + 1) : 0;
        if (lane == 0) {
          const int s = static_cast<int>(gp % kStages);
          if (gp >= kStages)
            ok = wait_or_abort(&sm.kv_empty[s], ((gp / kStages) & 1) ^ 1, ctx, abort_flag);
          if (ok) {
            uint8_t* st = sKV + s * kStageBytes;
            mbar_arrive_expect_tx(&sm.kv_full[s], (two ? 8 : 4) * kSlotBytes);
            for (int slot = 0; slot < (two ? 2 : 1); ++slot) {
              const int r0 = (slot ? blk1 : blk0) * kBlock;
              uint8_t* d = st + slot * kSlotBytes;
              tma_load_4d(d, &tmK, &sm.kv_full[s], 0, item.g, r0, item.b);
              tma_load_4d(d + kHalf, &tmK, &sm.kv_full[s], 64, item.g, r0, item.b);
              tma_load_4d(d + 2 * kHalf, &tmV, &sm.kv_full[s], 0, item.g, r0, item.b);
              tma_load_4d(d + 3 * kHalf, &tmV, &sm.kv_full[s], 64, item.g, r0, item.b);
            }
            ++kv_issued;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    // drain: never leave with copies of this CTA in flight (matters only when
    // a wait above gave up; otherwise these phases completed long ago)
    if (lane == 0) {
      for (int x = 0; x < 2 && x < q_issued; ++x)
        mbar_wait(&sm.q_full[x], ((q_issued - 1 - x) / 2) & 1, ctx.wait_ns);
      for (int x = 0; x < kStages && x < kv_issued; ++x)
        mbar_wait(&sm.kv_full[x], ((kv_issued - 1 - x) / kStages) & 1, ctx.wait_ns);
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer ------------------------------
    // The whole warp walks the items (the index scan is warp-collective);
    // lane 0 waits on barriers and issues the tensor-core work.
    constexpr uint32_t idesc_s = instr_desc_bf16(128, 16, 0, 0);
    constexpr uint32_t idesc_pv = instr_desc_bf16(128, 16, 1, 0);
    int64_t gp = 0;
    int qk = 0;
    bool ok = true;
    bool pv_pending = false;  // P V of pair gp-1 not yet issued
    auto issue_pv = [&](int64_t q) -> bool {
      const int a = static_cast<int>(q & 1);
      const int s = static_cast<int>(q % kStages);
      if (!wait_or_abort(&sm.p_full[a], (q >> 1) & 1, ctx, abort_flag)) return false;
      if (q >= 2 && !wait_or_abort(&sm.pv_empty[a], ((q >> 1) & 1) ^ 1, ctx, abort_flag))
        return false;
      tc_fence_after();
      const uint32_t v_addr = smem_u32(sKV + s * kStageBytes + 2 * kHalf);
      const uint32_t p_addr = smem_u32(sP + a * kPBytes);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint64_t ad = smem_desc(v_addr + k * 2048, kHalf, 1024, 2);
        const uint64_t bd = smem_desc(p_addr + (k >> 2) * 2048 + (k & 3) * 32, 16, 1024, 2);
        umma_bf16(tmem + 32 + a * 16, ad, bd, idesc_pv, k > 0 ? 1u : 0u);
      }
      umma_commit(&sm.pv_full[a]);
      umma_commit(&sm.kv_empty[s]);
      return true;
    };
    for (int64_t it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
      const Item item = resolve_item(it, args, lane);
      if (item.n_pairs == 0) continue;
      const int qb = qk & 1;
      if (lane == 0) {
        ok = wait_or_abort(&sm.q_full[qb], (qk >> 1) & 1, ctx, abort_flag);
        const uint32_t q_addr = smem_u32(sQ + qb * kQBytes);
        for (int p = 0; ok && p < item.n_pairs; ++p, ++gp) {
          const int s = static_cast<int>(gp % kStages);
          const int a = static_cast<int>(gp & 1);
          if (!wait_or_abort(&sm.kv_full[s], (gp / kStages) & 1, ctx, abort_flag) ||
              (gp >= 2 && !wait_or_abort(&sm.s_empty[a], ((gp >> 1) & 1) ^ 1, ctx, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sKV + s * kStageBytes);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t off = (k >> 2) * kHalf + (k & 3) * 32;
            const uint64_t ad = smem_desc(k_addr + off, 16, 1024, 2);
            const uint64_t bd = smem_desc(q_addr + (k >> 2) * 2048 + (k & 3) * 32, 16, 1024, 2);
            umma_bf16(tmem + a * 16, ad, bd, idesc_s, k > 0 ? 1u : 0u);
          }
          umma_commit(&sm.s_full[a]);
          if (p == item.n_pairs - 1) umma_commit(&sm.q_empty[qb]);
          if (pv_pending && !issue_pv(gp - 1)) {
            ok = false;
            break;
          }
          pv_pending = true;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      gp = __shfl_sync(0xffffffffu, gp, 0);
      ++qk;
    }
    if (lane == 0) {
      if (ok && pv_pending) issue_pv(gp - 1);
      // drain: all MMAs of this CTA complete before TMEM is released
      umma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, ctx.wait_ns);
    }
  } else {
    // ------------------------------ softmax ------------------------------
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // key row of S^T and channel d of O^T
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const int slot = r >> 6;         // which block of the pair this key row belongs to
    const int krow = r & 63;
    int64_t gp = 0;
    bool ok = true;
    // P^T operand byte offset of this thread's key column (K-major, 128-byte swizzle)
    const uint32_t p_col = (r >> 6) * 2048 + (krow & 7) * 2;
    for (int64_t it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
      const Item item = resolve_item(it, args, lane);
      float m[16], l[16], o[16], alpha_prev[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
        o[h] = 0.f;
        alpha_prev[h] = 0.f;
      }
      for (int p = 0; p <= item.n_pairs; ++p) {
        float alpha[16];
        if (p < item.n_pairs) {
          const int a = static_cast<int>(gp & 1);
          const bool w = !*abort_flag && mbar_wait(&sm.s_full[a], (gp >> 1) & 1, ctx.wait_ns);
          if (named_bar_or(2, 128, !w)) {
            if (!w) report_status(ctx.status, INFLLMV2_STATUS_TIMEOUT);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          float x[16];
          tmem_ld16(lane_addr + a * 16, x);
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(&sm.s_empty[a]);
          const int e = 2 * p + slot;
          const int blk = e < item.n ? item_block(item, e) : -1;
          const bool valid = blk >= 0 && blk * kBlock + krow <= item.t;
          float s[16];
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            s[h] = valid ? x[h] * scale_log2 : -INFINITY;
            const float wm = warp_max(s[h]);
            if (lane == 0) sm.red[a][quad][h] = wm;
          }
          named_bar_sync(1, 128);
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            const float tm = fmaxf(fmaxf(sm.red[a][0][h], sm.red[a][1][h]),
                                   fmaxf(sm.red[a][2][h], sm.red[a][3][h]));
            const float mn = fmaxf(m[h], tm);
            alpha[h] = fast_exp2(m[h] - mn);
            m[h] = mn;
            const float pr = fast_exp2(s[h] - mn);
            l[h] = l[h] * alpha[h] + pr;
            s[h] = pr;
          }
          // P^T (bf16) into this pair's P buffer: row = head, column = key
          uint8_t* pb = sP + a * kPBytes;
#pragma unroll
          for (int h = 0; h < 16; ++h) {
            const uint32_t off =
                p_col + (h >> 3) * 1024 + (h & 7) * 128 + (((krow >> 3) ^ (h & 7)) << 4);
            *reinterpret_cast<__nv_bfloat16*>(pb + off) = __float2bfloat16_rn(s[h]);
          }
          fence_proxy_async_smem();
          mbar_arrive(&sm.p_full[a]);
        }
        if (p > 0) {
          // fold in P V of the previous pair
          const int64_t q = gp - 1;
          const int a = static_cast<int>(q & 1);
          const bool w = !*abort_flag && mbar_wait(&sm.pv_full[a], (q >> 1) & 1, ctx.wait_ns);
          if (named_bar_or(2, 128, !w)) {
            if (!w) report_status(ctx.status, INFLLMV2_STATUS_TIMEOUT);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          float pv[16];
          tmem_ld16(lane_addr + 32 + a * 16, pv);
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(&sm.pv_empty[a]);
#pragma unroll
          for (int h = 0; h < 16; ++h) o[h] = o[h] * alpha_prev[h] + pv[h];
        }
        if (p < item.n_pairs) {
#pragma unroll
          for (int h = 0; h < 16; ++h) alpha_prev[h] = alpha[h];
          ++gp;
        }
      }
      if (!ok) break;
      // ---- item epilogue: row sums, then final output or decode partial ----
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        const float ws = warp_sum(l[h]);
        if (lane == 0) sm.lsum[quad][h] = ws;
      }
      named_bar_sync(1, 128);
      if (args.mode == 2) {
        float* po = args.part + it * (G * kHeadDim);
        float* pml = args.part + n_items * (G * kHeadDim) + it * (2 * G);
#pragma unroll
        for (int h = 0; h < G; ++h) po[h * kHeadDim + r] = item.n_pairs > 0 ? o[h] : 0.f;
        if (r < G) {
          const float L = sm.lsum[0][r] + sm.lsum[1][r] + sm.lsum[2][r] + sm.lsum[3][r];
          float mr = -INFINITY;
#pragma unroll
          for (int h = 0; h < 16; ++h)
            if (h == r) mr = m[h];
          pml[2 * r] = item.n_pairs > 0 ? mr : -INFINITY;
          pml[2 * r + 1] = item.n_pairs > 0 ? L : 0.f;
        }
      } else {
        const int64_t orow = (static_cast<int64_t>(item.b) * args.T + item.t) * args.Hq + item.g * G;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float L = sm.lsum[0][h] + sm.lsum[1][h] + sm.lsum[2][h] + sm.lsum[3][h];
          const float val = item.n_pairs > 0 ? o[h] / L : 0.f;
          args.O[(orow + h) * kHeadDim + r] = __float2bfloat16_rn(val);
        }
        if (r < G) {
          const float L = sm.lsum[0][r] + sm.lsum[1][r] + sm.lsum[2][r] + sm.lsum[3][r];
          float mr = -INFINITY;
#pragma unroll
          for (int h = 0; h < 16; ++h)
            if (h == r) mr = m[h];
          args.lse[(static_cast<int64_t>(item.b) * args.Hq + item.g * G + r) * args.T + item.t] =
              item.n_pairs > 0 ? (mr + __log2f(L)) * kLn2 : -INFINITY;
        }
      }
      named_bar_sync(1, 128);  // lsum is reused by the next item
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int G>
int launch_attn_g(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                  const AttnArgs& args, int64_t n_items, const DevCtx& ctx, cudaStream_t st) {
  const size_t smem = 1024 + kStages * kStageBytes + 2 * kQBytes + 2 * kPBytes + sizeof(AttnSmem);
  static bool configured = false;
  if (!configured) {
    if (cudaFuncSetAttribute(sparse_attn_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return INFLLMV2_ERR_CUDA;
    configured = true;
  }
  const int64_t grid = n_items < sm_count() ? n_items : sm_count();
  sparse_attn_kernel<G><<<static_cast<unsigned>(grid), kThreads, smem, st>>>(tq, tk, tv, args, ctx);
  return cudaGetLastError() == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

int launch_attn(const Geometry& g, const void* Q, int q_tokens, const void* K, const void* V,
                int kv_tokens, const AttnArgs& args, int64_t n_items, const DevCtx& ctx,
                cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  {
    const uint64_t dims[4] = {static_cast<uint64_t>(kHeadDim), static_cast<uint64_t>(g.Hq),
                              static_cast<uint64_t>(q_tokens), static_cast<uint64_t>(g.B)};
    const uint64_t strides[3] = {static_cast<uint64_t>(kHeadDim) * 2,
                                 static_cast<uint64_t>(g.Hq) * kHeadDim * 2,
                                 static_cast<uint64_t>(q_tokens) * g.Hq * kHeadDim * 2};
    const uint32_t box[4] = {64u, static_cast<uint32_t>(g.G), 1u, 1u};
    if (int e = make_tmap_bf16_4d(&tq, Q, dims, strides, box)) return e;
  }
  {
    const uint64_t dims[4] = {static_cast<uint64_t>(kHeadDim), static_cast<uint64_t>(g.Hkv),
                              static_cast<uint64_t>(kv_tokens), static_cast<uint64_t>(g.B)};
    const uint64_t strides[3] = {static_cast<uint64_t>(kHeadDim) * 2,
                                 static_cast<uint64_t>(g.Hkv) * kHeadDim * 2,
                                 static_cast<uint64_t>(kv_tokens) * g.Hkv * kHeadDim * 2};
    const uint32_t box[4] = {64u, 1u, static_cast<uint32_t>(kBlock), 1u};
    if (int e = make_tmap_bf16_4d(&tk, K, dims, strides, box)) return e;
    if (int e = make_tmap_bf16_4d(&tv, V, dims, strides, box)) return e;
  }
  switch (g.G) {
    case 1: return launch_attn_g<1>(tq, tk, tv, args, n_items, ctx, st);
    case 2: return launch_attn_g<2>(tq, tk, tv, args, n_items, ctx, st);
    case 4: return launch_attn_g<4>(tq, tk, tv, args, n_items, ctx, st);
    case 8: return launch_attn_g<8>(tq, tk, tv, args, n_items, ctx, st);
    case 16: return launch_attn_g<16>(tq, tk, tv, args, n_items, ctx, st);
    default: return INFLLMV2_ERR_UNSUPPORTED;
  }
}

}  // namespace

int launch_sparse_attn(const Geometry& g, const void* Q, const void* K, const void* V,
                       const int32_t* idx, void* O, float* lse, int dense, const DevCtx& ctx,
                       cudaStream_t st) {
  if (g.B == 0 || g.T == 0) return INFLLMV2_OK;
  AttnArgs a{};
  a.idx = idx;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.lse = lse;
  a.B = g.B;
  a.T = g.T;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.topk = g.topk;
  a.mode = dense ? 1 : 0;
  a.scale_log2 = g.scale_log2;
  const int64_t n_items = static_cast<int64_t>(g.B) * g.Hkv * g.T;
  return launch_attn(g, Q, g.T, K, V, g.T, a, n_items, ctx, st);
}

int launch_decode_attn(const Geometry& g, const void* q, const void* Kcache, const void* Vcache,
                       const int32_t* idx, const int32_t* seqlens, float* part, int n_chunks,
                       int chunk_blocks, const DevCtx& ctx, cudaStream_t st) {
  AttnArgs a{};
  a.idx = idx;
  a.part = part;
  a.seqlens = seqlens;
  a.B = g.B;
  a.T = g.T;  // cache capacity
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.topk = g.topk;
  a.mode = 2;
  a.n_chunks = n_chunks;
  a.chunk_blocks = chunk_blocks;
  a.scale_log2 = g.scale_log2;
  const int64_t n_items = static_cast<int64_t>(g.B) * g.Hkv * n_chunks;
  return launch_attn(g, q, 1, Kcache, Vcache, g.T, a, n_items, ctx, st);
}

}  // namespace infllmv2
