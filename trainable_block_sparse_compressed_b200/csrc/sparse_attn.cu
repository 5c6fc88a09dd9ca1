// sparse_attn.cu -- block-sparse causal attention over selected key blocks
// (reportify digest, Technical Mechanism: after block selection, attention is
// computed only over the selected key/value subsets), one work item per query
// token: the per-token schedule of the prefill, and the decode step's
// attention.
//
// Work item = one query token t of one (batch, kv head): its G query heads
// share the item's selected blocks.  On i.i.d. data neighbouring tokens share
// almost no blocks, so a query tile of several tokens would multiply tensor
// work by the union size; the kernel therefore runs each token on its own and
// swaps the operands so that the 128-row side of tcgen05.mma is keys:
//
//   S^T[128 keys x 16 heads]  = K_pair (A, K-major)   x Q^T (B, K-major)
//   O^T[128 d    x 16 heads]  = V_pair^T (A, MN-major) x P^T (B, MN-major)
//
// A "pair" is two selected 64-key blocks gathered into one 128-row operand:
// from the packed tiles of pack.cu (one 16 KB bulk copy per block and
// tensor, already in the MMA's canonical layout) or, without a workspace and
// in decode mode, by TMA boxes straight from K and V (2 boxes of 64 rows x
// 128 B per block and tensor, 128-byte swizzle).  Heads beyond G are padding.
// Persistent CTAs (one per SM) stream the pairs of their items without
// draining between items.  Queries may be a chunk q0 .. q0+Tq-1 of a longer
// sequence (chunked prefill); keys are addressed by their absolute position.
//
// What bounds this kernel is shared memory: every pair moves 64 KB from L2
// into shared memory through the SM's copy engine, and the tensor core reads
// the same 64 KB back as the A operands of S and P V.  K and V of a pair share
// one 64 KB stage of a 3-stage ring, requested together by one producer and
// released after the pair's P V.  Two threads issue the MMAs, one the S
// products and one the P V products, each in pair order with blocking waits:
// issuing a tcgen05.mma holds its thread for about as long as the tensor core
// takes to read the operand, and a barrier wait costs a few hundred cycles
// even when already complete, so one issuer alone could not keep up.  Each
// issuer waits only for what no other wait implies: the S issuer for its
// stage (S has four TMEM buffers, and a refilled stage means the softmax has
// read S four pairs back), the P V issuer for P (written only after the
// softmax read out P V two pairs back, and after S, issued once the stage
// had landed).  The
// softmax is split over two warpgroups by heads (heads 0-7 and 8-15 of the
// same key rows), halving each thread's dependent chain.
//
// Softmax (thread = TMEM lane = key row of S^T, = channel d of O^T, for eight
// heads): each head keeps a reference maximum m that only moves when a score
// exceeds it by more than 8 (log2 units), so the common pair needs a single
// barrier-OR and no cross-lane reduction; P = exp2(s - m) <= 256 stays exact
// enough in bf16.  Each pair's P V lands in one of two TMEM buffers and is
// folded into an fp32 register accumulator with the rescale of its own
// reference, so the accumulator is never rescaled inside tensor memory.
//
// Decode mode: one query token per sequence at t = seqlens[b]; the selected
// blocks of each (sequence, kv head) are split into chunks so that enough
// items exist to occupy every SM, and each item writes an unnormalised
// partial (o, m, l) that decode.cu merges.
#include "common.cuh"
#include "sm100.cuh"

namespace infllmv2 {
namespace {

constexpr int kStages = 3;                           // K+V ring depth
constexpr int kHalves = 2;                           // softmax warpgroups, 8 heads each
constexpr int kHH = 8;                               // heads per warpgroup
constexpr int kSlotBytes = 64 * 128;                 // 64 rows x 128 B (one TMA box)
constexpr int kHalf = 2 * kSlotBytes;                // 128 rows x 64 channels
constexpr int kPairBytes = 2 * kHalf;                // K or V of one pair: 32 KB
constexpr int kStageBytes = 2 * kPairBytes;          // K then V of one pair: 64 KB
constexpr int kQBytes = 16 * 256;                    // 16 rows x 128 channels
constexpr int kPBytes = 16 * 256;                    // 16 heads x 128 keys
constexpr int kSBufs = 4;                            // S^T TMEM buffers (pair q uses q % 4)
constexpr int kSoftmaxThreads = 128 * kHalves;
constexpr int kThreads = 96 + kSoftmaxThreads;       // producer, S issuer, P V issuer, softmax
constexpr uint32_t kTmemCols = 128;                  // S^T x4 (cols 0-63), PV x2 (64-95)
constexpr uint32_t kPVCol = 64;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleSlack = 8.0f;                // log2 units

struct AttnSmem {
  uint64_t full[kStages], empty[kStages];
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[kSBufs];
  uint64_t p_full[2];
  uint64_t pv_full[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  float red[kHalves][4][kHH];   // per-warp head maxima (rescale path)
  float lsum[kHalves][4][kHH];  // per-warp row sums at item end
  int blocks[kMaxTopk];
};

struct AttnArgs {
  const uint8_t* Kp;        // packed K / V tiles (pack.cu), or null: tensor-map gather
  const uint8_t* Vp;
  int nb;                   // blocks per (batch, kv head) of the packed tiles
  const int32_t* idx;       // selected blocks
  __nv_bfloat16* O;         // final output (prefill)
  float* lse;
  float* part;              // decode partials: [items][G][128] o, then [items][G][2] (m, l)
  const int32_t* seqlens;   // decode: query position of each sequence
  int B, T, Hq, Hkv, topk;  // T: key tokens (prefill) or cache capacity (decode)
  int q0, Tq;               // prefill: the queries are tokens q0 .. q0+Tq-1
  int mode;                 // 0 sparse prefill, 2 decode
  int n_chunks, chunk_blocks;
  float scale_log2;
};

struct Item {
  int b, g, t, qtok, cur, e0, n, n_pairs;
  const int32_t* row;  // index row
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
    int nv = 0;
    if (r.t >= 0 && r.t < a.T) nv = count_valid(r.row, a.topk, r.cur, lane);
    r.e0 = c * a.chunk_blocks;
    r.n = max(0, min(a.chunk_blocks, nv - r.e0));
  } else {
    const int64_t per_g = static_cast<int64_t>(a.B) * a.Tq;
    r.g = static_cast<int>(it / per_g);
    const int64_t rem = it % per_g;
    r.b = static_cast<int>(rem / a.Tq);
    r.qtok = static_cast<int>(rem % a.Tq);  // the query's row in Q, O and lse
    r.t = a.q0 + r.qtok;                    // its token position
    r.cur = r.t / kBlock;
    r.e0 = 0;
    r.row = a.idx + ((static_cast<int64_t>(r.b) * a.Hkv + r.g) * a.Tq + r.qtok) * a.topk;
    r.n = count_valid(r.row, a.topk, r.cur, lane);
  }
  r.n_pairs = (r.n + 1) >> 1;
  return r;
}

// The k-th item of this CTA (>= n_items when there is none).  Items are dealt
// in chunks of consecutive ones, chunk j to CTA j % gridDim.x: tokens that
// CTAs process at the same time are then far apart, so they do not all fetch
// the same local blocks from the same L2 lines at once, as they would if
// consecutive tokens went to consecutive CTAs.
// With few items (decode) the chunks shrink to single items so that every
// CTA gets work.
constexpr int kChunkItems = 16;
__device__ __forceinline__ int64_t item_of(int64_t k, int64_t n_items) {
  const int64_t per_cta = n_items / gridDim.x;
  const int64_t c = per_cta >= kChunkItems ? kChunkItems : (per_cta > 1 ? per_cta : 1);
  const int64_t chunk = k / c;
  const int64_t it = (chunk * gridDim.x + blockIdx.x) * c + k % c;
  return it < n_items ? it : n_items;
}

// Block of entry e (0 <= e < n) of an item, from global memory.
__device__ __forceinline__ int item_block(const Item& it, int e) {
  return __ldg(it.row + it.e0 + e);
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, const DevCtx& ctx,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;  // the common case: already complete
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
  uint8_t* sKV = base;                                   // kStages x (K 32 KB, V 32 KB)
  uint8_t* sQ = sKV + kStages * kStageBytes;             // 2 x 4 KB
  uint8_t* sP = sQ + 2 * kQBytes;                        // 2 x 4 KB
  AttnSmem& sm = *reinterpret_cast<AttnSmem*>(sP + 2 * kPBytes);

  const int warp = warp_id(), lane = lane_id();
  const int64_t n_items = args.mode == 2
                              ? static_cast<int64_t>(args.B) * args.Hkv * args.n_chunks
                              : static_cast<int64_t>(args.Hkv) * args.B * args.Tq;
  const float scale_log2 = args.scale_log2;

  // A pair with a single block leaves its second slot stale.  Stale K rows
  // only produce scores that the softmax masks to -inf, but stale V rows are
  // multiplied by P = 0, so they must be finite: zero, once, the V bytes that
  // second blocks occupy in either layout (packed: 16..32 KB of the V pair,
  // boxes: 8..16 KB and 24..32 KB).
  {
    constexpr int kZero = (kPairBytes - kSlotBytes) / 16;  // 8..32 KB of the V pair
    for (int i = threadIdx.x; i < kStages * kZero; i += blockDim.x) {
      const int st = i / kZero, k = i % kZero;
      reinterpret_cast<uint4*>(base + st * kStageBytes + kPairBytes + kSlotBytes)[k] =
          make_uint4(0, 0, 0, 0);
    }
    // query rows past G (padding heads) stay zero as well
    for (int i = threadIdx.x; i < 2 * kQBytes / 16; i += blockDim.x)
      reinterpret_cast<uint4*>(sQ)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.q_full[a], 1);
      mbar_init(&sm.q_empty[a], 1);
      // softmax-side barriers take one arrival per warp: 256 per-thread
      // arrivals per barrier per pair cost shared-memory atomic bandwidth
      // that the copies into the K / V rings need
      mbar_init(&sm.p_full[a], kSoftmaxThreads / 32);
      mbar_init(&sm.pv_full[a], 1);
    }
    for (int a = 0; a < kSBufs; ++a) mbar_init(&sm.s_full[a], 1);
    mbar_init(&sm.drain, 2);  // one commit from each MMA issuer
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
    struct PairLoad {
      int64_t gp;
      int b, g, blk0, blk1;
      bool two;
    };
    // K and V of a pair share one stage and one barrier, requested together.
    // Packed tiles: one 16 KB bulk copy per block, block b of the pair at
    // slot offset 16 KB; otherwise two 64-channel tensor-map boxes per block,
    // 128-byte swizzled, halves 16 KB apart.
    auto issue = [&](const PairLoad& pl) -> bool {
      const int s = static_cast<int>(pl.gp % kStages);
      uint64_t* full = &sm.full[s];
      if (pl.gp >= kStages &&
          !wait_or_abort(&sm.empty[s], ((pl.gp / kStages) & 1) ^ 1, ctx, abort_flag))
        return false;
      const int64_t tile0 = (static_cast<int64_t>(pl.b) * args.Hkv + pl.g) * args.nb;
      mbar_arrive_expect_tx(full, (pl.two ? 8 : 4) * kSlotBytes);
      for (int v = 0; v < 2; ++v) {
        uint8_t* st = sKV + s * kStageBytes + v * kPairBytes;
        const uint8_t* packed = v ? args.Vp : args.Kp;
        const CUtensorMap* tm = v ? &tmV : &tmK;
        for (int slot = 0; slot < (pl.two ? 2 : 1); ++slot) {
          const int blk = slot ? pl.blk1 : pl.blk0;
          // (checked build) a skipped copy leaves the stage short, so the
          // bounded waits on it expire and the kernel aborts cleanly
          if (!INFLLMV2_CHECK(ctx.status, pl.b >= 0 && pl.b < args.B && pl.g >= 0 &&
                                              pl.g < args.Hkv && blk >= 0 &&
                                              static_cast<int64_t>(blk) * kBlock < args.T))
            continue;
          if (packed) {
            bulk_load(st + slot * kHalf, packed + (tile0 + blk) * kHalf, kHalf, full);
          } else {
            tma_load_4d(st + slot * kSlotBytes, tm, full, 0, pl.g, blk * kBlock, pl.b);
            tma_load_4d(st + kHalf + slot * kSlotBytes, tm, full, 64, pl.g, blk * kBlock, pl.b);
          }
        }
      }
      return true;
    };
    int64_t gp = 0;       // pairs issued
    int qk = 0;           // Q loads issued
    bool ok = true;
    for (int64_t k = 0, it; ok && (it = item_of(k, n_items)) < n_items; ++k) {
      const Item item = resolve_item(it, args, lane);
      if (item.n_pairs == 0) continue;
      if (lane == 0) {
        const int qb = qk & 1;
        if (qk >= 2) ok = wait_or_abort(&sm.q_empty[qb], ((qk >> 1) & 1) ^ 1, ctx, abort_flag);
        if (ok) {
          uint8_t* qdst = sQ + qb * kQBytes;
          mbar_arrive_expect_tx(&sm.q_full[qb], G * 256);
          tma_load_4d(qdst, &tmQ, &sm.q_full[qb], 0, item.g * G, item.qtok, item.b);
          tma_load_4d(qdst + 2048, &tmQ, &sm.q_full[qb], 64, item.g * G, item.qtok, item.b);
          ++qk;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      for (int p = 0; ok && p < item.n_pairs; ++p) {
        PairLoad pl;
        pl.gp = gp;
        pl.b = item.b;
        pl.g = item.g;
        pl.blk0 = item_block(item, 2 * p);
        pl.two = 2 * p + 1 < item.n;
        pl.blk1 = pl.two ? item_block(item, 2 * p + 1) : 0;
        if (lane == 0) ok = issue(pl);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (ok) ++gp;
      }
    }
    // drain: never leave with copies of this CTA in flight (matters only when
    // a wait above gave up; otherwise these phases completed long ago)
    if (lane == 0) {
      for (int x = 0; x < 2 && x < qk; ++x)
        mbar_wait(&sm.q_full[x], ((qk - 1 - x) >> 1) & 1, ctx.wait_ns);
      for (int64_t q = gp - 1; q >= 0 && q >= gp - kStages; --q)
        mbar_wait(&sm.full[q % kStages], (q / kStages) & 1, ctx.wait_ns);
    }
  } else if (warp == 1 || warp == 2) {
    // ----------------------------- MMA issuers -----------------------------
    // Issuing a tcgen05.mma holds the issuing thread for about as long as the
    // tensor core takes to read its operand (~70 cycles for 128 x 16 bf16),
    // and a wait on an mbarrier, even one already complete, costs the thread
    // a few hundred cycles.  One thread doing both for S and P V would spend
    // a pair's whole budget, so warp 1 issues the S products and warp 2 the
    // P V products; each one's waits overlap the other's MMAs.  No order
    // between the two streams is needed: S(p) and P V(p-1) touch disjoint
    // TMEM and shared memory, a stage is refilled only after its P V (which
    // follows its S through the softmax), and the softmax folds P V(p) before
    // it overwrites P(p) with P(p+2).  Each warp resolves items together;
    // lane 0 waits and issues.
    const bool pv_role = warp == 2;
    constexpr uint32_t idesc_s = instr_desc_bf16(128, 16, 0, 0);
    constexpr uint32_t idesc_pv = instr_desc_bf16(128, 16, 1, 1);
    int64_t gp = 0;  // pairs issued by this warp
    int qk = 0;      // items whose Q has been used (S issuer)
    bool ok = true;
    for (int64_t k = 0, it; ok && (it = item_of(k, n_items)) < n_items; ++k) {
      const Item item = resolve_item(it, args, lane);
      if (item.n_pairs == 0) continue;
      if (lane == 0 && pv_role) {
        for (int p = 0; ok && p < item.n_pairs; ++p, ++gp) {
          const int a = static_cast<int>(gp & 1);
          const int st = static_cast<int>(gp % kStages);
          // P(q) complete implies everything else P V(q) needs: each softmax
          // warp arrives on p_full(q) only after it has read P V(q-2) out of
          // this TMEM buffer, and after S(q), which was issued once the
          // stage's K and V had landed
          ok = wait_or_abort(&sm.p_full[a], (gp >> 1) & 1, ctx, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sKV + st * kStageBytes + kPairBytes);
          const uint32_t p_addr = smem_u32(sP + a * kPBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // A: V^T, MN-major.  Packed tiles: no swizzle, channel groups 128 B
            // apart (SBO), 8-key groups 2 KB apart (LBO), 16 keys = 4 KB.
            // Boxes: 128-byte swizzle, 16 keys = two 8-row groups (2 KB).
            const uint64_t ad = args.Vp ? smem_desc(v_addr + kk * 4096, 2048, 128, 0)
                                        : smem_desc(v_addr + kk * 2048, kHalf, 1024, 2);
            // B: P^T, MN-major, no swizzle: 8x8 core matrices of 128 B, heads
            // 0-7 / 8-15 128 B apart (SBO), 8-key groups 256 B apart (LBO)
            const uint64_t bd = smem_desc(p_addr + kk * 512, 256, 128, 0);
            umma_bf16(tmem + kPVCol + a * 16, ad, bd, idesc_pv, kk > 0 ? 1u : 0u);
          }
          umma_commit(&sm.pv_full[a]);
          umma_commit(&sm.empty[st]);
        }
      } else if (lane == 0) {
        const int qb = qk & 1;
        ok = wait_or_abort(&sm.q_full[qb], (qk >> 1) & 1, ctx, abort_flag);
        const uint32_t q_addr = smem_u32(sQ + qb * kQBytes);
        for (int p = 0; ok && p < item.n_pairs; ++p, ++gp) {
          const int st = static_cast<int>(gp % kStages);
          // S(q) overwrites the TMEM buffer of S(q-4).  The stage of pair q
          // is refilled only after P V(q-3) completed, which followed P(q-3),
          // which every softmax warp wrote after reading S(q-3): the wait for
          // the stage covers the buffer too.
          const int a = static_cast<int>(gp % kSBufs);
          ok = wait_or_abort(&sm.full[st], (gp / kStages) & 1, ctx, abort_flag);
          if (!ok) break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(sKV + st * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            // packed tiles: K-major, no swizzle, 16 channels = two 128 B
            // core-matrix columns (LBO), 8-row groups 2 KB apart (SBO);
            // boxes: K-major 128-byte swizzle, 64-channel halves 16 KB apart
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            const uint64_t ad = args.Kp ? smem_desc(k_addr + kk * 256, 128, 2048, 0)
                                        : smem_desc(k_addr + off, 16, 1024, 2);
            const uint64_t bd = smem_desc(q_addr + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024, 2);
            umma_bf16(tmem + a * 16, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(&sm.s_full[a]);
          if (p + 1 == item.n_pairs) umma_commit(&sm.q_empty[qb]);
        }
        ++qk;
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (lane == 0) {
      // drain: all MMAs of this thread complete before TMEM is released
      umma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, ctx.wait_ns);
    }
  } else {
    // ------------------------------ softmax ------------------------------
    // two warpgroups on the same items: warpgroup hf owns heads 8hf .. 8hf+7
    const int hf = (warp - 3) >> 2;
    const int quad = warp & 3;       // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;  // key row of S^T and channel d of O^T
    const int gt = threadIdx.x - 96; // index among all softmax threads
    // this thread's TMEM lane, at the first of its warpgroup's eight columns
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + hf * kHH;
    // Every named barrier spans all 256 softmax threads: a decision taken
    // there (rescale, abort) is the same for both warpgroups, so neither can
    // leave the loop while the other waits at a later barrier.
    constexpr uint32_t bar_sync_id = 1, bar_or_id = 2;
    const int slot = r >> 6;         // which block of the pair this key row belongs to
    const int krow = r & 63;
    // P^T (MN-major, no swizzle): key r's heads 8hf..8hf+7 form one 16-byte
    // row of core matrix (r / 8, hf) at (r / 8) * 256 + hf * 128 + (r % 8) * 16
    const uint32_t p_off = (r >> 3) * 256 + hf * 128 + (r & 7) * 16;
    int64_t gp = 0;
    bool ok = true;
    for (int64_t k = 0, it; ok && (it = item_of(k, n_items)) < n_items; ++k) {
      const Item item = resolve_item(it, args, lane);
      // the item's blocks, staged once in shared memory by all 256 threads
      for (int e = gt; e < item.n; e += kSoftmaxThreads)
        sm.blocks[e] = __ldg(item.row + item.e0 + e);
      named_bar_sync(bar_sync_id, kSoftmaxThreads);
      float m[kHH], l[kHH], o[kHH], alpha_prev[kHH];
#pragma unroll
      for (int h = 0; h < kHH; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
        o[h] = 0.f;
        alpha_prev[h] = 0.f;
      }
      for (int p = 0; p <= item.n_pairs; ++p) {
        float alpha[kHH];
        if (p < item.n_pairs) {
          const int a = static_cast<int>(gp % kSBufs);
          const int pb = static_cast<int>(gp & 1);
          if (!*abort_flag && !mbar_wait(&sm.s_full[a], (gp / kSBufs) & 1, ctx.wait_ns)) {
            report_status(ctx.status, INFLLMV2_STATUS_TIMEOUT);
            *abort_flag = 1;
          }
          tc_fence_after();
          float x[kHH];
          tmem_ld8(lane_addr + a * 16, x);
          tmem_ld_wait();
          tc_fence_before();
          const int e = 2 * p + slot;
          const int blk = e < item.n ? sm.blocks[e] : -1;
          const bool valid = blk >= 0 && blk * kBlock + krow <= item.t;
          float s[kHH];
          bool exceed = false;
#pragma unroll
          for (int h = 0; h < kHH; ++h) {
            s[h] = valid ? x[h] * scale_log2 : -INFINITY;
            exceed |= s[h] > m[h] + kRescaleSlack;
          }
          // one barrier decides for the warpgroup: move the references (first
          // pair, or a score far above them) or abort after a timeout.
          // Decisions use barrier-ORed snapshots of the CTA-wide abort flag,
          // which other threads may set at any moment, so that the group's
          // threads never split at a later named barrier.
          const bool ab = *abort_flag != 0;
          if (named_bar_or(bar_or_id, kSoftmaxThreads, exceed || ab)) {
            if (named_bar_or(bar_or_id, kSoftmaxThreads, ab)) {
              ok = false;
              break;
            }
#pragma unroll
            for (int h = 0; h < kHH; ++h) {
              float wm;
              asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(wm) : "f"(s[h]));
              if (lane == 0) sm.red[hf][quad][h] = wm;
            }
            named_bar_sync(bar_sync_id, kSoftmaxThreads);
#pragma unroll
            for (int h = 0; h < kHH; ++h) {
              const float tm = fmaxf(fmaxf(sm.red[hf][0][h], sm.red[hf][1][h]),
                                     fmaxf(sm.red[hf][2][h], sm.red[hf][3][h]));
              const float mn = fmaxf(m[h], tm);
              alpha[h] = fast_exp2(m[h] - mn);
              m[h] = mn;
            }
            named_bar_sync(bar_sync_id, kSoftmaxThreads);  // red[] is rewritten later
          } else {
#pragma unroll
            for (int h = 0; h < kHH; ++h) alpha[h] = 1.f;
          }
          uint32_t pk[4];
#pragma unroll
          for (int h = 0; h < kHH; h += 2) {
            const float p0 = fast_exp2(s[h] - m[h]);
            const float p1 = fast_exp2(s[h + 1] - m[h + 1]);
            l[h] = l[h] * alpha[h] + p0;
            l[h + 1] = l[h + 1] * alpha[h + 1] + p1;
            __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
            pk[h >> 1] = *reinterpret_cast<uint32_t*>(&b2);
          }
          *reinterpret_cast<uint4*>(sP + pb * kPBytes + p_off) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.p_full[pb]);
        }
        if (p > 0) {
          // fold in P V of the previous pair
          const int64_t q = gp - 1;
          const int a = static_cast<int>(q & 1);
          if (!*abort_flag && !mbar_wait(&sm.pv_full[a], (q >> 1) & 1, ctx.wait_ns)) {
            report_status(ctx.status, INFLLMV2_STATUS_TIMEOUT);
            *abort_flag = 1;
          }
          tc_fence_after();
          float pv[kHH];
          tmem_ld8(lane_addr + kPVCol + a * 16, pv);
          tmem_ld_wait();
          tc_fence_before();  // orders this read before P(q+2), see the P V issuer
#pragma unroll
          for (int h = 0; h < kHH; ++h) o[h] = o[h] * alpha_prev[h] + pv[h];
        }
        if (p < item.n_pairs) {
#pragma unroll
          for (int h = 0; h < kHH; ++h) alpha_prev[h] = alpha[h];
          ++gp;
        }
      }
      if (!ok) break;
      // ---- item epilogue: row sums, then final output or decode partial ----
#pragma unroll
      for (int h = 0; h < kHH; ++h) {
        const float ws = warp_sum(l[h]);
        if (lane == 0) sm.lsum[hf][quad][h] = ws;
      }
      if (named_bar_or(bar_or_id, kSoftmaxThreads, *abort_flag)) {
        ok = false;
        break;
      }
      // heads of this warpgroup that exist (G < 16 leaves padding heads)
      const int h_begin = hf * kHH;
      if (args.mode == 2) {
        float* po = args.part + it * (G * kHeadDim);
        float* pml = args.part + n_items * (G * kHeadDim) + it * (2 * G);
#pragma unroll
        for (int h = 0; h < kHH; ++h)
          if (h_begin + h < G) po[(h_begin + h) * kHeadDim + r] = item.n_pairs > 0 ? o[h] : 0.f;
        if (r < kHH && h_begin + r < G) {
          const float L = sm.lsum[hf][0][r] + sm.lsum[hf][1][r] + sm.lsum[hf][2][r] +
                          sm.lsum[hf][3][r];
          float mr = -INFINITY;
#pragma unroll
          for (int h = 0; h < kHH; ++h)
            if (h == r) mr = m[h];
          pml[2 * (h_begin + r)] = item.n_pairs > 0 ? mr : -INFINITY;
          pml[2 * (h_begin + r) + 1] = item.n_pairs > 0 ? L : 0.f;
        }
      } else if (INFLLMV2_CHECK(ctx.status, item.b >= 0 && item.b < args.B && item.qtok >= 0 &&
                                                item.qtok < args.Tq && item.g >= 0 &&
                                                item.g < args.Hkv)) {
        const int64_t orow =
            (static_cast<int64_t>(item.b) * args.Tq + item.qtok) * args.Hq + item.g * G;
#pragma unroll
        for (int h = 0; h < kHH; ++h) {
          if (h_begin + h < G) {
            const float L = sm.lsum[hf][0][h] + sm.lsum[hf][1][h] + sm.lsum[hf][2][h] +
                            sm.lsum[hf][3][h];
            const float val = item.n_pairs > 0 ? o[h] / L : 0.f;
            args.O[(orow + h_begin + h) * kHeadDim + r] = __float2bfloat16_rn(val);
          }
        }
        if (r < kHH && h_begin + r < G) {
          const float L = sm.lsum[hf][0][r] + sm.lsum[hf][1][r] + sm.lsum[hf][2][r] +
                          sm.lsum[hf][3][r];
          float mr = -INFINITY;
#pragma unroll
          for (int h = 0; h < kHH; ++h)
            if (h == r) mr = m[h];
          args.lse[(static_cast<int64_t>(item.b) * args.Hq + item.g * G + h_begin + r) * args.Tq +
                   item.qtok] = item.n_pairs > 0 ? (mr + __log2f(L)) * kLn2 : -INFINITY;
        }
      }
      // lsum and the staged blocks are reused by the next item
      named_bar_sync(bar_sync_id, kSoftmaxThreads);
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
  const size_t smem =
      1024 + kStages * kStageBytes + 2 * kQBytes + 2 * kPBytes + sizeof(AttnSmem);
  static std::atomic<uint64_t> smem_set{0};
  if (int e = set_smem_limit(sparse_attn_kernel<G>, smem, smem_set)) return e;
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
                       const int32_t* idx, void* O, float* lse, const void* packed,
                       const DevCtx& ctx, cudaStream_t st) {
  if (g.B == 0 || g.Tq == 0) return INFLLMV2_OK;
  AttnArgs a{};
  if (packed) {
    a.Kp = static_cast<const uint8_t*>(packed);
    a.Vp = a.Kp + packed_kv_bytes(g) / 2;
    a.nb = (g.T + kBlock - 1) / kBlock;
  }
  a.idx = idx;
  a.O = static_cast<__nv_bfloat16*>(O);
  a.lse = lse;
  a.B = g.B;
  a.T = g.T;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.topk = g.topk;
  a.q0 = g.q0;
  a.Tq = g.Tq;
  a.mode = 0;
  a.scale_log2 = g.scale_log2;
  const int64_t n_items = static_cast<int64_t>(g.B) * g.Hkv * g.Tq;
  return launch_attn(g, Q, g.Tq, K, V, g.T, a, n_items, ctx, st);
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
