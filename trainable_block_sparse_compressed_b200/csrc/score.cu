// score.cu -- block scores for block selection.
//
// For every query token t of a (batch, kv head g) the method needs
//   p[h, j] = softmax_j(scale * q[t,h] . Kc[j])   over the visible windows j < v(t),
//   S[j]    = sum over the query heads h of group g of p[h, j],
//   bs[blk] = max of S over the windows overlapping block blk
// (InfLLM-V2 skill write-up, Architecture Overview, Hardware Kernel bullet:
// scores are summed over the heads of a group; block size 64, Implementation
// Step 2; windows of 32 tokens every 16, Core Concept).  The softmax needs
// each head's log-sum-exp over all visible windows before any probability can
// be summed, so the kernel makes two passes over the compressed keys.
//
// A query tile is 128 rows: 128/G consecutive tokens x the G heads of one
// group, rows ordered (token, head) -- exactly the box a single TMA load of
// the BSHD query tensor produces.  One CTA owns two consecutive query tiles,
// so that every compressed-key tile it streams from L2 (the kernel's bound:
// each CTA reads all the windows its tokens see) serves 256 rows.
// Compressed-key tiles of 128 rows stream through a 2-stage TMA ring.  Both
// passes run tcgen05.mma (bf16 in, fp32 accumulate in tensor memory).  Pass
// 2 runs over K = 2 x 128: each compressed key is the bf16 pair hi + lo, so
// q . Kc = q . hi + q . lo is accumulated in one tile (a single bf16 rounding
// of the keys would move block scores by up to ~1e-2 relative).  Pass 1 only
// needs each row's log-sum-exp, which scales all of that head's
// probabilities by one common factor; the hi plane alone keeps that factor
// within ~2e-4 of exact (a fp64 emulation over the T=2048 and T=32768
// workloads stays inside the selection band on every row), so pass 1 reads
// and multiplies the hi plane only:
//
//   pass 1  D_i = Q_i x Kc^T (M = N = 128, one per query tile): a TMEM lane
//           is a query row; each thread keeps the running max / sum of its
//           row -> per-row LSE, no cross-lane work;
//   pass 2  D = Kc x [Q_0; Q_1]^T (M = 128, N = 256): operands swapped, a
//           TMEM lane is a compressed key j and the thread holds all (token,
//           head) scores of that key, so the group sum over heads is a
//           register sum, and the max-pool over windows 4b-1 .. 4b+3 is two
//           xor-shuffles plus one shuffle-up across neighbouring lanes
//           (neighbouring windows); a block that starts a 32-lane quadrant
//           takes its first window from the previous quadrant's warp by an
//           atomic max in global memory.
//
// Warp roles: warp 0 issues TMA, warp 1 owns TMEM and issues the MMAs, warps
// 2-17 (four warpgroups, two per query tile) run the softmax / pooling
// epilogue.  The accumulator (256 columns) is double-buffered in TMEM so the
// MMAs of tile i+1 overlap the epilogue of tile i.  Block scores go to a
// causally packed fp32 workspace (row t holds t/64 + 1 scores) for the top-k
// kernel.
#include "common.cuh"
#include "sm100.cuh"

namespace infllmv2 {
namespace {

constexpr int kRows = 128;                 // query rows per query tile (M of pass 1)
constexpr int kQT = 2;                     // query tiles per CTA (pass 2: N = 256)
constexpr int kKcTile = 128;               // compressed keys per tile
constexpr int kStages = 2;
constexpr int kHalfBytes = kRows * 64 * 2; // one 64-channel half of a 128-row tile
constexpr int kTileBytes = 2 * kHalfBytes; // 32 KB: one query tile, or one plane of a key tile
constexpr int kQBytes = kQT * kTileBytes;  // both query tiles: [half][tile][row]
constexpr int kKcBytes = 4 * kHalfBytes;   // 64 KB: hi and lo planes of 128 compressed keys
constexpr int kEpiWG = 4;                  // epilogue warpgroups: two per query tile
constexpr int kCW = kQT * 128 / kEpiWG;    // accumulator columns per warpgroup (two chunks of 32)
constexpr int kEpiThreads = 128 * kEpiWG;
constexpr int kThreads = 64 + kEpiThreads;
constexpr uint32_t kAccCols = kQT * 128;   // one accumulator: both query tiles
constexpr uint32_t kTmemCols = 2 * kAccCols;

struct ScoreSmem {
  uint64_t q_full;
  uint64_t kc_full[kStages];
  uint64_t kc_empty[kStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  alignas(16) float nlse2[kQT * kRows];  // per query row: minus the log2-domain LSE
  float part_m[kEpiWG][kRows], part_l[kEpiWG][kRows];  // pass 1: each column half's max / sum
};

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
    score_blocks_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmKc, float* __restrict__ scores,
                        int B, int q0, int Tq, int Hkv, int n_c, float scale_log2,
                        DevCtx ctx) {
  constexpr int TPT = kRows / G;  // tokens per query tile
  constexpr int TPC = 32 / G;     // tokens per 32-column chunk in pass 2 (G <= 32)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* sQ = base;
  uint8_t* sKc = base + kQBytes;
  ScoreSmem& sm = *reinterpret_cast<ScoreSmem*>(base + kQBytes + kKcBytes * kStages);

  // A CTA takes the query tiles 2p and 2p+1 of one (b, g), heaviest (latest)
  // pairs first.  Queries are tokens q0 .. q0+Tq-1 (a whole prefill: q0 = 0);
  // keys and compressed keys cover tokens 0 .. q0+Tq-1.
  const int q_end = q0 + Tq;
  const int n_qt = (Tq + TPT - 1) / TPT;
  const int n_pair = (n_qt + kQT - 1) / kQT;
  const int bg = blockIdx.x % (B * Hkv);
  const int pair = n_pair - 1 - static_cast<int>(blockIdx.x / (B * Hkv));
  const int b = bg / Hkv, g = bg % Hkv;
  const int t0 = q0 + pair * kQT * TPT;  // first token of the CTA
  const int t_last = min(t0 + kQT * TPT - 1, q_end - 1);
  const int v_max = min(n_c, visible_windows(t_last));
  const int n_t = (v_max + kKcTile - 1) / kKcTile;
  const int n_it = 2 * n_t;

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kc_full[s], 1);
      mbar_init(&sm.kc_empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.acc_full[a], 1);
      mbar_init(&sm.acc_empty[a], kEpiThreads / 32);  // one arrival per epilogue warp
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
    // ---------------- TMA producer ----------------
    if (lane == 0 && n_t > 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmKc);
      // query tile i, channel half h at h * 64 KB + i * 32 KB (a tile past
      // the last query token is filled with zeros)
      mbar_arrive_expect_tx(&sm.q_full, kQBytes);
      for (int i = 0; i < kQT; ++i)
        for (int h = 0; h < 2; ++h)
          tma_load_4d(sQ + h * kQT * kHalfBytes + i * kHalfBytes, &tmQ, &sm.q_full, 64 * h, g * G,
                      t0 - q0 + i * TPT, b);
      int issued = 0;
      for (int it = 0; it < n_it; ++it) {
        const int s = it % kStages;
        const int i = it < n_t ? it : it - n_t;
        if (it >= kStages &&
            !wait_or_abort(&sm.kc_empty[s], ((it / kStages) & 1) ^ 1, ctx, abort_flag))
          break;
        uint8_t* dst = sKc + s * kKcBytes;
        // pass 1 needs the hi plane only, pass 2 hi and lo
        const int nbox = it < n_t ? 2 : 4;
        mbar_arrive_expect_tx(&sm.kc_full[s], nbox * kHalfBytes);
        for (int x = 0; x < nbox; ++x)  // hi d[0:64], hi d[64:128], lo d[0:64], lo d[64:128]
          tma_load_4d(dst + x * kHalfBytes, &tmKc, &sm.kc_full[s], 64 * x, g, i * kKcTile, b);
        ++issued;
      }
      // drain: never leave with copies of this CTA in flight (matters only
      // when a wait above gave up; otherwise these phases completed long ago)
      mbar_wait(&sm.q_full, 0, ctx.wait_ns);
      for (int s = 0; s < kStages && s < issued; ++s) {
        const int fills = (issued - 1 - s) / kStages + 1;  // fills of stage s
        mbar_wait(&sm.kc_full[s], (fills - 1) & 1, ctx.wait_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0 && n_t > 0) {
      constexpr uint32_t idesc1 = instr_desc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc2 = instr_desc_bf16(128, kQT * 128, 0, 0);
      bool ok = wait_or_abort(&sm.q_full, 0, ctx, abort_flag);
      const uint32_t q_addr = smem_u32(sQ);
      for (int it = 0; ok && it < n_it; ++it) {
        const int s = it % kStages, a = it & 1;
        if (!wait_or_abort(&sm.kc_full[s], (it / kStages) & 1, ctx, abort_flag)) break;
        if (it >= 2 && !wait_or_abort(&sm.acc_empty[a], ((it >> 1) & 1) ^ 1, ctx, abort_flag))
          break;
        tc_fence_after();
        const uint32_t kc_addr = smem_u32(sKc + s * kKcBytes);
        const uint32_t d = tmem + a * kAccCols;
        if (it < n_t) {
          // pass 1: S_i = Q_i x hi^T (K = 128) into columns i * 128 of the
          // accumulator, for both query tiles
#pragma unroll
          for (int i = 0; i < kQT; ++i)
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t off = ((k >> 2) & 1) * kHalfBytes + (k & 3) * 32;
              const uint64_t qd = smem_desc(
                  q_addr + ((k >> 2) & 1) * kQT * kHalfBytes + i * kHalfBytes + (k & 3) * 32, 16,
                  1024, 2);
              const uint64_t kd = smem_desc(kc_addr + off, 16, 1024, 2);
              umma_bf16(d + i * 128, qd, kd, idesc1, k > 0 ? 1u : 0u);
            }
        } else {
          // pass 2: D = Kc x [Q_0; Q_1]^T (M = 128 keys, N = 256 query rows,
          // K = 2 x 128: q . Kc = q . hi + q . lo); the 256 rows of a channel
          // half are contiguous, so one descriptor spans both tiles
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const uint32_t off = ((k >> 2) & 1) * kHalfBytes + (k & 3) * 32;
            const uint64_t qd =
                smem_desc(q_addr + ((k >> 2) & 1) * kQT * kHalfBytes + (k & 3) * 32, 16, 1024, 2);
            const uint64_t kd = smem_desc(kc_addr + (k >> 3) * kTileBytes + off, 16, 1024, 2);
            umma_bf16(d, kd, qd, idesc2, k > 0 ? 1u : 0u);
          }
        }
        umma_commit(&sm.kc_empty[s]);
        umma_commit(&sm.acc_full[a]);
      }
      // drain: all MMAs of this CTA complete before TMEM is released
      umma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, ctx.wait_ns);
    }
  } else {
    // -------------- epilogue: 16 warps, thread <-> TMEM lane --------------
    // Warpgroup hf reads accumulator columns kCW hf .. kCW hf + kCW - 1 of its
    // lanes, two chunks of 32: in pass 1 half (hf & 1) of the key columns of
    // query tile hf / 2 (a lane is a query row of that tile); in pass 2 the
    // (token, head) columns of tokens (hf & 1) TPT/2 .. of tile hf / 2 (a
    // lane is a compressed key).  Pass 1 keeps a partial running max / sum
    // per row, merged at the end of the pass.
    const int hf = (warp - 2) >> 2;
    const int qi = hf >> 1;          // the warpgroup's query tile
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // TMEM lane this thread reads
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + hf * kCW;
    // the queries' rows of the causally packed workspace, from row q0 on
    const int64_t row0 = score_row_offset(q0);
    const int64_t slab = score_row_offset(q_end) - row0;
    float* srow_base = scores + (static_cast<int64_t>(b) * Hkv + g) * slab;
    constexpr uint32_t bar_sync_all = 1;  // every epilogue thread
    const int tq0 = t0 + qi * TPT;        // first token of the warpgroup's query tile

    // pass-1 row identity
    const int my_t = tq0 + r / G;
    const int my_v = my_t < q_end ? min(n_c, visible_windows(my_t)) : 0;
    float m_run = -INFINITY, l_run = 0.f;

    for (int it = 0; it < n_it; ++it) {
      const int a = it & 1;
      // A wait that gives up sets the abort flag, after which no thread waits
      // again; every epilogue thread still runs all n_it iterations (on
      // whatever the accumulator holds), so the named barriers below are
      // always met by all of them, without a vote per iteration.
      if (!*abort_flag && !mbar_wait(&sm.acc_full[a], (it >> 1) & 1, ctx.wait_ns)) {
        report_status(ctx.status, INFLLMV2_STATUS_TIMEOUT);
        *abort_flag = 1;
      }
#pragma unroll
      for (int c = 0; c < kCW / 32; ++c) {
        tc_fence_after();
        float x[32];
        tmem_ld32(lane_addr + a * kAccCols + 32 * c, x);
        tmem_ld_wait();
        if (c == kCW / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.acc_empty[a]);
        }
        if (it < n_t) {
          // ---- pass 1: running max / sum of row r over its visible windows ----
          const int j0 = it * kKcTile + (hf & 1) * kCW + 32 * c;
          const int nv = min(32, my_v - j0);  // valid columns of this chunk (may be <= 0)
          // windows the row may not see yet weigh exp2(-inf) = 0; only chunks
          // where a lane of the warp has some pay for the masking
          if (!__all_sync(0xffffffffu, nv >= 32)) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (j >= nv) x[j] = -INFINITY;
          }
          float tm2[2] = {-INFINITY, -INFINITY};
#pragma unroll
          for (int j = 0; j < 32; j += 4) {
            tm2[0] = fmax3(tm2[0], x[j], x[j + 1]);
            tm2[1] = fmax3(tm2[1], x[j + 2], x[j + 3]);
          }
          const float m_new = fmaxf(m_run, fmaxf(tm2[0], tm2[1]));
          if (m_new > -INFINITY) {
            const float2 sl2x2 = make_float2(scale_log2, scale_log2);
            const float2 nmb = make_float2(-m_new * scale_log2, -m_new * scale_log2);
            float2 a2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float2 e = fma2(make_float2(x[j], x[j + 1]), sl2x2, nmb);
              a2[(j >> 1) & 1] = add2(a2[(j >> 1) & 1], make_float2(fast_exp2(e.x), fast_exp2(e.y)));
            }
            l_run = l_run * fast_exp2((m_run - m_new) * scale_log2) +
                    ((a2[0].x + a2[0].y) + (a2[1].x + a2[1].y));
            m_run = m_new;
          }
        } else {
          // ---- pass 2: lane r is compressed key j; columns are (token, head) pairs ----
          const int i = it - n_t;
          const int j = i * kKcTile + r;
          const int tc0 = ((hf & 1) * kCW + 32 * c) / G;  // first token of the chunk in its tile
          float S[TPC];
#pragma unroll
          for (int tl = 0; tl < TPC; ++tl) {
            const int tok = tc0 + tl;
            const int t = tq0 + tok;
            const int v = t < q_end ? min(n_c, visible_windows(t)) : 0;
            float sum;
            if constexpr (G >= 4) {
              // head pairs: one packed FMA for both arguments, one packed add;
              // the heads' -LSE four at a time (one 128-bit shared load)
              const float2 sl2x2 = make_float2(scale_log2, scale_log2);
              const float4* nl = reinterpret_cast<const float4*>(sm.nlse2 + qi * kRows + tok * G);
              float2 a2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
              for (int h = 0; h < G; h += 4) {
                const float4 n4 = nl[h / 4];
                const float2 e0 = fma2(make_float2(x[tl * G + h], x[tl * G + h + 1]), sl2x2,
                                       make_float2(n4.x, n4.y));
                const float2 e1 = fma2(make_float2(x[tl * G + h + 2], x[tl * G + h + 3]), sl2x2,
                                       make_float2(n4.z, n4.w));
                a2[0] = add2(a2[0], make_float2(fast_exp2(e0.x), fast_exp2(e0.y)));
                a2[1] = add2(a2[1], make_float2(fast_exp2(e1.x), fast_exp2(e1.y)));
              }
              sum = (a2[0].x + a2[0].y) + (a2[1].x + a2[1].y);
            } else if constexpr (G == 2) {
              const float2 e = fma2(make_float2(x[2 * tl], x[2 * tl + 1]),
                                    make_float2(scale_log2, scale_log2),
                                    *reinterpret_cast<const float2*>(sm.nlse2 + qi * kRows + 2 * tok));
              sum = fast_exp2(e.x) + fast_exp2(e.y);
            } else {
              sum = fast_exp2(fmaf(x[tl], scale_log2, sm.nlse2[qi * kRows + tok]));
            }
            S[tl] = j < v ? sum : -INFINITY;
          }
          const int blk = i * (kKcTile / 4) + quad * 8 + (lane >> 2);
#pragma unroll
          for (int tl = 0; tl < TPC; ++tl) {
            float m4 = fmaxf(S[tl], __shfl_xor_sync(0xffffffffu, S[tl], 1));
            m4 = fmaxf(m4, __shfl_xor_sync(0xffffffffu, m4, 2));
            const float prev = __shfl_up_sync(0xffffffffu, S[tl], 1);
            const int t = tq0 + tc0 + tl;
            if (t < q_end) {
              const int cur = t / kBlock;
              float* srow = srow_base + score_row_offset(t) - row0;
              // block blk = max over windows 4 blk - 1 .. 4 blk + 3
              if ((lane & 3) == 0 && blk <= cur &&
                  INFLLMV2_CHECK(ctx.status, blk >= 0 && score_row_offset(t) - row0 + blk < slab)) {
                if (lane == 0)  // window 4 blk - 1 is the previous quadrant's
                  atomicMax(reinterpret_cast<int*>(srow + blk), __float_as_int(m4));
                else
                  srow[blk] = fmaxf(m4, prev);
              }
              // this lane's window is the first of block blk + 1, which starts
              // the next quadrant (or tile)
              if (lane == 31 && blk + 1 <= cur &&
                  INFLLMV2_CHECK(ctx.status, score_row_offset(t) - row0 + blk + 1 < slab))
                atomicMax(reinterpret_cast<int*>(srow + blk + 1), __float_as_int(S[tl]));
            }
          }
        }
      }
      if (it == n_t - 1) {
        // merge the two column halves of row r of query tile qi
        if (hf & 1) {
          sm.part_m[hf][r] = m_run;
          sm.part_l[hf][r] = l_run;
        }
        named_bar_sync(bar_sync_all, kEpiThreads);
        if (!(hf & 1)) {
          const float m2 = sm.part_m[hf + 1][r];
          const float mm = fmaxf(m_run, m2);
          float ll = 0.f;
          if (mm > -INFINITY) {
            if (m_run > -INFINITY) ll += l_run * fast_exp2((m_run - mm) * scale_log2);
            if (m2 > -INFINITY) ll += sm.part_l[hf + 1][r] * fast_exp2((m2 - mm) * scale_log2);
          }
          sm.nlse2[qi * kRows + r] = my_v > 0 ? -(mm * scale_log2 + __log2f(ll)) : -INFINITY;
        }
        // Blocks 8k start a 32-lane quadrant of pass 2: their windows come
        // from two warps (the first one is the previous quadrant's last
        // lane), which combine them by atomic max on the score's bits
        // (scores are >= 0 or -inf, so integer order is float order).
        // Start them at -inf.
        for (int e = threadIdx.x - 64; e < kQT * TPT * (t_last / (8 * kBlock) + 1);
             e += kEpiThreads) {
          const int tok = e % (kQT * TPT), k8 = 8 * (e / (kQT * TPT));
          const int t = t0 + tok;
          if (t < q_end && k8 <= t / kBlock &&
              INFLLMV2_CHECK(ctx.status, score_row_offset(t) - row0 + k8 < slab))
            srow_base[score_row_offset(t) - row0 + k8] = -INFINITY;
        }
        named_bar_sync(bar_sync_all, kEpiThreads);
      }
    }
    // blocks past the last compressed-key tile have no visible window, except
    // block 32 n_t (a quadrant start, combined above), whose window before it
    // is the final tile's last
    if (!*abort_flag) {
      for (int tok = hf * (kQT * TPT / kEpiWG) + r; tok < (hf + 1) * (kQT * TPT / kEpiWG);
           tok += 128) {
        const int t = t0 + tok;
        if (t >= q_end) continue;
        const int cur = t / kBlock;
        for (int blk = n_t > 0 ? n_t * (kKcTile / 4) + 1 : 0; blk <= cur; ++blk)
          if (INFLLMV2_CHECK(ctx.status, score_row_offset(t) - row0 + blk < slab))
            srow_base[score_row_offset(t) - row0 + blk] = -INFINITY;
      }
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
int launch_score_g(const Geometry& g, const CUtensorMap& tq, const CUtensorMap& tk, float* scores,
                   const DevCtx& ctx, cudaStream_t st) {
  constexpr int TPT = kRows / G;
  const size_t smem = 1024 + kQBytes + kKcBytes * kStages + sizeof(ScoreSmem);
  static_assert(1024 + kQBytes + kKcBytes * kStages + sizeof(ScoreSmem) <= 227 * 1024,
                "scoring tiles exceed the shared memory of a CTA");
  static std::atomic<uint64_t> smem_set{0};
  if (int e = set_smem_limit(score_blocks_kernel<G>, smem, smem_set)) return e;
  const int n_qt = (g.Tq + TPT - 1) / TPT;
  const unsigned grid = static_cast<unsigned>((n_qt + kQT - 1) / kQT) * g.B * g.Hkv;
  score_blocks_kernel<G><<<grid, kThreads, smem, st>>>(tq, tk, scores, g.B, g.q0, g.Tq, g.Hkv, g.n_c,
                                                       g.scale_log2, ctx);
  return cudaGetLastError() == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

}  // namespace

int launch_score_blocks(const Geometry& g, const void* Q, const void* Kc, float* scores,
                        const DevCtx& ctx, cudaStream_t st) {
  if (g.B == 0 || g.Tq == 0) return INFLLMV2_OK;
  const int TPT = kRows / g.G;
  CUtensorMap tq, tk;
  {
    const uint64_t dims[4] = {static_cast<uint64_t>(kHeadDim), static_cast<uint64_t>(g.Hq),
                              static_cast<uint64_t>(g.Tq), static_cast<uint64_t>(g.B)};
    const uint64_t strides[3] = {static_cast<uint64_t>(kHeadDim) * 2,
                                 static_cast<uint64_t>(g.Hq) * kHeadDim * 2,
                                 static_cast<uint64_t>(g.Tq) * g.Hq * kHeadDim * 2};
    const uint32_t box[4] = {64u, static_cast<uint32_t>(g.G), static_cast<uint32_t>(TPT), 1u};
    if (int e = make_tmap_bf16_4d(&tq, Q, dims, strides, box)) return e;
  }
  {
    // n_c may be 0: give the map one row so that it stays encodable; no
    // tile is loaded in that case.
    const uint64_t rows = g.n_c > 0 ? static_cast<uint64_t>(g.n_c) : 1u;
    const uint64_t dims[4] = {static_cast<uint64_t>(kKcRow), static_cast<uint64_t>(g.Hkv), rows,
                              static_cast<uint64_t>(g.B)};
    const uint64_t strides[3] = {static_cast<uint64_t>(kKcRow) * 2,
                                 static_cast<uint64_t>(g.Hkv) * kKcRow * 2,
                                 rows * g.Hkv * kKcRow * 2};
    const uint32_t box[4] = {64u, 1u, static_cast<uint32_t>(kKcTile), 1u};
    if (int e = make_tmap_bf16_4d(&tk, g.n_c > 0 ? Kc : Q, dims, strides, box)) return e;
  }
  switch (g.G) {
    case 1: return launch_score_g<1>(g, tq, tk, scores, ctx, st);
    case 2: return launch_score_g<2>(g, tq, tk, scores, ctx, st);
    case 4: return launch_score_g<4>(g, tq, tk, scores, ctx, st);
    case 8: return launch_score_g<8>(g, tq, tk, scores, ctx, st);
    case 16: return launch_score_g<16>(g, tq, tk, scores, ctx, st);
    default: return INFLLMV2_ERR_UNSUPPORTED;
  }
}

}  // namespace infllmv2
