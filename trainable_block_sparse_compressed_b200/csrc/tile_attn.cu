// tile_attn.cu -- causal softmax attention over query tiles.
//
// A query tile is 128 rows: the 128/G consecutive tokens x the G query heads
// of one GQA group, the rows that one TMA box of the BSHD query tensor holds.
// Every row of the tile runs over the same stream of key tiles, so each key
// tile is loaded once for 128 rows and both products are full tensor-core
// tiles (tcgen05.mma, M = 128):
//
//   S[128 rows x KT keys] = Q (K-major, 128-byte swizzle) x K_tile^T
//   O[128 rows x 128 d ] += P (tensor memory)            x V_tile (MN-major)
//
// with S double-buffered in tensor memory, P written over its S (the A
// operand straight from tensor memory, so it never touches shared memory) and
// O accumulated in tensor memory, one accumulator per softmax warpgroup.
// Three key streams share the kernel:
//
//   dense      every key 0 .. t: exact dense causal attention (InfLLM-V2 skill
//              write-up, Architecture Overview, the dense pathway bullet);
//              key tiles of 128 keys, the blocks past the tile's last token
//              are not loaded.
//   union      the union of the 64-key blocks the tile's tokens selected, two
//              blocks per key tile, each row masked to its own token's
//              blocks (block-sparse attention over the selected blocks:
//              reportify digest, Technical Mechanism).  A block that several
//              tokens of the tile selected is loaded and multiplied once.
//   compressed the window means Kc, Vc (skill write-up, Core Concept: the
//              compressed pattern aggregates tokens hierarchically); window
//              j is visible to token t iff 16 j + 31 <= t.  Key tiles of 64
//              windows; q . Kc takes both bf16 planes of the compressed key
//              (K = 2 x 128), Vc its high plane.
//
// Warp roles: warp 0 loads Q and the K tiles by TMA (or bulk copies), warp
// 11 the V tiles, each into its own ring (a K stage is released once S has
// read it, a V stage once P V has); warp 1 owns tensor memory and one of its
// threads issues the S products, one thread of warp 10 the P V products.
// Warps 2-9 are the softmax: two warpgroups on the same 128 rows (thread =
// TMEM lane = query row), warpgroup w taking the keys w*KT/2 .. (w+1)*KT/2 - 1
// of every tile (in the union stream: one selected block each), with its own
// running maximum m_w and sum l_w per row and its own O accumulator O_w in
// tensor memory; it writes P_w over its half of S.  The two never wait for
// each other inside an item; at the item's end they merge
// O = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / (l_0 2^(m_0 - M) + l_1 2^(m_1 - M)).
// A row's reference maximum moves only when a score exceeds it by more than
// 8 (log2 units): P = exp2(s - m) <= 256 is exact enough in bf16, and O_w is
// rescaled in tensor memory only on those (rare) moves.  A half whose keys no
// row of its warp may see skips its exponentials.
// Persistent CTAs, one per SM, take the query tiles heaviest first.
#include "common.cuh"
#include "sm100.cuh"

namespace infllmv2 {

constexpr int kTileDense = 0, kTileUnion = 1, kTileCompressed = 2;

// Union lists (tile_attn.cu and its builder): entry = (block, mask of the
// tile's tokens that selected it).
struct TileArgs {
  __nv_bfloat16* O;         // [B, Tq, Hq, 128]
  float* lse;               // [B, Hq, Tq]
  const uint2* ulist;       // union: per query tile, its blocks ascending
  const int32_t* ucount;    // union: entries per query tile
  int ustride;              // union: list capacity per query tile
  const uint8_t* Kp;        // union: K and V repacked into 16 KB block tiles (pack.cu)
  const uint8_t* Vp;
  int nb;                   // union: blocks per (batch, kv head) of the tiles
  int B, Hq, Hkv, q0, Tq;   // queries are tokens q0 .. q0+Tq-1
  int n_c;                  // compressed: windows in Kc / Vc
  float scale_log2;
};

namespace {

template <int MODE>
struct TileCfg {
  static constexpr int KT = MODE == kTileCompressed ? 64 : 128;  // keys per tile
  static constexpr int KP = MODE == kTileCompressed ? 2 : 1;     // bf16 planes of K
  // K/V ring depth and query buffers: the 64 KB key tiles of the dense and
  // union streams take three stages and a single query buffer (a 227 KB
  // budget); the compressed stream's 48 KB tiles leave room for two
  static constexpr int kStages = 3;
  static constexpr int kQBufs = MODE == kTileCompressed ? 2 : 1;
  static constexpr int kBox = 64 * 128;                          // 64 rows x 64 channels
  static constexpr int kKBytes = KP * KT * 256;
  static constexpr int kVBytes = KT * 256;
  static constexpr int kStageBytes = kKBytes + kVBytes;
  static constexpr int kQBytes = 128 * 256;
  static constexpr int H = KT / 2;                               // keys per softmax warpgroup
  // tensor memory: S0, S1 (KT fp32 columns each; P(gt), KT/2 columns of
  // packed bf16 pairs, is written over S(gt)), then O0, O1 (128 each)
  static constexpr uint32_t kOCol = 2 * KT;
  static constexpr uint32_t kTmemCols = 512;
  // warps: Q/K producer, S issuer, softmax x 8, P V issuer, V producer
  static constexpr int kThreads = 64 + 256 + 64;
};

struct TileSmem {
  uint64_t q_full[2], q_empty[2];
  uint64_t k_full[3], k_empty[3], v_full[3], v_empty[3];
  uint64_t s_full[2][2], p_full[2][2], pv_done[2][2];  // [TMEM buffer][warpgroup]
  uint64_t o_free, drain;
  uint32_t tmem_base;
  int abort_flag;
  // at an item's end, for the merge: [0] each warpgroup's reference maximum
  // and [1] its sum, per row
  float xch[2][2][128];
};

constexpr float kTileSlack = 8.0f;   // log2 units
constexpr float kLn2f = 0.6931471805599453f;

struct TileItem {
  int b, g, qt, qtok0, t_last, n_kt, n_u;
  int64_t list;  // union: index of the tile's list
};

template <int G, int MODE>
__device__ __forceinline__ TileItem tile_item(int64_t k, const TileArgs& a, int n_qt) {
  constexpr int TPT = 128 / G;
  using C = TileCfg<MODE>;
  TileItem r;
  const int bgn = a.B * a.Hkv;
  r.qt = n_qt - 1 - static_cast<int>(k / bgn);  // heaviest (latest) tiles first
  const int bg = static_cast<int>(k % bgn);
  r.b = bg / a.Hkv;
  r.g = bg % a.Hkv;
  r.qtok0 = r.qt * TPT;
  r.t_last = a.q0 + min(r.qtok0 + TPT, a.Tq) - 1;
  r.list = static_cast<int64_t>(bg) * n_qt + r.qt;
  r.n_u = 0;
  if (MODE == kTileDense) {
    r.n_kt = r.t_last / C::KT + 1;
  } else if (MODE == kTileUnion) {
    r.n_u = a.ucount[r.list];
    r.n_kt = (r.n_u + 1) >> 1;
  } else {
    const int v = min(a.n_c, visible_windows(r.t_last));
    r.n_kt = (v + C::KT - 1) / C::KT;
  }
  return r;
}

__device__ __forceinline__ bool tile_wait(uint64_t* bar, uint32_t parity, const DevCtx& ctx,
                                          volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  if (*abort_flag) return false;
  if (mbar_wait(bar, parity, ctx.wait_ns)) return true;
  report_status(ctx.status, INFLLMV2_STATUS_TIMEOUT);
  *abort_flag = 1;
  return false;
}

template <int G, int MODE>
__global__ void __launch_bounds__(TileCfg<MODE>::kThreads, 1)
    tile_attn_kernel(const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const TileArgs args, DevCtx ctx) {
  using C = TileCfg<MODE>;
  constexpr int TPT = 128 / G;
  constexpr int KT = C::KT;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  // 128-byte swizzled tiles need 1024-byte alignment; dynamic shared memory
  // starts on a 1 KB boundary (the launch leaves no slack for more)
  uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  if (base != smem_raw) {
    if (threadIdx.x == 0) report_status(ctx.status, INFLLMV2_STATUS_CHECK);
    return;
  }
  uint8_t* sQ = base;                                   // kQBufs x 32 KB
  uint8_t* sKV = sQ + C::kQBufs * C::kQBytes;           // stages: K planes, then V
  TileSmem& sm = *reinterpret_cast<TileSmem*>(sKV + C::kStages * C::kStageBytes);

  const int warp = warp_id(), lane = lane_id();
  const int n_qt = (args.Tq + TPT - 1) / TPT;
  const int64_t n_items = static_cast<int64_t>(args.B) * args.Hkv * n_qt;

  // A key tile may fill only its first block (dense past the last token,
  // union with an odd count).  The softmax gives the other block's keys the
  // weight exp2(s - inf) = 0, which needs finite scores s, and their V rows
  // meet P = 0, which needs finite V: zero every stage once, so that a block
  // never loaded holds zeros and one loaded before holds finite data.
  for (int i = threadIdx.x; i < C::kStages * C::kStageBytes / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(sKV)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
      mbar_init(&sm.s_full[i][0], 1);
      mbar_init(&sm.s_full[i][1], 1);
      mbar_init(&sm.p_full[i][0], 4);  // one arrival per warp of the warpgroup
      mbar_init(&sm.p_full[i][1], 4);
      mbar_init(&sm.pv_done[i][0], 1);
      mbar_init(&sm.pv_done[i][1], 1);
    }
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    mbar_init(&sm.o_free, 8);
    mbar_init(&sm.drain, 2);  // one commit from each MMA issuer
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0 || warp == 11) {
    // ------------------------------ producers -----------------------------
    // Warp 0 loads the query tiles and the K tiles, warp 11 the V tiles.  A
    // K stage is released once S has read it and a V stage once P V has, so
    // the K loads of the next tiles need not wait for the softmax and the
    // P V product of the tile that held the stage.
    const bool v_role = warp == 11;
    if (lane == 0) {
      if (v_role) {
        tma_prefetch_desc(&tmV);
      } else {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
      }
      const CUtensorMap* tm = v_role ? &tmV : &tmK;
      const uint8_t* packed = v_role ? args.Vp : args.Kp;
      int qk = 0;
      int64_t gt = 0;
      bool ok = true;
      for (int64_t k = blockIdx.x; ok && k < n_items; k += gridDim.x) {
        const TileItem it = tile_item<G, MODE>(k, args, n_qt);
        if (it.n_kt == 0) continue;
        if (!v_role) {
          const int qb = qk % C::kQBufs;
          if (qk >= C::kQBufs &&
              !(ok = tile_wait(&sm.q_empty[qb], ((qk / C::kQBufs) & 1) ^ 1, ctx, abort_flag)))
            break;
          mbar_arrive_expect_tx(&sm.q_full[qb], C::kQBytes);
          uint8_t* q = sQ + qb * C::kQBytes;
          tma_load_4d(q, &tmQ, &sm.q_full[qb], 0, it.g * G, it.qtok0, it.b);
          tma_load_4d(q + C::kQBytes / 2, &tmQ, &sm.q_full[qb], 64, it.g * G, it.qtok0, it.b);
          ++qk;
        }
        uint2 ent[2] = {make_uint2(0u, 0u), make_uint2(0u, 0u)};  // union entries of tile i
        if (MODE == kTileUnion) {
          const uint2* L = args.ulist + it.list * args.ustride;
          ent[0] = __ldg(L);
          if (it.n_u > 1) ent[1] = __ldg(L + 1);
        }
        for (int i = 0; i < it.n_kt; ++i, ++gt) {
          const int s = static_cast<int>(gt % C::kStages);
          uint64_t* empty = v_role ? &sm.v_empty[s] : &sm.k_empty[s];
          uint64_t* full = v_role ? &sm.v_full[s] : &sm.k_full[s];
          if (gt >= C::kStages &&
              !(ok = tile_wait(empty, ((gt / C::kStages) & 1) ^ 1, ctx, abort_flag)))
            break;
          uint8_t* dst = sKV + s * C::kStageBytes + (v_role ? C::kKBytes : 0);
          if (MODE == kTileCompressed) {
            // 64 windows: K hi / lo planes x 2 channel halves, or V hi x 2 halves
            const int nbox = v_role ? 2 : 4;
            mbar_arrive_expect_tx(full, nbox * C::kBox);
            for (int x = 0; x < nbox; ++x)
              tma_load_4d(dst + x * C::kBox, tm, full, 64 * x, it.g, i * KT, it.b);
          } else {
            int blk[2];
            int nblk;
            if (MODE == kTileDense) {
              blk[0] = 2 * i;
              blk[1] = 2 * i + 1;
              nblk = blk[1] * kBlock <= it.t_last ? 2 : 1;
            } else {
              blk[0] = static_cast<int>(ent[0].x);
              nblk = 2 * i + 1 < it.n_u ? 2 : 1;
              blk[1] = nblk == 2 ? static_cast<int>(ent[1].x) : 0;
              // the next tile's entries, loaded while this tile's copies fly
              const uint2* L = args.ulist + it.list * args.ustride;
              if (2 * i + 2 < it.n_u) ent[0] = __ldg(L + 2 * i + 2);
              if (2 * i + 3 < it.n_u) ent[1] = __ldg(L + 2 * i + 3);
            }
            mbar_arrive_expect_tx(full, nblk * 2 * C::kBox);
            for (int e = 0; e < nblk; ++e) {
              if (MODE == kTileUnion) {
                // one 16 KB bulk copy per block from the packed tiles
                // (no-swizzle canonical image; block e at e * 16 KB)
                const int64_t tile = (static_cast<int64_t>(it.b) * args.Hkv + it.g) * args.nb + blk[e];
                bulk_load(dst + e * 16384, packed + tile * 16384, 16384, full);
              } else {
                // 128-byte swizzled boxes: half h of block e at h * (KT rows) + e * 64 rows
                for (int h = 0; h < 2; ++h)
                  tma_load_4d(dst + h * KT * 128 + e * C::kBox, tm, full, 64 * h, it.g,
                              blk[e] * kBlock, it.b);
              }
            }
          }
        }
      }
      // drain: never leave with copies of this CTA in flight
      if (!v_role)
        for (int x = 0; x < C::kQBufs && x < qk; ++x)
          mbar_wait(&sm.q_full[(qk - 1 - x) % C::kQBufs], ((qk - 1 - x) / C::kQBufs) & 1,
                    ctx.wait_ns);
      for (int64_t q = gt - 1; q >= 0 && q >= gt - C::kStages; --q)
        mbar_wait(v_role ? &sm.v_full[q % C::kStages] : &sm.k_full[q % C::kStages],
                  (q / C::kStages) & 1, ctx.wait_ns);
    }
  } else if (warp == 1 || warp == 10) {
    // ---------------------------- MMA issuers ----------------------------
    // Issuing a tcgen05.mma holds the issuing thread for about as long as the
    // tensor core takes to read a 128-wide operand, and a barrier wait costs
    // a few hundred cycles even when already complete, so one thread issuing
    // both products of every tile would be the bottleneck.  Warp 1 issues the
    // S products, warp 10 the P V products, each waiting only for what it
    // needs:
    //  - S_w(gt), warpgroup w's half, needs the K tile and its half of the
    //    TMEM buffer, which holds P_w(gt-2) until P V_w(gt-2) has completed;
    //    completion of both halves releases the K tile;
    //  - P V(gt) needs its V tile, first in its item both O accumulators
    //    read out by the previous item's merge, and per warpgroup w its
    //    P_w(gt), which it multiplies into O_w; its completion releases the
    //    V tile.
    if (lane == 0) {
      const bool pv_role = warp == 10;
      constexpr uint32_t idesc_s =
          instr_desc_bf16(128, MODE == kTileCompressed ? KT : C::H, 0, 0);
      constexpr uint32_t idesc_pv = instr_desc_bf16(128, 128, 0, 1);
      int qk = 0, ik = 0;
      int64_t gt = 0;
      bool ok = true;
      for (int64_t k = blockIdx.x; ok && k < n_items; k += gridDim.x) {
        const TileItem it = tile_item<G, MODE>(k, args, n_qt);
        if (it.n_kt == 0) continue;
        if (pv_role) {
          for (int i = 0; ok && i < it.n_kt; ++i, ++gt) {
            if (i == 0 && ik > 0 && !(ok = tile_wait(&sm.o_free, (ik - 1) & 1, ctx, abort_flag)))
              break;
            const int s = static_cast<int>(gt % C::kStages);
            if (!(ok = tile_wait(&sm.v_full[s], (gt / C::kStages) & 1, ctx, abort_flag))) break;
            const uint32_t v_addr = smem_u32(sKV + s * C::kStageBytes + C::kKBytes);
            for (int w = 0; ok && w < 2; ++w) {
              // warpgroup w's P (over its S segment) times the V rows of its keys
              if (!(ok = tile_wait(&sm.p_full[gt & 1][w], static_cast<uint32_t>((gt >> 1) & 1),
                                   ctx, abort_flag)))
                break;
              tc_fence_after();
              const uint32_t p_tmem = tmem + static_cast<uint32_t>(gt & 1) * KT + w * C::H;
              const uint32_t o_tmem = tmem + C::kOCol + static_cast<uint32_t>(w) * 128;
#pragma unroll
              for (int kk = 0; kk < C::H / 16; ++kk) {
                // A = P in tensor memory: 16 keys = 8 columns of bf16 pairs.
                // B = V: MN-major, 128-byte swizzle: 16 keys = 2 KB, the two
                // 64-channel halves KT rows apart.
                // (union: packed tiles, MN-major no swizzle: 8-key groups 2 KB
                // apart, 8-channel groups 128 B apart, 16 keys = 4 KB)
                const int kv = w * (C::H / 16) + kk;  // 16-key step within the tile
                const uint64_t bd = MODE == kTileUnion
                                        ? smem_desc(v_addr + kv * 4096, 2048, 128, 0)
                                        : smem_desc(v_addr + kv * 2048, KT * 128, 1024, 2);
                // the item's first tile starts the accumulator
                umma_bf16_ts(o_tmem, p_tmem + 8 * kk, bd, idesc_pv, (i == 0 && kk == 0) ? 0u : 1u);
              }
              umma_commit(&sm.pv_done[gt & 1][w]);
            }
            if (!ok) break;
            umma_commit(&sm.v_empty[s]);
          }
        } else {
          const int qb = qk % C::kQBufs;
          if (!(ok = tile_wait(&sm.q_full[qb], (qk / C::kQBufs) & 1, ctx, abort_flag))) break;
          const uint32_t q_addr = smem_u32(sQ + qb * C::kQBytes);
          for (int i = 0; ok && i < it.n_kt; ++i, ++gt) {
            const int s = static_cast<int>(gt % C::kStages);
            if (!(ok = tile_wait(&sm.k_full[s], (gt / C::kStages) & 1, ctx, abort_flag))) break;
            const uint32_t k_addr = smem_u32(sKV + s * C::kStageBytes);
            for (int w = 0; ok && w < 2; ++w) {
              // S_w(gt), the half of warpgroup w (N = KT/2 keys), needs its
              // half of the TMEM buffer: P_w(gt-2) until P V_w(gt-2) completed.
              // (Compressed stream: N = KT/2 = 32 would leave the tensor core
              // waiting on issue, so S is one N = KT product after both.)
              if (gt >= 2 && !(ok = tile_wait(&sm.pv_done[gt & 1][w],
                                              static_cast<uint32_t>(((gt >> 1) & 1) ^ 1), ctx,
                                              abort_flag)))
                break;
              if (MODE == kTileCompressed && w == 0) continue;
              const int w0 = MODE == kTileCompressed ? 0 : w;  // first half of the product
              tc_fence_after();
#pragma unroll
              for (int kk = 0; kk < 8 * C::KP; ++kk) {
                // K-major, 128-byte swizzle: 16 channels = 32 B inside a
                // 64-channel half; plane p, half h at (2p + h) * KT rows, the
                // warpgroup's keys w * KT/2 rows further
                const uint32_t off =
                    ((kk >> 2) & 1) * (KT * 128) + (kk & 3) * 32 + w0 * (C::H * 128);
                const uint64_t qd = smem_desc(
                    q_addr + ((kk >> 2) & 1) * (C::kQBytes / 2) + (kk & 3) * 32, 16, 1024, 2);
                // (union: packed tiles, block w at w * 16 KB, K-major no
                // swizzle: 8-channel core matrices 128 B apart, 8-key groups
                // 2 KB apart)
                const uint64_t kd =
                    MODE == kTileUnion
                        ? smem_desc(k_addr + w * 16384 + kk * 256, 128, 2048, 0)
                        : smem_desc(k_addr + (kk >> 3) * (2 * KT * 128) + off, 16, 1024, 2);
                umma_bf16(tmem + static_cast<uint32_t>(gt & 1) * KT + w0 * C::H, qd, kd, idesc_s,
                          kk > 0 ? 1u : 0u);
              }
              if (MODE == kTileCompressed) umma_commit(&sm.s_full[gt & 1][0]);
              umma_commit(&sm.s_full[gt & 1][w]);
            }
            if (!ok) break;
            umma_commit(&sm.k_empty[s]);
            if (i == it.n_kt - 1) umma_commit(&sm.q_empty[qb]);
          }
          ++qk;
        }
        ++ik;
      }
      // drain: every MMA of this thread completes before TMEM is released
      umma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, ctx.wait_ns);
    }
  } else {
    // ------------------------------ softmax ------------------------------
    // Warpgroup w (warps 2-5, 6-9) takes segment w of every key tile (keys
    // w*H .. w*H+H-1: one 64-key block, or 32 windows) for all 128 rows,
    // with its own running maximum and sum per row and its own accumulator
    // O_w, so the two never wait for each other inside an item; P_w is
    // written over the segment's S.  At the item's end the two partial
    // results are merged, each warpgroup writing 64 of the 128 channels.
    constexpr int H = C::H;               // keys per segment
    const int w = (warp - 2) >> 2;
    const int quad = warp & 3;            // TMEM lane quadrant of this warp
    const int r = quad * 32 + lane;       // query row of the tile
    const int tok = r / G, h = r % G;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t o_addr = lane_addr + C::kOCol;
    const float sl2 = args.scale_log2;
    const float2 sl2x2 = make_float2(sl2, sl2);
    // named barriers over the 256 softmax threads, met once per item by both
    // warpgroups, so neither leaves the item loop while the other waits
    constexpr uint32_t bar_sync = 1, bar_or = 2, kSm = 256;
    int64_t gt = 0;
    bool ok = true;
    for (int64_t k = blockIdx.x; ok && k < n_items; k += gridDim.x) {
      const TileItem it = tile_item<G, MODE>(k, args, n_qt);
      const int qtok = it.qtok0 + tok;
      const bool row_ok = qtok < args.Tq;
      const int t = args.q0 + qtok;
      const int64_t orow = (static_cast<int64_t>(it.b) * args.Tq + qtok) * args.Hq + it.g * G + h;
      const int64_t lrow = (static_cast<int64_t>(it.b) * args.Hq + it.g * G + h) * args.Tq + qtok;
      if (it.n_kt == 0) {
        // no visible key for any row of the tile (compressed, t < 31)
        if (row_ok) {
          uint4* o = reinterpret_cast<uint4*>(args.O + orow * kHeadDim + 64 * w);
          for (int c = 0; c < 8; ++c) o[c] = make_uint4(0, 0, 0, 0);
          if (w == 0) args.lse[lrow] = -INFINITY;
        }
        continue;
      }
      // the last key (or, compressed, window count) this row may see
      const int lim = MODE == kTileCompressed ? min(args.n_c, visible_windows(t)) : t + 1;
      float m = -INFINITY, l = 0.f;
      const int64_t gt0 = gt;
      // union stream: this segment's list entry of tile i, loaded one tile
      // ahead so that its latency overlaps the previous tile
      const uint2* ul = args.ulist + it.list * args.ustride + w;
      uint2 e_next = make_uint2(0u, 0u);
      if (MODE == kTileUnion && w < it.n_u) e_next = __ldg(ul);
      bool t_ok = true;
      for (int i = 0; t_ok && i < it.n_kt; ++i) {
        const int64_t g = gt0 + i;
        const uint2 e_cur = e_next;  // an absent second block: entry 0, mask 0
        if (MODE == kTileUnion)
          e_next = 2 * (i + 1) + w < it.n_u ? __ldg(ul + 2 * (i + 1)) : make_uint2(0u, 0u);
        const uint32_t s_addr = lane_addr + static_cast<uint32_t>(g & 1) * KT + w * H;
        const bool s_ok = __all_sync(
            0xffffffffu,
            tile_wait(&sm.s_full[g & 1][w], static_cast<uint32_t>((g >> 1) & 1), ctx, abort_flag));
        // this segment's keys: [lo, lo + H) of a block (dense, union) or
        // window range (compressed); sel: the row's token selected the block
        int lo;
        bool sel = true;
        if (MODE == kTileUnion) {
          sel = ((e_cur.y >> tok) & 1u) != 0u;
          lo = static_cast<int>(e_cur.x) * kBlock;
        } else {
          lo = i * KT + w * H;
        }
        // none: no key of the segment visible to the row; full: every key is
        const bool none = !(row_ok && sel && lo < lim) || !s_ok;
        const bool full = !none && lo + H <= lim;
        const bool any = __any_sync(0xffffffffu, !none);
        const bool diag = __any_sync(0xffffffffu, !none && !full);
        // pass 1: the row's maximum over the segment
        float mx = -INFINITY;
        if (any) {
          float x[H];
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < H / 32; ++c)
            tmem_ld32(s_addr + 32 * c, *reinterpret_cast<float(*)[32]>(x + 32 * c));
          tmem_ld_wait();
          // keys past the row's last visible one: only where a lane of the
          // warp is on its causal diagonal (rows without a visible key in
          // the segment are handled per row, not per key)
          if (diag) {
#pragma unroll
            for (int c = 0; c < H; ++c)
              if (lo + c >= lim) x[c] = -INFINITY;
          }
          float m2[2] = {-INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < H; c += 4) {
            m2[0] = fmax3(m2[0], x[c], x[c + 1]);
            m2[1] = fmax3(m2[1], x[c + 2], x[c + 3]);
          }
          if (!none) mx = fmaxf(m2[0], m2[1]) * sl2;
        }
        // the reference maximum moves only when a score exceeds it by more
        // than the slack (P <= 2^slack stays exact in bf16 and fp32)
        float alpha = 1.f;
        if (mx > m + kTileSlack) {
          alpha = fast_exp2(m - mx);  // 0 while the row had no key
          m = mx;
        }
        // move O_w to the new reference once P V of the previous tile has
        // added into it (the item's first tile overwrites O_w)
        if (i > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
          t_ok = __all_sync(0xffffffffu,
                            tile_wait(&sm.pv_done[(g - 1) & 1][w],
                                      static_cast<uint32_t>(((g - 1) >> 1) & 1), ctx, abort_flag));
          if (!t_ok) break;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            float o[32];
            tmem_ld32(o_addr + 128 * w + 32 * c, o);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const float2 v = mul2(make_float2(o[j], o[j + 1]), make_float2(alpha, alpha));
              o[j] = v.x;
              o[j + 1] = v.y;
            }
            tmem_st32(o_addr + 128 * w + 32 * c, o);
          }
        }
        // pass 2: P = exp2(s - m) as bf16 pairs written over the segment's S
        // (keys 2c, 2c + 1 -> column c; the segment is read first), 32 keys
        // at a time
        float2 s2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
        if (any) {
          float x[H];
#pragma unroll
          for (int c = 0; c < H / 32; ++c)
            tmem_ld32(s_addr + 32 * c, *reinterpret_cast<float(*)[32]>(x + 32 * c));
          tmem_ld_wait();
          if (diag) {
#pragma unroll
            for (int c = 0; c < H; ++c)
              if (lo + c >= lim) x[c] = -INFINITY;
          }
          // a row without a visible key in the segment takes offset -inf, so
          // that every exp2 of it is 0 (its scores are finite: every K row in
          // shared memory is); otherwise m is finite
          const float mo = none ? -INFINITY : -m;
          const float2 mo2 = make_float2(mo, mo);
#pragma unroll
          for (int q = 0; q < H / 32; ++q) {
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) {
              const float2 a = fma2(make_float2(x[32 * q + 2 * c], x[32 * q + 2 * c + 1]), sl2x2, mo2);
              const float2 pp = make_float2(fast_exp2(a.x), fast_exp2(a.y));
              s2[c & 1] = add2(s2[c & 1], pp);  // masked keys: exp2(-inf) = 0
              __nv_bfloat162 b2 = __floats2bfloat162_rn(pp.x, pp.y);
              pk[c] = *reinterpret_cast<uint32_t*>(&b2);
            }
            tmem_st16(s_addr + 16 * q, pk);
          }
        } else {
          uint32_t pk[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) pk[c] = 0u;
#pragma unroll
          for (int q = 0; q < H / 32; ++q) tmem_st16(s_addr + 16 * q, pk);
        }
        l = l * alpha + ((s2[0].x + s2[0].y) + (s2[1].x + s2[1].y));
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && s_ok) mbar_arrive(&sm.p_full[g & 1][w]);
        t_ok = s_ok;
      }
      gt = gt0 + it.n_kt;
      // ---- merge: O = (O_0 2^(m_0 - M) + O_1 2^(m_1 - M)) / L, and the LSE ----
      // P V_1 of the item's last tile completes after all the others (the
      // item's first tile overwrote both accumulators)
      const int64_t gl = gt - 1;
      const bool e_ok = t_ok && __all_sync(0xffffffffu,
                                           tile_wait(&sm.pv_done[gl & 1][1],
                                                     static_cast<uint32_t>((gl >> 1) & 1), ctx,
                                                     abort_flag));
      sm.xch[0][w][r] = m;
      sm.xch[1][w][r] = l;
      if (named_bar_or(bar_or, kSm, !e_ok || *abort_flag != 0)) {
        ok = false;
        break;
      }
      const float m0 = sm.xch[0][0][r], m1 = sm.xch[0][1][r];
      const float M = fmaxf(m0, m1);
      const float c0 = m0 > -INFINITY ? fast_exp2(m0 - M) : 0.f;
      const float c1 = m1 > -INFINITY ? fast_exp2(m1 - M) : 0.f;
      const float L = sm.xch[1][0][r] * c0 + sm.xch[1][1][r] * c1;
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const float2 f0 = make_float2(c0 * inv, c0 * inv), f1 = make_float2(c1 * inv, c1 * inv);
      named_bar_sync(bar_sync, kSm);  // the exchange slots are free for the next item
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float o0[32], o1[32];
        tmem_ld32(o_addr + 64 * w + 32 * c, o0);
        tmem_ld32(o_addr + 128 + 64 * w + 32 * c, o1);
        tmem_ld_wait();
        if (row_ok && INFLLMV2_CHECK(ctx.status, it.b < args.B && it.g < args.Hkv)) {
          uint4* dst = reinterpret_cast<uint4*>(args.O + orow * kHeadDim + 64 * w + 32 * c);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint32_t wd[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int n = 8 * j + 2 * e;
              // a half no key of which the row saw has c = 0 (and O = 0)
              const float2 v = fma2(make_float2(o1[n], o1[n + 1]), f1,
                                    mul2(make_float2(o0[n], o0[n + 1]), f0));
              __nv_bfloat162 b2 = __floats2bfloat162_rn(v.x, v.y);
              wd[e] = *reinterpret_cast<uint32_t*>(&b2);
            }
            dst[j] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
          }
        }
      }
      if (row_ok && w == 0) args.lse[lrow] = L > 0.f ? (M + __log2f(L)) * kLn2f : -INFINITY;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.o_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// union lists: for every query tile (b, g, qt), the blocks its TPT tokens
// selected, ascending, each with the mask of the tokens that selected it.
// One CTA per tile: a token mask per block the tile's tokens may see (in
// shared memory) takes one bit per (token, selected block); the non-empty
// masks are then compacted in block order.
// ---------------------------------------------------------------------------
constexpr int kUnionThreads = 256;

template <int TPT>
__global__ void __launch_bounds__(kUnionThreads) union_build_kernel(
    const int32_t* __restrict__ idx, uint2* __restrict__ ulist, int32_t* __restrict__ ucount,
    int q0, int Tq, int topk, int n_qt) {
  extern __shared__ uint32_t mask[];  // per block 0 .. nbt-1: the tokens that selected it
  __shared__ int scan[kUnionThreads / 32 + 1];
  const int64_t tile = blockIdx.x;
  const int64_t bg = tile / n_qt;
  const int qt = static_cast<int>(tile % n_qt);
  const int t_last = q0 + min((qt + 1) * TPT, Tq) - 1;
  const int nbt = t_last / kBlock + 1;  // blocks the tile's tokens may see
  for (int b = threadIdx.x; b < nbt; b += blockDim.x) mask[b] = 0u;
  __syncthreads();
  const int n = TPT * topk;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int tk = e / topk, j = e % topk;
    const int qtok = qt * TPT + tk;
    if (qtok < Tq) {
      const int v = __ldg(idx + ((bg * Tq + qtok) * topk + j));
      const int t = q0 + qtok;
      if (v >= 0 && v <= t / kBlock) atomicOr(&mask[v], 1u << tk);
    }
  }
  __syncthreads();
  // compaction in block order: thread i takes blocks [i per, (i+1) per)
  const int per = (nbt + kUnionThreads - 1) / kUnionThreads;
  const int b0 = threadIdx.x * per, b1 = min(b0 + per, nbt);
  int nh = 0;
  for (int b = b0; b < b1; ++b) nh += mask[b] != 0u;
  // exclusive scan of the counts over threads
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = nh;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scan[wid] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int w = 0; w < kUnionThreads / 32; ++w) {
      const int v = scan[w];
      scan[w] = acc;
      acc += v;
    }
    scan[kUnionThreads / 32] = acc;
  }
  __syncthreads();
  int pos = scan[wid] + x - nh;
  uint2* L = ulist + tile * static_cast<int64_t>(n);
  for (int b = b0; b < b1; ++b) {
    const uint32_t m = mask[b];
    if (m != 0u) L[pos++] = make_uint2(static_cast<uint32_t>(b), m);
  }
  if (threadIdx.x == 0) ucount[tile] = scan[kUnionThreads / 32];
}

template <int G, int MODE>
int launch_tile_g(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                  const TileArgs& a, const DevCtx& ctx, cudaStream_t st) {
  using C = TileCfg<MODE>;
  constexpr int TPT = 128 / G;
  const size_t smem = C::kQBufs * C::kQBytes + C::kStages * C::kStageBytes + sizeof(TileSmem);
  static std::atomic<uint64_t> smem_set{0};
  if (int e = set_smem_limit(tile_attn_kernel<G, MODE>, smem, smem_set)) return e;
  const int64_t n_items = static_cast<int64_t>(a.B) * a.Hkv * ((a.Tq + TPT - 1) / TPT);
  const int64_t grid = n_items < sm_count() ? n_items : sm_count();
  tile_attn_kernel<G, MODE><<<static_cast<unsigned>(grid), C::kThreads, smem, st>>>(tq, tk, tv, a,
                                                                                  ctx);
  return cudaGetLastError() == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

template <int MODE>
int launch_tile(const Geometry& g, const CUtensorMap& tq, const CUtensorMap& tk,
                const CUtensorMap& tv, const TileArgs& a, const DevCtx& ctx, cudaStream_t st) {
  switch (g.G) {
    case 4: return launch_tile_g<4, MODE>(tq, tk, tv, a, ctx, st);
    case 8: return launch_tile_g<8, MODE>(tq, tk, tv, a, ctx, st);
    case 16: return launch_tile_g<16, MODE>(tq, tk, tv, a, ctx, st);
    default: break;
  }
  if constexpr (MODE != kTileUnion) {  // the union lists' token masks hold 32 tokens
    switch (g.G) {
      case 1: return launch_tile_g<1, MODE>(tq, tk, tv, a, ctx, st);
      case 2: return launch_tile_g<2, MODE>(tq, tk, tv, a, ctx, st);
      default: break;
    }
  }
  return INFLLMV2_ERR_UNSUPPORTED;
}

// Q box: 64 channels x G heads x 128/G tokens.
int q_map(const Geometry& g, const void* Q, CUtensorMap* tq) {
  const uint64_t dims[4] = {static_cast<uint64_t>(kHeadDim), static_cast<uint64_t>(g.Hq),
                            static_cast<uint64_t>(g.Tq), static_cast<uint64_t>(g.B)};
  const uint64_t strides[3] = {static_cast<uint64_t>(kHeadDim) * 2,
                               static_cast<uint64_t>(g.Hq) * kHeadDim * 2,
                               static_cast<uint64_t>(g.Tq) * g.Hq * kHeadDim * 2};
  const uint32_t box[4] = {64u, static_cast<uint32_t>(g.G), static_cast<uint32_t>(128 / g.G), 1u};
  return make_tmap_bf16_4d(tq, Q, dims, strides, box);
}

// K / V box: 64 channels x 64 tokens of one kv head.
int kv_map(const Geometry& g, const void* X, CUtensorMap* tm) {
  const uint64_t dims[4] = {static_cast<uint64_t>(kHeadDim), static_cast<uint64_t>(g.Hkv),
                            static_cast<uint64_t>(g.T), static_cast<uint64_t>(g.B)};
  const uint64_t strides[3] = {static_cast<uint64_t>(kHeadDim) * 2,
                               static_cast<uint64_t>(g.Hkv) * kHeadDim * 2,
                               static_cast<uint64_t>(g.T) * g.Hkv * kHeadDim * 2};
  const uint32_t box[4] = {64u, 1u, static_cast<uint32_t>(kBlock), 1u};
  return make_tmap_bf16_4d(tm, X, dims, strides, box);
}

TileArgs tile_args(const Geometry& g, void* O, float* lse) {
  TileArgs a{};
  a.O = static_cast<__nv_bfloat16*>(O);
  a.lse = lse;
  a.B = g.B;
  a.Hq = g.Hq;
  a.Hkv = g.Hkv;
  a.q0 = g.q0;
  a.Tq = g.Tq;
  a.n_c = g.n_c;
  a.scale_log2 = g.scale_log2;
  return a;
}

}  // namespace

bool union_supported(const Geometry& g) { return g.G >= 4; }

namespace {
int64_t union_tiles(const Geometry& g) {
  const int TPT = 128 / g.G;
  return static_cast<int64_t>(g.B) * g.Hkv * ((g.Tq + TPT - 1) / TPT);
}
size_t union_lists_bytes(const Geometry& g) {
  const size_t b = static_cast<size_t>(union_tiles(g)) * (128 / g.G) * g.topk * sizeof(uint2);
  return (b + 255) & ~static_cast<size_t>(255);
}
}  // namespace

size_t union_lists_ws_bytes(const Geometry& g) {
  if (!union_supported(g) || g.B == 0 || g.Tq == 0) return 0;
  const size_t counts = static_cast<size_t>(union_tiles(g)) * sizeof(int32_t);
  return union_lists_bytes(g) + ((counts + 255) & ~static_cast<size_t>(255));
}

// The query-tile schedule's workspace: the union lists, then K and V
// repacked into block tiles.
size_t union_ws_bytes(const Geometry& g) {
  const size_t lists = union_lists_ws_bytes(g);
  return lists ? lists + packed_kv_bytes(g) : 0;
}

int launch_union_build(const Geometry& g, const int32_t* idx, void* ws, const uint2** ulist,
                       const int32_t** ucount, int* stride, cudaStream_t st) {
  if (!union_supported(g)) return INFLLMV2_ERR_UNSUPPORTED;
  const int TPT = 128 / g.G;
  const int n_qt = (g.Tq + TPT - 1) / TPT;
  const int64_t tiles = union_tiles(g);
  const int n = TPT * g.topk;
  uint2* L = static_cast<uint2*>(ws);
  int32_t* C = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + union_lists_bytes(g));
  // one token mask per block the last query token may see (<= 16 KB within
  // the selection size limit)
  const size_t ush = static_cast<size_t>((g.q0 + g.Tq - 1) / kBlock + 1) * sizeof(uint32_t);
  if (ush > 48 * 1024) return INFLLMV2_ERR_UNSUPPORTED;
  const unsigned grid = static_cast<unsigned>(tiles);
  if (TPT == 8)
    union_build_kernel<8><<<grid, kUnionThreads, ush, st>>>(idx, L, C, g.q0, g.Tq, g.topk, n_qt);
  else if (TPT == 16)
    union_build_kernel<16><<<grid, kUnionThreads, ush, st>>>(idx, L, C, g.q0, g.Tq, g.topk, n_qt);
  else
    union_build_kernel<32><<<grid, kUnionThreads, ush, st>>>(idx, L, C, g.q0, g.Tq, g.topk, n_qt);
  if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
  *ulist = L;
  *ucount = C;
  *stride = n;
  return INFLLMV2_OK;
}

int launch_dense_tile(const Geometry& g, const void* Q, const void* K, const void* V, void* O,
                      float* lse, const DevCtx& ctx, cudaStream_t st) {
  if (g.B == 0 || g.Tq == 0) return INFLLMV2_OK;
  CUtensorMap tq, tk, tv;
  if (int e = q_map(g, Q, &tq)) return e;
  if (int e = kv_map(g, K, &tk)) return e;
  if (int e = kv_map(g, V, &tv)) return e;
  return launch_tile<kTileDense>(g, tq, tk, tv, tile_args(g, O, lse), ctx, st);
}

int launch_union_tile(const Geometry& g, const void* Q, const void* K, const void* V,
                      const int32_t* idx, void* O, float* lse, void* ws, const DevCtx& ctx,
                      cudaStream_t st) {
  if (g.B == 0 || g.Tq == 0) return INFLLMV2_OK;
  TileArgs a = tile_args(g, O, lse);
  if (int e = launch_union_build(g, idx, ws, &a.ulist, &a.ucount, &a.ustride, st)) return e;
  uint8_t* packed = static_cast<uint8_t*>(ws) + union_lists_ws_bytes(g);
  if (int e = launch_pack_kv(g, K, V, packed, st)) return e;
  a.Kp = packed;
  a.Vp = packed + packed_kv_bytes(g) / 2;
  a.nb = (g.T + kBlock - 1) / kBlock;
  CUtensorMap tq, tk, tv;
  if (int e = q_map(g, Q, &tq)) return e;
  if (int e = kv_map(g, K, &tk)) return e;
  if (int e = kv_map(g, V, &tv)) return e;
  return launch_tile<kTileUnion>(g, tq, tk, tv, a, ctx, st);
}

int launch_compressed_tile(const Geometry& g, const void* Q, const void* Kc, const void* Vc,
                           void* O, float* lse, const DevCtx& ctx, cudaStream_t st) {
  if (g.B == 0 || g.Tq == 0) return INFLLMV2_OK;
  CUtensorMap tq, tk, tv;
  if (int e = q_map(g, Q, &tq)) return e;
  // compressed rows [B, n_c, Hkv, 2 planes x 128]; box 64 channels x 64 windows
  const uint64_t rows = g.n_c > 0 ? static_cast<uint64_t>(g.n_c) : 1u;
  const uint64_t dims[4] = {static_cast<uint64_t>(kKcRow), static_cast<uint64_t>(g.Hkv), rows,
                            static_cast<uint64_t>(g.B)};
  const uint64_t strides[3] = {static_cast<uint64_t>(kKcRow) * 2,
                               static_cast<uint64_t>(g.Hkv) * kKcRow * 2,
                               rows * g.Hkv * kKcRow * 2};
  const uint32_t box[4] = {64u, 1u, 64u, 1u};
  if (int e = make_tmap_bf16_4d(&tk, g.n_c > 0 ? Kc : Q, dims, strides, box)) return e;
  if (int e = make_tmap_bf16_4d(&tv, g.n_c > 0 ? Vc : Q, dims, strides, box)) return e;
  return launch_tile<kTileCompressed>(g, tq, tk, tv, tile_args(g, O, lse), ctx, st);
}

}  // namespace infllmv2
