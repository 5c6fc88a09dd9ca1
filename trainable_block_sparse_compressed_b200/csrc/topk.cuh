// topk.cuh -- warp-collective block selection for one query row.
//
// For query token t (cur = t / 64) the selection keeps the forced blocks --
// the initial blocks 0 .. n_init-1 and the n_local most recent blocks
// cur-n_local+1 .. cur (InfLLM-V2 skill write-up, Core Concept: the sliding
// pattern keeps local context) -- and fills the remaining topk - |forced|
// slots with the highest-scoring other blocks b <= cur (reportify digest,
// Technical Mechanism: block selection).  Equal scores go to the lower block
// index; -inf (no visible compressed window) ranks below every finite score.
// The output row lists the kept blocks in ascending order, padded with -1.
//
// Scores become order-preserving 32-bit keys (non-candidates get key 0), each
// lane holds VPL keys in registers (block i at lane i % 32, slot i / 32), and
// the warp finds the exact free-th largest key tau by a most-significant-bit-
// first search: up to 32 rounds of "count keys >= candidate", stopping early
// once exactly the free slots hold keys >= the candidate.  Blocks with key > tau
// are kept; among keys == tau the lowest indices fill the remaining slots,
// ranked with ballots in index order.
#pragma once

#include "common.cuh"

namespace infllmv2 {

__device__ __forceinline__ uint32_t order_key(float s) {
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// srow: the nb = cur + 1 block scores of the row (global or shared memory).
// orow: topk output entries.  All 32 lanes of the warp must call.
template <int VPL>
__device__ __forceinline__ void warp_select_row(const float* srow, int cur, int topk, int n_init,
                                                int n_local, int32_t* orow) {
  const int lane = threadIdx.x & 31;
  const int nb = cur + 1;
  auto forced = [&](int i) { return i < n_init || i > cur - n_local; };
  const int a = min(n_init, nb);
  const int lo = max(0, cur - n_local + 1);
  const int n_forced = a + (nb - lo) - max(0, a - lo);
  const int free_slots = topk - n_forced;
  const int n_cand = nb - n_forced;

  uint32_t key[VPL];
#pragma unroll
  for (int s = 0; s < VPL; ++s) {
    const int i = s * 32 + lane;
    key[s] = (i < nb && !forced(i)) ? order_key(srow[i]) : 0u;
  }

  uint32_t tau = 0;
  int need_eq = 0;
  const bool take_all = free_slots >= n_cand;
  if (!take_all) {
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t c = tau | (1u << bit);
      int cnt = 0;
#pragma unroll
      for (int s = 0; s < VPL; ++s) cnt += key[s] >= c ? 1 : 0;
      cnt = __reduce_add_sync(0xffffffffu, cnt);
      if (cnt >= free_slots) tau = c;
      // exactly free_slots keys are >= c: they are the free_slots largest,
      // with no tie at the boundary, so the remaining bits change nothing
      if (cnt == free_slots) break;
    }
    int gt = 0;
#pragma unroll
    for (int s = 0; s < VPL; ++s) gt += key[s] > tau ? 1 : 0;
    gt = __reduce_add_sync(0xffffffffu, gt);
    need_eq = free_slots - gt;
  }

  const uint32_t lt_mask = (1u << lane) - 1u;
  int written = 0, eq_seen = 0;
#pragma unroll
  for (int s = 0; s < VPL; ++s) {
    const int i = s * 32 + lane;
    const bool valid = i < nb;
    const bool is_forced = valid && forced(i);
    bool keep = is_forced || (valid && (take_all || key[s] > tau));
    const bool eq = valid && !is_forced && !take_all && key[s] == tau;
    const uint32_t eq_ballot = __ballot_sync(0xffffffffu, eq);
    if (eq) keep = (eq_seen + __popc(eq_ballot & lt_mask)) < need_eq;
    eq_seen += __popc(eq_ballot);
    const uint32_t kb = __ballot_sync(0xffffffffu, keep);
    if (keep) orow[written + __popc(kb & lt_mask)] = i;
    written += __popc(kb);
  }
  for (int k = written + lane; k < topk; k += 32) orow[k] = -1;
}

// Exclusive prefix sum of one int per thread over a CTA of NT threads (NT a
// multiple of 32, at most 1024); returns the thread's offset and, in *total,
// the CTA sum.  `scratch` holds NT / 32 + 1 ints of shared memory.  All
// threads must call.
template <int NT>
__device__ __forceinline__ int cta_exclusive_scan(int v, int* scratch, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) scratch[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NT / 32 ? scratch[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NT / 32) scratch[lane] = w;  // inclusive warp totals
    if (lane == NT / 32 - 1) scratch[NT / 32] = w;
  }
  __syncthreads();
  const int off = (warp > 0 ? scratch[warp - 1] : 0) + x - v;
  *total = scratch[NT / 32];
  __syncthreads();  // scratch is reused by the next call
  return off;
}

// The same selection as warp_select_row, by a whole CTA of NT threads: thread
// i holds blocks i*PER .. i*PER+PER-1 (rows of up to NT*PER blocks).  The
// free_slots-th largest candidate key tau is found bit by bit, most
// significant first, with a CTA-wide count per bit (warp reductions, one
// barrier per round over a double-buffered array of warp counts).  Keys
// above tau are kept; among keys equal to tau the lowest block indices fill
// the remaining slots (a prefix sum over threads in index order); a second
// prefix sum places the kept blocks in ascending order.  All threads must
// call.
template <int NT>
__device__ __forceinline__ int cta_count(int v, int (*buf)[NT / 32], int round) {
  const int s = __reduce_add_sync(0xffffffffu, v);
  if ((threadIdx.x & 31) == 0) buf[round & 1][threadIdx.x >> 5] = s;
  __syncthreads();
  int tot = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) tot += buf[round & 1][w];
  return tot;
}

template <int NT, int PER>
__device__ __forceinline__ void cta_select_row(const float* srow, int cur, int topk, int n_init,
                                               int n_local, int32_t* orow) {
  __shared__ int cnt_buf[2][NT / 32];
  __shared__ int scan_buf[NT / 32 + 1];
  const int nb = cur + 1;
  auto forced = [&](int i) { return i < n_init || i > cur - n_local; };
  const int a = min(n_init, nb);
  const int lo = max(0, cur - n_local + 1);
  const int n_forced = a + (nb - lo) - max(0, a - lo);
  const int free_slots = topk - n_forced;
  const int n_cand = nb - n_forced;
  const int base = threadIdx.x * PER;

  uint32_t key[PER];
#pragma unroll
  for (int s = 0; s < PER; ++s) {
    const int i = base + s;
    key[s] = (i < nb && !forced(i)) ? order_key(srow[i]) : 0u;
  }
  const bool take_all = free_slots >= n_cand;
  uint32_t tau = 0;
  int need_eq = 0;
  if (!take_all) {
    int round = 0;
    for (int bit = 31; bit >= 0; --bit, ++round) {
      const uint32_t c = tau | (1u << bit);
      int n = 0;
#pragma unroll
      for (int s = 0; s < PER; ++s) n += key[s] >= c ? 1 : 0;
      const int tot = cta_count<NT>(n, cnt_buf, round);
      if (tot >= free_slots) tau = c;
      if (tot == free_slots) {  // the free_slots largest keys are exactly those >= c
        ++round;                // the next count uses the other buffer
        break;
      }
    }
    int n = 0;
#pragma unroll
    for (int s = 0; s < PER; ++s) n += key[s] > tau ? 1 : 0;
    need_eq = free_slots - cta_count<NT>(n, cnt_buf, round);
  }
  // keys equal to tau, ranked by block index
  int n_eq = 0;
#pragma unroll
  for (int s = 0; s < PER; ++s)
    n_eq += (!take_all && base + s < nb && key[s] != 0u && key[s] == tau) ? 1 : 0;
  int tot;
  int eq_rank = cta_exclusive_scan<NT>(n_eq, scan_buf, &tot);
  bool keep[PER];
  int n_keep = 0;
#pragma unroll
  for (int s = 0; s < PER; ++s) {
    const int i = base + s;
    const bool valid = i < nb;
    const bool is_forced = valid && forced(i);
    bool kp = is_forced || (valid && (take_all || key[s] > tau));
    if (valid && !is_forced && !take_all && key[s] == tau) kp = eq_rank++ < need_eq;
    keep[s] = kp;
    n_keep += kp ? 1 : 0;
  }
  int written;
  int pos = cta_exclusive_scan<NT>(n_keep, scan_buf, &written);
#pragma unroll
  for (int s = 0; s < PER; ++s)
    if (keep[s]) orow[pos++] = base + s;
  for (int k2 = written + threadIdx.x; k2 < topk; k2 += NT) orow[k2] = -1;
}

// Values per lane needed for rows of up to nb_max blocks (0 if too many).
inline int topk_vpl(int nb_max) {
  if (nb_max <= 32 * 4) return 4;
  if (nb_max <= 32 * 16) return 16;
  if (nb_max <= 32 * 64) return 64;
  if (nb_max <= 32 * 128) return 128;
  return 0;
}

}  // namespace infllmv2
