// gather_peak.cu -- the L2 -> shared-memory gather ceiling of this GPU.
//
// The block-sparse attention moves every selected 64-key block of K and V
// from L2 into shared memory with 16 KB bulk copies; on inputs whose tokens
// share few blocks that movement, not the tensor core, bounds it.  This
// kernel performs the same movement and nothing else, so that a benchmark can
// measure the ceiling the attention's gather is held against: one CTA per
// SM, one thread issuing 16 KB bulk copies from pseudo-random 16 KB-aligned
// offsets of an (L2-resident) source buffer into a ring of three 64 KB stages
// (the attention's ring), each stage refilled as soon as its previous fill
// has landed.  Waits are bounded like every other wait of the library.
#include "common.cuh"
#include "sm100.cuh"

namespace infllmv2 {
namespace {

constexpr int kCopy = 16384;          // one packed block of K or V
constexpr int kPerStage = 4;          // a pair of blocks of K and of V
constexpr int kStages = 3;
constexpr int kStageBytes = kCopy * kPerStage;

__global__ void __launch_bounds__(32, 1)
    gather_peak_kernel(const uint8_t* __restrict__ src, uint64_t n_tiles, int rounds,
                       DevCtx ctx) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t full[kStages];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* ring = smem_raw + (((raw + 127u) & ~127u) - raw);
  if (threadIdx.x != 0) return;
  for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
  fence_mbar_init();
  uint64_t x = 0x9E3779B97F4A7C15ull * (blockIdx.x + 1);  // per-CTA xorshift state
  int issued = 0;
  for (int r = 0; r < rounds; ++r) {
    for (int s = 0; s < kStages; ++s, ++issued) {
      if (issued >= kStages && !mbar_wait(&full[s], ((issued / kStages) - 1) & 1, ctx.wait_ns)) {
        report_status(ctx.status, INFLLMV2_STATUS_TIMEOUT);
        r = rounds;
        break;
      }
      mbar_arrive_expect_tx(&full[s], kStageBytes);
      for (int c = 0; c < kPerStage; ++c) {
        x ^= x << 13;
        x ^= x >> 7;
        x ^= x << 17;
        const uint64_t tile = x % n_tiles;
        bulk_load(ring + s * kStageBytes + c * kCopy, src + tile * kCopy, kCopy, &full[s]);
      }
    }
  }
  // never leave with copies in flight
  for (int q = issued - 1; q >= 0 && q >= issued - kStages; --q)
    mbar_wait(&full[q % kStages], (q / kStages) & 1, ctx.wait_ns);
}

}  // namespace
}  // namespace infllmv2

using namespace infllmv2;

extern "C" int infllmv2_gather_peak(const void* src, size_t src_bytes, int32_t rounds,
                                    int32_t* ctas_out, void* stream) {
  if (!src || rounds < 1 || src_bytes < static_cast<size_t>(kCopy))
    return INFLLMV2_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(src) & 15u) return INFLLMV2_ERR_UNSUPPORTED;
  DevCtx ctx;
  if (get_dev_ctx(&ctx) != cudaSuccess) return INFLLMV2_ERR_CUDA;
  const size_t smem = 128 + kStages * kStageBytes;
  static std::atomic<uint64_t> smem_set{0};
  if (int e = set_smem_limit(gather_peak_kernel, smem, smem_set)) return e;
  const int grid = sm_count();
  gather_peak_kernel<<<grid, 32, smem, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(src), src_bytes / kCopy, rounds, ctx);
  if (cudaGetLastError() != cudaSuccess) return INFLLMV2_ERR_CUDA;
  if (ctas_out) *ctas_out = grid;
  return INFLLMV2_OK;
}
