// topk.cu -- prefill block selection: one warp per (batch, kv head, token)
// row of the causally packed block-score workspace (see topk.cuh for the
// selection rule).  Each warp holds as few keys per lane as its own row
// needs (row t has t/64 + 1 blocks), up to VPL.
#include "common.cuh"
#include "topk.cuh"

namespace infllmv2 {
namespace {

template <int VPL>
__global__ void __launch_bounds__(256) topk_kernel(const float* __restrict__ scores,
                                                    int32_t* __restrict__ idx, int B, int Hkv,
                                                    int q0, int Tq, int topk, int n_init,
                                                    int n_local) {
  // rows: (batch, kv head, query token q0 .. q0+Tq-1); the workspace holds
  // the causally packed score rows of those tokens, from row q0 on
  const int64_t row = blockIdx.x * static_cast<int64_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
  const int64_t n_rows = static_cast<int64_t>(B) * Hkv * Tq;
  if (row >= n_rows) return;
  const int t = q0 + static_cast<int>(row % Tq);
  const int64_t bg = row / Tq;
  const int64_t row0 = score_row_offset(q0);
  const float* srow = scores + bg * (score_row_offset(q0 + Tq) - row0) + score_row_offset(t) - row0;
  const int cur = t / kBlock;
  int32_t* orow = idx + row * topk;
  if (VPL > 4 && cur < 32 * 4)
    warp_select_row<4>(srow, cur, topk, n_init, n_local, orow);
  else if (VPL > 16 && cur < 32 * 16)
    warp_select_row<16>(srow, cur, topk, n_init, n_local, orow);
  else if (VPL > 32 && cur < 32 * 32)
    warp_select_row<32>(srow, cur, topk, n_init, n_local, orow);
  else if (VPL > 64 && cur < 32 * 64)
    warp_select_row<64>(srow, cur, topk, n_init, n_local, orow);
  else
    warp_select_row<VPL>(srow, cur, topk, n_init, n_local, orow);
}

}  // namespace

int launch_topk(const Geometry& g, const float* scores, int32_t* idx, cudaStream_t st) {
  if (g.B == 0 || g.Tq == 0) return INFLLMV2_OK;
  const int nb_max = (g.q0 + g.Tq - 1) / kBlock + 1;
  const int64_t rows = static_cast<int64_t>(g.B) * g.Hkv * g.Tq;
  const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
  const int vpl = topk_vpl(nb_max);
#define INFLLMV2_TOPK(V)                                                             \
  topk_kernel<V><<<blocks, 256, 0, st>>>(scores, idx, g.B, g.Hkv, g.q0, g.Tq, g.topk, \
                                         g.n_init, g.n_local)
  switch (vpl) {
    case 4: INFLLMV2_TOPK(4); break;
    case 16: INFLLMV2_TOPK(16); break;
    case 64: INFLLMV2_TOPK(64); break;
    case 128: INFLLMV2_TOPK(128); break;
    default: return INFLLMV2_ERR_UNSUPPORTED;
  }
#undef INFLLMV2_TOPK
  return cudaGetLastError() == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

}  // namespace infllmv2
