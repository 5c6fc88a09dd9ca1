// pack.cu -- repacks K and V ([B, T, Hkv, 128] bf16) into block tiles: one
// contiguous 16 KB chunk per (batch, kv head, 64-key block), laid out as the
// tensor core's canonical no-swizzle operand image:
//
//   byte offset of (key r, channel c) = (r / 8) * 2048 + (c / 8) * 128
//                                       + (r % 8) * 16 + (c % 8) * 2
//
// i.e. 8x8 core matrices of 128 bytes, channel groups 128 B apart and key
// groups 2 KB apart.  Two such chunks placed back to back form a 128-key
// operand with uniform strides, both for K (K-major: row groups 2 KB apart)
// and for V^T (MN-major: key groups 2 KB apart, channel groups 128 B apart),
// so the attention kernel gathers a selected block with a single 16 KB bulk
// copy -- contiguous 16 KB copies move ~1.5x the bytes per second of 8 KB
// tensor-map boxes when thousands of blocks are gathered from L2.  Keys past
// the end of the sequence are zero.
//
// HBM-bound permutation: each CTA stages one block of K and V in shared memory
// so that both the row-major reads and the tile writes are coalesced.
#include "common.cuh"

namespace infllmv2 {
namespace {

constexpr int kTileBytes = kBlock * kHeadDim * 2;  // 16 KB

__global__ void __launch_bounds__(256) pack_kv_kernel(const __nv_bfloat16* __restrict__ K,
                                                      const __nv_bfloat16* __restrict__ V,
                                                      uint8_t* __restrict__ Kp,
                                                      uint8_t* __restrict__ Vp, int T, int Hkv,
                                                      int nb) {
  __shared__ __align__(16) uint8_t tile[2][kTileBytes];
  const int blk = blockIdx.x % nb;
  const int bg = blockIdx.x / nb;
  const int b = bg / Hkv, g = bg % Hkv;
  // 64 rows x 16 chunks of 16 bytes = 1024 pieces per tensor, 4 per thread
  for (int i = threadIdx.x; i < 1024; i += blockDim.x) {
    const int r = i >> 4, c8 = i & 15;
    const int t = blk * kBlock + r;
    uint4 kv = make_uint4(0, 0, 0, 0), vv = make_uint4(0, 0, 0, 0);
    if (t < T) {
      const int64_t off = ((static_cast<int64_t>(b) * T + t) * Hkv + g) * kHeadDim + 8 * c8;
      kv = __ldg(reinterpret_cast<const uint4*>(K + off));
      vv = __ldg(reinterpret_cast<const uint4*>(V + off));
    }
    const int dst = (r >> 3) * 2048 + c8 * 128 + (r & 7) * 16;
    *reinterpret_cast<uint4*>(&tile[0][dst]) = kv;
    *reinterpret_cast<uint4*>(&tile[1][dst]) = vv;
  }
  __syncthreads();
  const int64_t chunk = (static_cast<int64_t>(bg) * nb + blk) * kTileBytes;
  for (int i = threadIdx.x; i < kTileBytes / 16; i += blockDim.x) {
    reinterpret_cast<uint4*>(Kp + chunk)[i] = reinterpret_cast<const uint4*>(tile[0])[i];
    reinterpret_cast<uint4*>(Vp + chunk)[i] = reinterpret_cast<const uint4*>(tile[1])[i];
  }
}

}  // namespace

size_t packed_kv_bytes(const Geometry& g) {
  const int64_t nb = (static_cast<int64_t>(g.T) + kBlock - 1) / kBlock;
  return static_cast<size_t>(2) * g.B * g.Hkv * nb * kTileBytes;
}

int launch_pack_kv(const Geometry& g, const void* K, const void* V, void* packed,
                   cudaStream_t st) {
  const int nb = (g.T + kBlock - 1) / kBlock;
  if (g.B == 0 || nb == 0) return INFLLMV2_OK;
  uint8_t* Kp = static_cast<uint8_t*>(packed);
  uint8_t* Vp = Kp + packed_kv_bytes(g) / 2;
  const unsigned grid = static_cast<unsigned>(g.B) * g.Hkv * nb;
  pack_kv_kernel<<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(K),
                                       static_cast<const __nv_bfloat16*>(V), Kp, Vp, g.T, g.Hkv,
                                       nb);
  return cudaGetLastError() == cudaSuccess ? INFLLMV2_OK : INFLLMV2_ERR_CUDA;
}

}  // namespace infllmv2
