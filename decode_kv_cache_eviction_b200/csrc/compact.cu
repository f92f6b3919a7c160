// Gather compaction of the surviving rows (the R-KV-style "gather-based
// compaction" named in the ThinKV summary): K_out[u][j] = K[tok_off[u] +
// idx[u][j]], V likewise, bit-exact.  One 256-byte row is 16 x 128-bit words;
// 16 consecutive threads move one row, so every warp reads and writes two whole
// rows (full 32-byte sectors).  Each thread keeps four independent rows in
// flight.  Slots at or beyond n_kept[u] are zero-filled; an index outside the
// unit zero-fills its row and raises the bad-index status bit.
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

constexpr int kUnroll = 4;

__global__ void __launch_bounds__(256) compact_kernel(const int64_t* __restrict__ tok_off, int U,
                                                      int W, const int32_t* __restrict__ idx,
                                                      const int32_t* __restrict__ n_kept,
                                                      const uint4* __restrict__ K,
                                                      const uint4* __restrict__ V,
                                                      uint4* __restrict__ Ko,
                                                      uint4* __restrict__ Vo, int* status) {
  const int64_t total = static_cast<int64_t>(U) * W * 16;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t g0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g0 < total;
       g0 += kUnroll * stride) {
    uint4 kv[kUnroll], vv[kUnroll];
#pragma unroll
    for (int q = 0; q < kUnroll; ++q) {
      const int64_t g = g0 + q * stride;
      kv[q] = make_uint4(0, 0, 0, 0);
      vv[q] = kv[q];
      if (g < total) {
        const int row = static_cast<int>(g >> 4);
        const int part = static_cast<int>(g & 15);
        const int u = row / W;
        const int j = row - u * W;
        const int nk = min(__ldg(&n_kept[u]), W);
        if (j < nk) {
          const int k = __ldg(&idx[row]);
          const int64_t b = __ldg(&tok_off[u]);
          const int N = static_cast<int>(__ldg(&tok_off[u + 1]) - b);
          if (k >= 0 && k < N) {
            const int64_t src = (b + k) * 16 + part;
            kv[q] = __ldcs(K + src);
            vv[q] = __ldcs(V + src);
          } else if (part == 0) {
            atomicOr(status, kStatusBadIndex);
          }
        }
      }
    }
#pragma unroll
    for (int q = 0; q < kUnroll; ++q) {
      const int64_t g = g0 + q * stride;
      if (g < total) {
        Ko[g] = kv[q];
        Vo[g] = vv[q];
      }
    }
  }
}

}  // namespace

cudaError_t launch_compact(const int64_t* tok_off, int U, int W, const int32_t* idx,
                           const int32_t* n_kept, const void* K, const void* V, void* Ko,
                           void* Vo, int* status, int nsm, cudaStream_t st) {
  const int64_t total = static_cast<int64_t>(U) * W * 16;
  int64_t blocks = (total + 256 * kUnroll - 1) / (256 * kUnroll);
  blocks = blocks < 1 ? 1 : blocks;
  const int64_t cap = static_cast<int64_t>(nsm) * 8;
  if (blocks > cap) blocks = cap;
  compact_kernel<<<static_cast<int>(blocks), 256, 0, st>>>(
      tok_off, U, W, idx, n_kept, static_cast<const uint4*>(K), static_cast<const uint4*>(V),
      static_cast<uint4*>(Ko), static_cast<uint4*>(Vo), status);
  return cudaGetLastError();
}

}  // namespace rkv
