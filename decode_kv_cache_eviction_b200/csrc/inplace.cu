// In-place slot reuse (the ThinKV summary's Continuous Thinking step): instead
// of gathering the kept rows into a new buffer, every row stays where it is,
// a keep mask marks the live slots, and the evicted slots form a free list
// that new tokens overwrite, lowest slot first.
//
// evict_in_place_kernel: one CTA per unit (persistent over units).  The kept
//   indices are scattered into a shared-memory byte mask, the mask is written
//   out, and the free list is the mask's complement compacted with a block
//   scan (ballots within warps, one prefix over the 32 warps per 1024-slot
//   tile), written in ascending order.
// fill_slots_kernel: one CTA per unit.  New token t is copied (16 threads per
//   256-byte row, 128-bit accesses) to slot free[t]; the slot is marked live;
//   then the remaining free slots move to the front of the list, tile by tile
//   in ascending order (each tile is read completely before it is written,
//   and a tile only reads positions that no earlier tile wrote).
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

constexpr int kIpThreads = 1024;
constexpr int kIpWarps = kIpThreads / 32;

__global__ void __launch_bounds__(kIpThreads, 1)
    evict_in_place_kernel(const int64_t* __restrict__ tok_off, int U, int W,
                          const int32_t* __restrict__ idx, const int32_t* __restrict__ n_kept,
                          uint8_t* __restrict__ keep, int32_t* __restrict__ free_slots,
                          int32_t* __restrict__ n_free, int* status) {
  extern __shared__ uint8_t smask[];
  __shared__ int wsum[kIpWarps];
  __shared__ int running;
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  for (int u = blockIdx.x; u < U; u += gridDim.x) {
    const int64_t base = tok_off[u];
    const int N = static_cast<int>(tok_off[u + 1] - base);
    for (int i = tid; i < N; i += kIpThreads) smask[i] = 0;
    if (tid == 0) running = 0;
    __syncthreads();
    int nk = n_kept[u];
    if (nk < 0 || nk > W) {
      if (tid == 0) atomicOr(status, kStatusBadIndex);
      nk = nk < 0 ? 0 : W;
    }
    const int32_t* iu = idx + static_cast<int64_t>(u) * W;
    for (int j = tid; j < nk; j += kIpThreads) {
      const int k = iu[j];
      if (k >= 0 && k < N) smask[k] = 1;
      else atomicOr(status, kStatusBadIndex);
    }
    __syncthreads();
    for (int i = tid; i < N; i += kIpThreads) keep[base + i] = smask[i];
    // free list: ascending complement of the mask
    for (int t0 = 0; t0 < N; t0 += kIpThreads) {
      const int i = t0 + tid;
      const bool f = i < N && smask[i] == 0;
      const unsigned bal = __ballot_sync(0xffffffffu, f);
      if (lane == 0) wsum[wp] = __popc(bal);
      __syncthreads();
      if (wp == 0) {
        const int v = wsum[lane];
        int incl = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        wsum[lane] = incl - v;   // exclusive prefix of the warps
      }
      __syncthreads();
      const int at = running + wsum[wp] + __popc(bal & ((1u << lane) - 1u));
      if (f) free_slots[base + at] = i;
      __syncthreads();   // everyone has read running and wsum
      if (tid == kIpThreads - 1) running = at + (f ? 1 : 0);
      __syncthreads();
    }
    const int nf = running;
    for (int i = nf + tid; i < N; i += kIpThreads) free_slots[base + i] = -1;
    if (tid == 0) n_free[u] = nf;
    __syncthreads();   // shared state is reused by the next unit
  }
}

constexpr int kFillThreads = 256;

__global__ void __launch_bounds__(kFillThreads)
    fill_slots_kernel(const int64_t* __restrict__ tok_off, int U,
                      const int64_t* __restrict__ new_off, const uint4* __restrict__ Kn,
                      const uint4* __restrict__ Vn, uint4* __restrict__ K, uint4* __restrict__ V,
                      uint8_t* __restrict__ keep, int32_t* __restrict__ free_slots,
                      int32_t* __restrict__ n_free, int* status) {
  const int tid = threadIdx.x;
  const int sub = tid & 15;            // 16-byte word of the 256-byte row
  const int rsub = tid >> 4;           // one of 16 rows in flight
  for (int u = blockIdx.x; u < U; u += gridDim.x) {
    const int64_t base = tok_off[u];
    const int N = static_cast<int>(tok_off[u + 1] - base);
    const int64_t nb = new_off[u];
    const int want = static_cast<int>(new_off[u + 1] - nb);
    int nf = n_free[u];
    if (nf < 0 || nf > N) nf = 0;      // not produced by evict_in_place: take nothing
    const int n = want < nf ? want : nf;
    if (want > nf && tid == 0) atomicOr(status, kStatusBadIndex);
    int32_t* fu = free_slots + base;
    for (int t = rsub; t < n; t += kFillThreads / 16) {
      const int slot = fu[t];
      if (slot < 0 || slot >= N) {
        if (sub == 0) atomicOr(status, kStatusBadIndex);
        continue;
      }
      const int64_t dst = (base + slot) * 16 + sub;
      const int64_t src = (nb + t) * 16 + sub;
      K[dst] = __ldcs(&Kn[src]);
      V[dst] = __ldcs(&Vn[src]);
      if (sub == 0) keep[base + slot] = 1;
    }
    __syncthreads();   // every used slot has been read from the list
    // the remaining nf - n free slots move to the front; the tail becomes -1
    for (int t0 = 0; t0 < nf; t0 += kFillThreads) {
      const int t = t0 + tid;
      const int v = t + n < nf ? fu[t + n] : -1;
      __syncthreads();
      if (t < nf) fu[t] = v;
      __syncthreads();
    }
    if (tid == 0) n_free[u] = nf - n;
    __syncthreads();
  }
}

}  // namespace

cudaError_t inplace_configure() {
  return cudaFuncSetAttribute(evict_in_place_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kMaxTokensPerUnit);
}

cudaError_t launch_evict_in_place(const int64_t* tok_off, int U, int nmax, int W,
                                  const int32_t* idx, const int32_t* n_kept, uint8_t* keep,
                                  int32_t* free_slots, int32_t* n_free, int* status, int nsm,
                                  cudaStream_t st) {
  int grid = nsm * 2;
  if (grid > U) grid = U;
  evict_in_place_kernel<<<grid, kIpThreads, static_cast<size_t>(nmax), st>>>(
      tok_off, U, W, idx, n_kept, keep, free_slots, n_free, status);
  return cudaGetLastError();
}

cudaError_t launch_fill_slots(const int64_t* tok_off, int U, const int64_t* new_off,
                              const void* K_new, const void* V_new, void* K, void* V,
                              uint8_t* keep, int32_t* free_slots, int32_t* n_free, int* status,
                              int nsm, cudaStream_t st) {
  int grid = nsm * 4;
  if (grid > U) grid = U;
  fill_slots_kernel<<<grid, kFillThreads, 0, st>>>(
      tok_off, U, new_off, static_cast<const uint4*>(K_new), static_cast<const uint4*>(V_new),
      static_cast<uint4*>(K), static_cast<uint4*>(V), keep, free_slots, n_free, status);
  return cudaGetLastError();
}

}  // namespace rkv
