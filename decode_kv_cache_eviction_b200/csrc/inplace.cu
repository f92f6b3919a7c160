// In-place slot reuse (the ThinKV summary's Continuous Thinking step): instead
// of gathering the kept rows into a new buffer, every row stays where it is,
// a keep mask marks the live slots, and the evicted slots form a free list
// that new tokens overwrite, lowest slot first.
//
// evict_in_place_kernel: one CTA per unit (persistent over units).  The kept
//   indices set bits of a shared-memory bitmap; one block scan over the
//   words' free counts (each thread a contiguous run of words) gives every
//   word the number of free slots before it; then warps walk the words, lane
//   = slot, and write the keep bytes and the free slots (ascending) with one
//   coalesced store each per word.
// fill_slots_kernel: one CTA per unit.  New token t is copied (16 threads per
//   256-byte row, 128-bit accesses) to slot free[t]; the slot is marked live;
//   then the remaining free slots move to the front of the list, tile by tile
//   in ascending order (each tile is read completely before it is written,
//   and a tile only reads positions that no earlier tile wrote).
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

constexpr int kIpThreads = 256;
constexpr int kIpWarps = kIpThreads / 32;
constexpr int kIpWords = kMaxTokensPerUnit / 32;   // kept bitmap words of the longest unit

__global__ void __launch_bounds__(kIpThreads)
    evict_in_place_kernel(const int64_t* __restrict__ tok_off, int U, int W, int wcap,
                          const int32_t* __restrict__ idx, const int32_t* __restrict__ n_kept,
                          uint8_t* __restrict__ keep, int32_t* __restrict__ free_slots,
                          int32_t* __restrict__ n_free, int* status) {
  // kept bitmap (bit i of word i / 32) and, per word, the free slots before it
  extern __shared__ uint32_t sm_ip[];
  uint32_t* bits = sm_ip;                            // [wcap]
  int* wbase = reinterpret_cast<int*>(sm_ip + wcap);  // [wcap]
  __shared__ int wsum[kIpWarps];
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  for (int u = blockIdx.x; u < U; u += gridDim.x) {
    const int64_t base = tok_off[u];
    const int N = static_cast<int>(tok_off[u + 1] - base);
    const int nw = (N + 31) >> 5;
    for (int q = tid; q < nw; q += kIpThreads) bits[q] = 0u;
    __syncthreads();
    int nk = n_kept[u];
    if (nk < 0 || nk > W) {
      if (tid == 0) atomicOr(status, kStatusBadIndex);
      nk = nk < 0 ? 0 : W;
    }
    const int32_t* iu = idx + static_cast<int64_t>(u) * W;
    // kept indices, eight loads in flight per thread before their atomics
    for (int j0 = tid; j0 < nk; j0 += 8 * kIpThreads) {
      int kk[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const int j = j0 + x * kIpThreads;
        kk[x] = j < nk ? __ldg(&iu[j]) : 0;
      }
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        if (j0 + x * kIpThreads >= nk) break;
        const int k = kk[x];
        if (k >= 0 && k < N) atomicOr(&bits[k >> 5], 1u << (k & 31));
        else atomicOr(status, kStatusBadIndex);
      }
    }
    __syncthreads();
    // free slots per word; thread tid takes the contiguous words
    // [tid * per, (tid + 1) * per) and the block scans the per-thread totals
    const int per = (nw + kIpThreads - 1) / kIpThreads;
    const int q0 = min(nw, tid * per), q1 = min(nw, q0 + per);
    int cnt = 0;
    for (int q = q0; q < q1; ++q) {
      const int valid = min(32, N - 32 * q);
      const uint32_t vm = valid == 32 ? 0xffffffffu : ((1u << valid) - 1u);
      cnt += __popc(~bits[q] & vm);
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[wp] = incl;
    __syncthreads();
    if (wp == 0) {
      const int v = lane < kIpWarps ? wsum[lane] : 0;
      int x = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      if (lane < kIpWarps) wsum[lane] = x - v;   // exclusive prefix of the warps
    }
    __syncthreads();
    int run = wsum[wp] + incl - cnt;
    for (int q = q0; q < q1; ++q) {
      wbase[q] = run;
      const int valid = min(32, N - 32 * q);
      const uint32_t vm = valid == 32 ? 0xffffffffu : ((1u << valid) - 1u);
      run += __popc(~bits[q] & vm);
    }
    __syncthreads();
    // warps walk the words: lane = slot within the word, so the keep bytes and
    // the free slots of a word go out as one coalesced store each
    // four words per step, their shared-memory loads issued together
    for (int q0 = wp; q0 < nw; q0 += 4 * kIpWarps) {
      uint32_t x[4];
      int wb[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int q = q0 + e * kIpWarps;
        x[e] = q < nw ? bits[q] : 0u;
        wb[e] = q < nw ? wbase[q] : 0;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int q = q0 + e * kIpWarps;
        if (q >= nw) break;
        const int i = 32 * q + lane;
        const bool in = i < N;
        const bool kept = (x[e] >> lane) & 1u;
        if (in) keep[base + i] = kept ? 1 : 0;
        const unsigned fb = __ballot_sync(0xffffffffu, in && !kept);
        if (in && !kept) free_slots[base + wb[e] + __popc(fb & ((1u << lane) - 1u))] = i;
      }
    }
    int nfree = 0;   // free slots before the last word, plus its own
    if (nw > 0) {
      const int valid = N - 32 * (nw - 1);
      const uint32_t vm = valid == 32 ? 0xffffffffu : ((1u << valid) - 1u);
      nfree = wbase[nw - 1] + __popc(~bits[nw - 1] & vm);
    }
    for (int i = nfree + tid; i < N; i += kIpThreads) free_slots[base + i] = -1;
    if (tid == 0) n_free[u] = nfree;
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
                              2 * kIpWords * 4);
}

cudaError_t launch_evict_in_place(const int64_t* tok_off, int U, int nmax, int W,
                                  const int32_t* idx, const int32_t* n_kept, uint8_t* keep,
                                  int32_t* free_slots, int32_t* n_free, int* status, int nsm,
                                  cudaStream_t st) {
  int grid = nsm * 8;
  if (grid > U) grid = U;
  const int wcap = (nmax + 31) / 32;   // bitmap words of the longest unit
  evict_in_place_kernel<<<grid, kIpThreads, static_cast<size_t>(2 * wcap) * 4, st>>>(
      tok_off, U, W, wcap, idx, n_kept, keep, free_slots, n_free, status);
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
