// Joint eviction (R-KV 联合淘汰): s_i = lambda * a_i - (1 - lambda) * r_i and a
// deterministic top-B of the candidates.
//
// Persistent CTAs walk the units; while one unit is selected, the next unit's
// a and r are prefetched into L2.  A CTA has 1024 threads for long units and
// 256 for units of at most 8192 candidates, so that several CTAs share an SM
// where the per-unit steps are short.  Per unit:
//   1. s is computed in fp32 and mapped to order-preserving uint32 keys held
//      in shared memory (one read of a and r); the block also finds the
//      smallest and largest key.
//   2. Radix select of the exact key T of the B-th largest score, most
//      significant digit first.  Bits above the highest bit in which the min
//      and max keys differ are common to all keys, so the first 8-bit digit is
//      taken just below them: it spreads the keys over the bins even when all
//      scores share sign and exponent.  Histograms are kept per group of four
//      warps (plain shared-memory atomics).  After the first digit the
//      surviving keys (usually ~1/256 of them) are compacted into a short list
//      and the remaining digits only look at that list.
//   3. Keys equal to T are taken lowest index first.  The kept set is written
//      in ascending index order: each warp owns a contiguous segment of the
//      candidates, counts its "greater" and "equal" keys, and after one
//      block-level prefix over the warps writes its positions with ballots.
// Optional extensions: the first `sinks` tokens are always kept and excluded
// from the ranking (attention sinks), and each unit may have its own budget
// (budgets[u], clamped to 0 .. budget).  Row u of idx has stride W and ends in
// -1 past the n_kept[u] valid entries.
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

constexpr int kListCap = 4096;    // keys kept for the digits after the first
constexpr int kSmallUnitCands = 8192;   // longest unit for the 256-thread CTAs

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t b = __float_as_uint(s);
  if ((b << 1) == 0) b = 0;  // -0 and +0 compare equal
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ void prefetch_l2(const void* p, size_t bytes) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(p) & ~static_cast<uintptr_t>(15);
  const uintptr_t a1 = (reinterpret_cast<uintptr_t>(p) + bytes + 15) & ~static_cast<uintptr_t>(15);
  for (uintptr_t q = a0; q < a1; q += 32768) {
    const uintptr_t e = q + 32768 < a1 ? q + 32768 : a1;
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(q),
                 "r"(static_cast<uint32_t>(e - q))
                 : "memory");
  }
}

template <int kSelThreads>
__global__ void __launch_bounds__(kSelThreads, kSelThreads <= 256 ? 4 : 1)
    select_kernel(const int64_t* __restrict__ tok_off, int U, int w, const float* __restrict__ a,
                  const float* __restrict__ r, float lam, int max_budget,
                  const int32_t* __restrict__ budgets, int sinks, int W,
                  int32_t* __restrict__ idx, int32_t* __restrict__ n_kept) {
  constexpr int kSelWarps = kSelThreads / 32;
  constexpr int kHistGroups = kSelWarps / 4;   // histograms shared by four warps each
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist8[kHistGroups][256];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t list[kListCap];
  __shared__ int sh[8];
  __shared__ uint32_t wmin[kSelWarps], wmax[kSelWarps];
  __shared__ int wgt[kSelWarps], weq[kSelWarps], eqb[kSelWarps], outb[kSelWarps];
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const float lw = lam, rw = 1.f - lam;

  for (int u = blockIdx.x; u < U; u += gridDim.x) {
    const int64_t tbase = tok_off[u];
    const int N = static_cast<int>(tok_off[u + 1] - tbase);
    const int c0 = N - w;                       // candidates, sinks included
    const int m = min(sinks, c0);               // sinks: always kept, not ranked
    const int c = c0 - m;                       // ranked candidates m .. c0 - 1
    const int64_t base = tbase + m;             // a, r of ranked candidate i at base + i
    int budget = max_budget;
    if (budgets) budget = min(max(budgets[u], 0), max_budget);
    int32_t* out = idx + static_cast<int64_t>(u) * W;
    if (tid == 0 && u + static_cast<int>(gridDim.x) < U) {
      const int u2 = u + gridDim.x;
      const int64_t b2 = tok_off[u2];
      const int64_t c2 = tok_off[u2 + 1] - b2 - w;
      if (c2 > 0) {
        prefetch_l2(a + b2, static_cast<size_t>(c2) * 4);
        prefetch_l2(r + b2, static_cast<size_t>(c2) * 4);
      }
    }
    if (c <= budget) {  // every token is kept
      for (int i = tid; i < W; i += kSelThreads) out[i] = i < N ? i : -1;
      if (tid == 0) n_kept[u] = N;
      continue;
    }
    // sinks, the window after the selected candidates, and the unused tail
    for (int t = tid; t < W - budget; t += kSelThreads) {
      if (t < m) out[t] = t;
      else if (t < m + w) out[budget + t] = c0 + (t - m);
      else out[budget + t] = -1;
    }
    if (tid == 0) n_kept[u] = m + budget + w;
    if (budget == 0) continue;  // the radix step needs want >= 1
    out += m;                   // selected candidates follow the sinks

    // ---- 1. keys, min and max
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int i = tid; i < c; i += kSelThreads) {
      const float s = __fsub_rn(__fmul_rn(lw, a[base + i]), __fmul_rn(rw, r[base + i]));
      const uint32_t k = order_key(s);
      keys[i] = k;
      kmin = min(kmin, k);
      kmax = max(kmax, k);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
      kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    }
    if (lane == 0) {
      wmin[wp] = kmin;
      wmax[wp] = kmax;
    }
    __syncthreads();
    if (wp == 0) {
      kmin = lane < kSelWarps ? wmin[lane] : 0xffffffffu;
      kmax = lane < kSelWarps ? wmax[lane] : 0u;
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
        kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
      }
      if (lane == 0) {
        sh[4] = static_cast<int>(kmin);
        sh[5] = static_cast<int>(kmax);
      }
    }
    __syncthreads();
    kmin = static_cast<uint32_t>(sh[4]);
    kmax = static_cast<uint32_t>(sh[5]);

    // ---- 2. radix select below the common prefix
    const uint32_t diff = kmin ^ kmax;
    int lo = diff ? 32 - __clz(diff) : 0;     // bits [0, lo) still undetermined
    uint32_t pmask = lo >= 32 ? 0u : ~((1u << lo) - 1u);
    uint32_t prefix = kmin & pmask;
    int want = budget;                        // keys still to take among the prefix matches
    bool in_list = false;
    int nlist = 0;
    while (lo > 0) {
      const int d = min(8, lo);
      const int shift = lo - d;
      const uint32_t dmask = (1u << d) - 1u;
      for (int b = tid; b < kHistGroups * 256; b += kSelThreads) (&hist8[0][0])[b] = 0u;
      __syncthreads();
      uint32_t* hg = hist8[wp >> 2];
      if (!in_list) {
        for (int i = tid; i < c; i += kSelThreads) {
          const uint32_t k = keys[i];
          if ((k & pmask) == prefix) atomicAdd(&hg[(k >> shift) & dmask], 1u);
        }
      } else {
        for (int i = tid; i < nlist; i += kSelThreads) {
          const uint32_t k = list[i];
          if ((k & pmask) == prefix) atomicAdd(&hg[(k >> shift) & dmask], 1u);
        }
      }
      __syncthreads();
      if (tid < 256) {
        uint32_t t = 0;
#pragma unroll
        for (int g = 0; g < kHistGroups; ++g) t += hist8[g][tid];
        hist[tid] = t;
      }
      __syncthreads();
      if (wp == 0) {
        // lane l owns bins 255-8l .. 248-8l (descending)
        int cnt[8], tot = 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          cnt[k] = static_cast<int>(hist[255 - 8 * lane - k]);
          tot += cnt[k];
        }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const int excl = incl - tot;
        const unsigned hit = __ballot_sync(0xffffffffu, excl < want && want <= incl);
        if (lane == __ffs(hit) - 1) {
          int run = excl;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if (run + cnt[k] >= want) {
              sh[0] = 255 - 8 * lane - k;
              sh[1] = run;
              sh[2] = cnt[k];
              break;
            }
            run += cnt[k];
          }
        }
        if (lane == 0) sh[3] = 0;
      }
      __syncthreads();
      want -= sh[1];
      prefix |= static_cast<uint32_t>(sh[0]) << shift;
      pmask |= dmask << shift;
      lo = shift;
      const int cnt_bin = sh[2];
      if (!in_list && lo > 0 && cnt_bin <= kListCap) {
        // survivors of this digit -> short list (order irrelevant for T)
        for (int i0 = wp * 32; i0 < ((c + 31) & ~31); i0 += kSelThreads) {
          const int i = i0 + lane;
          const uint32_t k = i < c ? keys[i] : 0u;
          const bool hit = i < c && (k & pmask) == prefix;
          const unsigned bal = __ballot_sync(0xffffffffu, hit);
          int slot = 0;
          if (lane == 0 && bal) slot = atomicAdd(&sh[3], __popc(bal));
          slot = __shfl_sync(0xffffffffu, slot, 0);
          const int pos = slot + __popc(bal & ((1u << lane) - 1u));
          if (hit && pos < kListCap) list[pos] = k;
        }
        __syncthreads();
        nlist = sh[3];
        in_list = true;
      }
      __syncthreads();
    }
    const uint32_t T = prefix;  // key of the budget-th largest score
    const int take_eq = want;   // keys equal to T that are kept (lowest indices)

    // ---- 3. per-warp segments, counts, then ordered output
    const int seg = (((c + kSelWarps - 1) / kSelWarps) + 31) & ~31;
    const int s0 = wp * seg, s1 = min(c, s0 + seg);
    int gt = 0, eq = 0;
    for (int i0 = s0; i0 < s1; i0 += 32) {
      const int i = i0 + lane;
      const bool v = i < s1;
      const uint32_t k = v ? keys[i] : 0u;
      gt += __popc(__ballot_sync(0xffffffffu, v && k > T));
      eq += __popc(__ballot_sync(0xffffffffu, v && k == T));
    }
    if (lane == 0) {
      wgt[wp] = gt;
      weq[wp] = eq;
    }
    __syncthreads();
    if (tid == 0) {
      int eb = 0, ob = 0;
      for (int x = 0; x < kSelWarps; ++x) {
        eqb[x] = eb;
        outb[x] = ob;
        ob += wgt[x] + min(max(take_eq - eb, 0), weq[x]);
        eb += weq[x];
      }
    }
    __syncthreads();
    int eseen = eqb[wp], oseen = outb[wp];
    const unsigned lt = (1u << lane) - 1u;
    for (int i0 = s0; i0 < s1; i0 += 32) {
      const int i = i0 + lane;
      const bool v = i < s1;
      const uint32_t k = v ? keys[i] : 0u;
      const bool g = v && k > T, e = v && k == T;
      const unsigned be = __ballot_sync(0xffffffffu, e);
      const bool f = g || (e && eseen + __popc(be & lt) < take_eq);
      const unsigned bf = __ballot_sync(0xffffffffu, f);
      const int pos = oseen + __popc(bf & lt);
      if (f && pos < budget) out[pos] = m + i;
      eseen += __popc(be);
      oseen += __popc(bf);
    }
    __syncthreads();  // shared state is reused by the next unit
  }
}

}  // namespace

cudaError_t select_configure() {
  cudaError_t e = cudaFuncSetAttribute(select_kernel<1024>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kMaxTokensPerUnit * 4);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(select_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kSmallUnitCands * 4);
}

cudaError_t launch_select(const int64_t* tok_off, int U, int w, int cmax, const float* a,
                          const float* r, float lam, int budget, const int32_t* budgets,
                          int sinks, int W, int32_t* idx, int32_t* n_kept, cudaStream_t st) {
  // keys of the ranked candidates (budgets[u] <= budget, so a unit with at
  // most `budget` candidates never needs them)
  const size_t smem = cmax > budget ? static_cast<size_t>(cmax) * 4 : 0;
  const bool small = cmax <= kSmallUnitCands;
  const void* fn = small ? reinterpret_cast<const void*>(&select_kernel<256>)
                         : reinterpret_cast<const void*>(&select_kernel<1024>);
  const int threads = small ? 256 : 1024;
  int dev = 0, nsm = 0, per = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fn, threads, smem) != cudaSuccess ||
      per < 1) {
    cudaGetLastError();
    per = 1;
  }
  int grid = nsm * per;
  if (grid > U) grid = U;
  if (small)
    select_kernel<256><<<grid, 256, smem, st>>>(tok_off, U, w, a, r, lam, budget, budgets, sinks,
                                               W, idx, n_kept);
  else
    select_kernel<1024><<<grid, 1024, smem, st>>>(tok_off, U, w, a, r, lam, budget, budgets,
                                                 sinks, W, idx, n_kept);
  return cudaGetLastError();
}

}  // namespace rkv
