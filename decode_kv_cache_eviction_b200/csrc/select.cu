// Joint eviction (R-KV 联合淘汰): s_i = lambda * a_i - (1 - lambda) * r_i and a
// deterministic top-B of the candidates: the B largest by (s descending, index
// ascending), written in ascending index order.
//
// One CTA per unit (several CTAs share an SM).  s is mapped to an
// order-preserving uint32 key; keys are recomputed from a and r wherever they
// are needed, so a unit of any length needs no shared-memory copy of them.
//   1. Sample: the keys at S evenly spaced candidates.  Two order statistics of
//      the sample, about four standard deviations of the sampling error above
//      and below the budget's rank, give splitters hi >= lo.
//   2. Classify (the one pass that reads a and r from HBM): every candidate is
//      above the bracket (key > hi, kept for sure), inside it (lo <= key <= hi,
//      appended with its index to a short list) or below.  A warp handles 32
//      consecutive candidates at a time, so the "above" ballot is directly one
//      32-bit word of the kept bitmap.
//   3. If the budget's rank falls inside the bracket and the list fits, the
//      exact threshold key T and the tie cut (keys equal to T are taken lowest
//      index first) are found by radix selection on the list alone, and the
//      kept list entries are added to the bitmap.  Otherwise (rare: many equal
//      keys, or a sample far from the data) the same selection runs over all
//      candidates, reading a and r again.
//   4. The bitmap is turned into ascending indices: one block-wide prefix of
//      the words' popcounts, then each thread writes the set bits of its words.
// Optional extensions: the first `sinks` tokens are always kept and excluded
// from the ranking (attention sinks), and each unit may have its own budget
// (budgets[u], clamped to 0 .. budget).  Row u of idx has stride W and ends in
// -1 past the n_kept[u] valid entries.
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSample = 2048;     // sample size (at most the candidate count)
constexpr int kListCap = 4096;    // bracket entries kept on chip
constexpr float kSpread = 4.f;    // bracket half-width in sampling standard deviations

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t b = __float_as_uint(s);
  if ((b << 1) == 0) b = 0;  // -0 and +0 compare equal
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct SelShared {
  uint32_t hist[256];
  uint32_t sample[kSample];
  uint32_t lkey[kListCap];
  int32_t lidx[kListCap];
  int nlist;
  int cnt_above;
  int sh[8];
  uint32_t wred[kSelWarps];
  uint32_t wred2[kSelWarps];
};

// Block-wide: the k-th largest (1 <= k <= number of matches) of the values
// get(i) over i in [0, n) for which get returns valid, radix-selected most
// significant digit first.  `lo_bits` is the number of low bits in which the
// values may differ (bits above are common to all: `prefix`).  Returns the
// value; *above receives the number of matching values strictly greater.
template <class Get>
__device__ uint32_t kth_largest(SelShared& s, Get get, int n, int k, uint32_t prefix,
                                int lo_bits, int* above) {
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  uint32_t pmask = lo_bits >= 32 ? 0u : ~((1u << lo_bits) - 1u);
  prefix &= pmask;
  int want = k, gt = 0;
  int lo = lo_bits;
  while (lo > 0) {
    const int d = min(8, lo);
    const int shift = lo - d;
    const uint32_t dmask = (1u << d) - 1u;
    for (int b = tid; b < 256; b += kSelThreads) s.hist[b] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kSelThreads) {
      uint32_t v;
      if (get(i, v) && (v & pmask) == prefix) atomicAdd(&s.hist[(v >> shift) & dmask], 1u);
    }
    __syncthreads();
    if (wp == 0) {
      // lane l owns bins 255-8l .. 248-8l (descending)
      int cnt[8], tot = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnt[q] = static_cast<int>(s.hist[255 - 8 * lane - q]);
        tot += cnt[q];
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
        for (int q = 0; q < 8; ++q) {
          if (run + cnt[q] >= want) {
            s.sh[0] = 255 - 8 * lane - q;
            s.sh[1] = run;
            break;
          }
          run += cnt[q];
        }
      }
    }
    __syncthreads();
    want -= s.sh[1];
    gt += s.sh[1];
    prefix |= static_cast<uint32_t>(s.sh[0]) << shift;
    pmask |= dmask << shift;
    lo = shift;
    __syncthreads();   // sh and hist are reused
  }
  *above = gt;
  return prefix;
}

// Block-wide min and max of get(i) over the valid i in [0, n).
template <class Get>
__device__ void min_max(SelShared& s, Get get, int n, uint32_t* mn, uint32_t* mx) {
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  uint32_t a = 0xffffffffu, b = 0u;
  for (int i = tid; i < n; i += kSelThreads) {
    uint32_t v;
    if (get(i, v)) {
      a = min(a, v);
      b = max(b, v);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    a = min(a, __shfl_xor_sync(0xffffffffu, a, o));
    b = max(b, __shfl_xor_sync(0xffffffffu, b, o));
  }
  if (lane == 0) {
    s.wred[wp] = a;
    s.wred2[wp] = b;
  }
  __syncthreads();
  a = 0xffffffffu;
  b = 0u;
#pragma unroll
  for (int q = 0; q < kSelWarps; ++q) {
    a = min(a, s.wred[q]);
    b = max(b, s.wred2[q]);
  }
  __syncthreads();
  *mn = a;
  *mx = b;
}

__device__ __forceinline__ int diff_bits(uint32_t a, uint32_t b) {
  const uint32_t d = a ^ b;
  return d ? 32 - __clz(d) : 0;
}

__global__ void __launch_bounds__(kSelThreads)
    select_kernel(const int64_t* __restrict__ tok_off, int U, int w, const float* __restrict__ a,
                  const float* __restrict__ r, float lam, int max_budget,
                  const int32_t* __restrict__ budgets, int sinks, int W,
                  int32_t* __restrict__ idx, int32_t* __restrict__ n_kept) {
  __shared__ SelShared s;
  extern __shared__ uint32_t bits[];   // kept bitmap, ceil(c / 32) words
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const float lw = lam, rw = 1.f - lam;
  const int u = blockIdx.x;
  if (u >= U) return;

  const int64_t tbase = tok_off[u];
  const int N = static_cast<int>(tok_off[u + 1] - tbase);
  const int c0 = N - w;                       // candidates, sinks included
  const int m = min(sinks, c0);               // sinks: always kept, not ranked
  const int c = c0 - m;                       // ranked candidates m .. c0 - 1
  const int64_t base = tbase + m;             // a, r of ranked candidate i at base + i
  int budget = max_budget;
  if (budgets) budget = min(max(budgets[u], 0), max_budget);
  int32_t* out = idx + static_cast<int64_t>(u) * W;
  if (c <= budget) {  // every token is kept
    for (int i = tid; i < W; i += kSelThreads) out[i] = i < N ? i : -1;
    if (tid == 0) n_kept[u] = N;
    return;
  }
  // sinks, the window after the selected candidates, and the unused tail
  for (int t = tid; t < W - budget; t += kSelThreads) {
    if (t < m) out[t] = t;
    else if (t < m + w) out[budget + t] = c0 + (t - m);
    else out[budget + t] = -1;
  }
  if (tid == 0) n_kept[u] = m + budget + w;
  if (budget == 0) return;
  out += m;   // selected candidates follow the sinks

  const float* au = a + base;
  const float* ru = r + base;
  auto key_at = [&](int i) -> uint32_t {
    return order_key(__fsub_rn(__fmul_rn(lw, __ldg(au + i)), __fmul_rn(rw, __ldg(ru + i))));
  };
  const int nwords = (c + 31) >> 5;

  // ---- 1. sample and splitters
  const int S = min(kSample, c);
  for (int j = tid; j < S; j += kSelThreads)
    s.sample[j] = key_at(static_cast<int>((static_cast<int64_t>(j) * c) / S));
  if (tid == 0) {
    s.nlist = 0;
    s.cnt_above = 0;
  }
  __syncthreads();
  const float p = static_cast<float>(budget) / static_cast<float>(c);
  const float kpos = p * static_cast<float>(S);
  const float sd = sqrtf(kpos * (1.f - p)) + 1.f;
  const int r_hi = max(1, static_cast<int>(floorf(kpos - kSpread * sd)));   // 1-based ranks
  const int r_lo = min(S, static_cast<int>(ceilf(kpos + kSpread * sd)));
  auto get_sample = [&](int i, uint32_t& v) {
    v = s.sample[i];
    return true;
  };
  uint32_t smin, smax;
  min_max(s, get_sample, S, &smin, &smax);
  int dummy;
  const int sbits = diff_bits(smin, smax);
  const uint32_t hi = kth_largest(s, get_sample, S, r_hi, smin, sbits, &dummy);
  const uint32_t lo = kth_largest(s, get_sample, S, r_lo, smin, sbits, &dummy);

  // ---- 2. classify every candidate (a warp takes 32 consecutive ones)
  int above = 0;
  for (int wd = wp; wd < nwords; wd += kSelWarps) {
    const int i = wd * 32 + lane;
    const bool v = i < c;
    const uint32_t k = v ? key_at(i) : 0u;
    const unsigned ab = __ballot_sync(0xffffffffu, v && k > hi);
    const bool inb = v && k >= lo && k <= hi;
    const unsigned br = __ballot_sync(0xffffffffu, inb);
    if (lane == 0) bits[wd] = ab;
    above += __popc(ab);
    if (br) {
      int pos0 = 0;
      if (lane == 0) pos0 = atomicAdd(&s.nlist, __popc(br));
      pos0 = __shfl_sync(0xffffffffu, pos0, 0);
      const int pos = pos0 + __popc(br & ((1u << lane) - 1u));
      if (inb && pos < kListCap) {
        s.lkey[pos] = k;
        s.lidx[pos] = i;
      }
    }
  }
  if (lane == 0) atomicAdd(&s.cnt_above, above);
  __syncthreads();
  const int A = s.cnt_above;
  const int nl = s.nlist;
  const int want = budget - A;   // keys still to take from the bracket

  if (want >= 1 && want <= nl && nl <= kListCap) {
    // ---- 3. exact threshold inside the bracket
    auto get_list = [&](int i, uint32_t& v) {
      v = s.lkey[i];
      return true;
    };
    int gt;
    const int lbits = diff_bits(lo, hi);
    const uint32_t T = kth_largest(s, get_list, nl, want, lo, lbits, &gt);
    const int take_eq = want - gt;   // keys equal to T that are kept
    // the take_eq-th smallest index among the list keys equal to T
    // (values ~index: the largest is the smallest index)
    auto get_tied = [&](int i, uint32_t& v) {
      v = ~static_cast<uint32_t>(s.lidx[i]);
      return s.lkey[i] == T;
    };
    int dummy2;
    const uint32_t cut = kth_largest(s, get_tied, nl, take_eq, 0u, 32, &dummy2);
    const int imax = static_cast<int>(~cut);
    for (int i = tid; i < nl; i += kSelThreads) {
      const uint32_t k = s.lkey[i];
      const int ii = s.lidx[i];
      if (k > T || (k == T && ii <= imax)) atomicOr(&bits[ii >> 5], 1u << (ii & 31));
    }
  } else {
    // ---- 3'. the bracket missed the budget's rank or overflowed: select over
    // all candidates, reading a and r again
    auto get_all = [&](int i, uint32_t& v) {
      v = key_at(i);
      return true;
    };
    uint32_t kmin, kmax;
    min_max(s, get_all, c, &kmin, &kmax);
    int gt;
    const uint32_t T = kth_largest(s, get_all, c, budget, kmin, diff_bits(kmin, kmax), &gt);
    const int take_eq = budget - gt;
    auto get_tied = [&](int i, uint32_t& v) {
      v = ~static_cast<uint32_t>(i);
      return key_at(i) == T;
    };
    int dummy2;
    const uint32_t cut = kth_largest(s, get_tied, c, take_eq, 0u, 32, &dummy2);
    const int imax = static_cast<int>(~cut);
    for (int wd = wp; wd < nwords; wd += kSelWarps) {
      const int i = wd * 32 + lane;
      const bool v = i < c;
      const uint32_t k = v ? key_at(i) : 0u;
      const unsigned kb = __ballot_sync(0xffffffffu, v && (k > T || (k == T && i <= imax)));
      if (lane == 0) bits[wd] = kb;
    }
  }
  __syncthreads();

  // ---- 4. bitmap -> ascending indices
  const int per = (nwords + kSelThreads - 1) / kSelThreads;
  const int w0 = min(nwords, tid * per), w1 = min(nwords, w0 + per);
  int cnt = 0;
  for (int q = w0; q < w1; ++q) cnt += __popc(bits[q]);
  // block exclusive scan of cnt
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s.wred[wp] = static_cast<uint32_t>(incl);
  __syncthreads();
  int wbase = 0;
  for (int q = 0; q < wp; ++q) wbase += static_cast<int>(s.wred[q]);
  int pos = wbase + incl - cnt;
  for (int q = w0; q < w1; ++q) {
    uint32_t x = bits[q];
    while (x) {
      const int b = __ffs(x) - 1;
      x &= x - 1;
      if (pos < budget) out[pos] = m + q * 32 + b;
      ++pos;
    }
  }
}

}  // namespace

cudaError_t select_configure() {
  // the kept bitmap of the longest unit
  return cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (kMaxTokensPerUnit / 32 + 1) * 4);
}

cudaError_t launch_select(const int64_t* tok_off, int U, int w, int cmax, const float* a,
                          const float* r, float lam, int budget, const int32_t* budgets,
                          int sinks, int W, int32_t* idx, int32_t* n_kept, cudaStream_t st) {
  const size_t smem = (static_cast<size_t>(cmax > 0 ? cmax : 0) / 32 + 1) * 4;
  select_kernel<<<U, kSelThreads, smem, st>>>(tok_off, U, w, a, r, lam, budget, budgets, sinks,
                                              W, idx, n_kept);
  return cudaGetLastError();
}

}  // namespace rkv
