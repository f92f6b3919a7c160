// Joint eviction (R-KV 联合淘汰): s_i = lambda * a_i - (1 - lambda) * r_i and a
// deterministic top-B of the candidates: the B largest by (s descending, index
// ascending), written in ascending index order.
//
// One CTA per unit (several CTAs share an SM).  s is mapped to an
// order-preserving uint32 key; keys are recomputed from a and r wherever they
// are needed, so a unit of any length needs no shared-memory copy of them.
//   1. Sample: the keys of S candidates in evenly spaced blocks of 8 (whole
//      32-byte sectors).  Two order statistics of the sample, about four
//      standard deviations of the sampling error above and below the budget's
//      rank, give splitters hi >= lo.
//   2. Classify (the one pass that reads a and r from HBM): every candidate is
//      above the bracket (key > hi, kept for sure), inside it (lo <= key <= hi,
//      appended with its index to a short list) or below.  A warp handles runs
//      of 32 consecutive candidates, sixteen runs' loads in flight at once, so
//      the "above" ballot of a run is directly one 32-bit word of the kept
//      bitmap.
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

#ifdef RKV_TRACE
// Optional phase trace (build with -DRKV_TRACE): globaltimer stamps of the
// first kStCtas units' phases.
constexpr int kStCtas = 64, kStSlots = 8;
__device__ unsigned long long g_sel_trace[kStCtas * kStSlots];
#define RKV_SSTAMP(slot)                                                                  \
  do {                                                                                    \
    if (threadIdx.x == 0 && blockIdx.x < kStCtas)                                         \
      g_sel_trace[blockIdx.x * kStSlots + (slot)] = globaltimer_ns();                     \
  } while (0)
#else
#define RKV_SSTAMP(slot) do { } while (0)
#endif

constexpr int kSelThreads = 128;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSample = 2048;     // sample size (at most the candidate count)
constexpr int kListCap = 3072;    // bracket entries kept on chip
constexpr float kSpread = 4.f;    // bracket half-width in sampling standard deviations

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t b = __float_as_uint(s);
  if ((b << 1) == 0) b = 0;  // -0 and +0 compare equal
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct SelShared {
  uint32_t hist[512];
  union {                        // the sample is done with before the list fills
    uint32_t sample[kSample];
    uint32_t lkey[kListCap];
  };
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
                                int lo_bits, int* above, int* equal = nullptr) {
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  uint32_t pmask = lo_bits >= 32 ? 0u : ~((1u << lo_bits) - 1u);
  prefix &= pmask;
  int want = k, gt = 0, eq = -1;   // eq: matches equal to the result (-1: all of them)
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
            s.sh[2] = cnt[q];
            break;
          }
          run += cnt[q];
        }
      }
    }
    __syncthreads();
    want -= s.sh[1];
    gt += s.sh[1];
    eq = s.sh[2];
    prefix |= static_cast<uint32_t>(s.sh[0]) << shift;
    pmask |= dmask << shift;
    lo = shift;
    __syncthreads();   // sh and hist are reused
  }
  *above = gt;
  if (equal) *equal = eq;
  return prefix;
}

// Block-wide: the k1-th and k2-th largest (k1 <= k2) of the n sample values in
// shared memory, by radix selection on both ranks at once: while the two
// prefixes agree one histogram serves both, afterwards each value counts in
// the histogram of the prefix it matches.
__device__ void two_kth_largest(SelShared& s, const uint32_t* vals, int n, int k1, int k2,
                                uint32_t prefix, int lo_bits, uint32_t* out1, uint32_t* out2) {
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  uint32_t pmask = lo_bits >= 32 ? 0u : ~((1u << lo_bits) - 1u);
  uint32_t p1 = prefix & pmask, p2 = prefix & pmask;
  int want1 = k1, want2 = k2;
  int lo = lo_bits;
  while (lo > 0) {
    const int d = min(8, lo);
    const int shift = lo - d;
    const uint32_t dmask = (1u << d) - 1u;
    const bool same = p1 == p2;
    for (int b = tid; b < 512; b += kSelThreads) s.hist[b] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kSelThreads) {
      const uint32_t v = vals[i];
      const uint32_t bin = (v >> shift) & dmask;
      if ((v & pmask) == p1) atomicAdd(&s.hist[bin], 1u);
      else if (!same && (v & pmask) == p2) atomicAdd(&s.hist[256 + bin], 1u);
    }
    __syncthreads();
    if (wp < 2) {
      // warp 0 resolves rank 1, warp 1 rank 2 (from the shared histogram
      // while the prefixes agree)
      const uint32_t* h = s.hist + ((wp == 1 && !same) ? 256 : 0);
      const int want = wp == 0 ? want1 : want2;
      int cnt[8], tot = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        cnt[q] = static_cast<int>(h[255 - 8 * lane - q]);
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
            s.sh[2 * wp] = 255 - 8 * lane - q;
            s.sh[2 * wp + 1] = run;
            break;
          }
          run += cnt[q];
        }
      }
    }
    __syncthreads();
    want1 -= s.sh[1];
    want2 -= s.sh[3];
    p1 |= static_cast<uint32_t>(s.sh[0]) << shift;
    p2 |= static_cast<uint32_t>(s.sh[2]) << shift;
    pmask |= dmask << shift;
    lo = shift;
    __syncthreads();   // sh and hist are reused
  }
  *out1 = p1;
  *out2 = p2;
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

__global__ void __launch_bounds__(kSelThreads, 7)
    select_kernel(const int64_t* __restrict__ tok_off, int U, int64_t Ttot, int w,
                  const float* __restrict__ a,
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

  RKV_SSTAMP(0);
  const float* au = a + base;
  const float* ru = r + base;

  auto key_at = [&](int i) -> uint32_t {
    return order_key(__fsub_rn(__fmul_rn(lw, __ldg(au + i)), __fmul_rn(rw, __ldg(ru + i))));
  };
  // position p = i + delta of candidate i (see step 2); the kept bitmap has
  // one bit per position
  const bool vec_ok = ((reinterpret_cast<uintptr_t>(au) ^ reinterpret_cast<uintptr_t>(ru)) & 15) == 0;
  const int delta = vec_ok ? static_cast<int>((reinterpret_cast<uintptr_t>(au) >> 2) & 3) : 0;
  const int64_t p0 = base - delta;   // element of a and r at position 0
  const int npos = c + delta;
  const int nruns = (npos + 127) >> 7;
  const int nwords = (npos + 31) >> 5;

  // ---- 1. sample and splitters: S / 8 evenly spaced blocks of 8 consecutive
  // candidates (whole 32-byte sectors of a and r), S about c / 8 within
  // [256, kSample]
  const int S = min(c, min(kSample, max(256, ((c / 8) + 7) & ~7)));
  {
    const int nblk = S / 8;
    constexpr int kPer = kSample / kSelThreads;   // sample keys per thread (at most)
    float sa[kPer], sr[kPer];
#pragma unroll
    for (int x = 0; x < kPer; ++x) {   // every load first, then the keys
      const int j = tid + x * kSelThreads;
      int i = j;   // fewer than 8 candidates in a block's place: take them all
      if (j < nblk * 8)
        i = static_cast<int>((static_cast<int64_t>(j >> 3) * (c - 8)) / max(nblk - 1, 1)) +
            (j & 7);
      i = min(i, c - 1);
      sa[x] = j < S ? __ldg(au + i) : 0.f;
      sr[x] = j < S ? __ldg(ru + i) : 0.f;
    }
#pragma unroll
    for (int x = 0; x < kPer; ++x) {
      const int j = tid + x * kSelThreads;
      if (j < S) s.sample[j] = order_key(__fsub_rn(__fmul_rn(lw, sa[x]), __fmul_rn(rw, sr[x])));
    }
  }
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
  RKV_SSTAMP(1);
  uint32_t smin, smax;
  min_max(s, get_sample, S, &smin, &smax);
  uint32_t hi, lo;
  two_kth_largest(s, s.sample, S, r_hi, r_lo, smin, diff_bits(smin, smax), &hi, &lo);

  RKV_SSTAMP(2);
  // ---- 2. classify every candidate.  Positions p = i + delta, delta = the
  // offset of candidate 0 within its 16-byte group of scores, so that a run of
  // 128 positions is 32 aligned float4 of a and of r: lane l takes positions
  // 4l .. 4l+3, and the kept bitmap is kept per position (bit p).  Runs that
  // would read outside [0, T) take bounds-checked scalar loads.
  constexpr int kRuns = 4;   // runs per warp and iteration, all loads in flight
  int above = 0;
  for (int r0 = wp * kRuns; r0 < nruns; r0 += kSelWarps * kRuns) {
    float4 A[kRuns], R[kRuns];
#pragma unroll
    for (int x = 0; x < kRuns; ++x) {
      const int64_t ge = p0 + static_cast<int64_t>(r0 + x) * 128 + 4 * lane;   // element of a, r
      if (r0 + x < nruns && ge >= 0 && ge + 3 < Ttot && vec_ok) {
        A[x] = __ldg(reinterpret_cast<const float4*>(a + ge));
        R[x] = __ldg(reinterpret_cast<const float4*>(r + ge));
      } else {
        float ta[4], tr[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = (r0 + x) * 128 + 4 * lane + e - delta;
          ta[e] = (i >= 0 && i < c) ? __ldg(au + i) : 0.f;
          tr[e] = (i >= 0 && i < c) ? __ldg(ru + i) : 0.f;
        }
        A[x] = make_float4(ta[0], ta[1], ta[2], ta[3]);
        R[x] = make_float4(tr[0], tr[1], tr[2], tr[3]);
      }
    }
#pragma unroll
    for (int x = 0; x < kRuns; ++x) {
      if (r0 + x >= nruns) break;
      const float av[4] = {A[x].x, A[x].y, A[x].z, A[x].w};
      const float rv[4] = {R[x].x, R[x].y, R[x].z, R[x].w};
      uint32_t nab = 0, nin = 0, keys[4];
      const int i0 = (r0 + x) * 128 + 4 * lane - delta;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool v = i0 + e >= 0 && i0 + e < c;
        const uint32_t k = order_key(__fsub_rn(__fmul_rn(lw, av[e]), __fmul_rn(rw, rv[e])));
        keys[e] = k;
        nab |= (v && k > hi) ? (1u << e) : 0u;
        nin |= (v && k >= lo && k <= hi) ? (1u << e) : 0u;
      }
      // bitmap word 4 (r0 + x) + l / 8 holds the nibbles of lanes 8 (l / 8) ..
      uint32_t wv = nab << (4 * (lane & 7));
      wv |= __shfl_xor_sync(0xffffffffu, wv, 1);
      wv |= __shfl_xor_sync(0xffffffffu, wv, 2);
      wv |= __shfl_xor_sync(0xffffffffu, wv, 4);
      if ((lane & 7) == 0) bits[(r0 + x) * 4 + (lane >> 3)] = wv;
      above += __popc(nab);
      // bracket entries go to the list (warp prefix of the counts)
      const int cnt = __popc(nin);
      if (__any_sync(0xffffffffu, cnt > 0)) {
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        int pos0 = 0;
        if (lane == 31) pos0 = atomicAdd(&s.nlist, incl);
        pos0 = __shfl_sync(0xffffffffu, pos0, 31);
        int my = pos0 + incl - cnt;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if ((nin >> e) & 1u) {
            if (my < kListCap) {
              s.lkey[my] = keys[e];
              s.lidx[my] = i0 + e;
            }
            ++my;
          }
      }
    }
  }
  above = __reduce_add_sync(0xffffffffu, above);   // each lane counted its own candidates
  if (lane == 0) atomicAdd(&s.cnt_above, above);
  __syncthreads();
  RKV_SSTAMP(3);
  const int A = s.cnt_above;
  const int nl = s.nlist;
  const int want = budget - A;   // keys still to take from the bracket

  if (want >= 1 && want <= nl && nl <= kListCap) {
    // ---- 3. exact threshold inside the bracket
    auto get_list = [&](int i, uint32_t& v) {
      v = s.lkey[i];
      return true;
    };
    int gt, eq;
    const int lbits = diff_bits(lo, hi);
    const uint32_t T = kth_largest(s, get_list, nl, want, lo, lbits, &gt, &eq);
    const int take_eq = want - gt;   // keys equal to T that are kept
    int imax = 0x7fffffff;           // every key equal to T is kept ...
    if (eq < 0 || take_eq < eq) {
      // ... unless only some are: the take_eq-th smallest index among the list
      // keys equal to T (values ~index: the largest is the smallest index)
      auto get_tied = [&](int i, uint32_t& v) {
        v = ~static_cast<uint32_t>(s.lidx[i]);
        return s.lkey[i] == T;
      };
      int dummy2;
      imax = static_cast<int>(~kth_largest(s, get_tied, nl, take_eq, 0u, 32, &dummy2));
    }
    for (int i = tid; i < nl; i += kSelThreads) {
      const uint32_t k = s.lkey[i];
      const int ii = s.lidx[i];
      if (k > T || (k == T && ii <= imax))
        atomicOr(&bits[(ii + delta) >> 5], 1u << ((ii + delta) & 31));
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
      const int i = wd * 32 + lane - delta;
      const bool v = i >= 0 && i < c;
      const uint32_t k = v ? key_at(i) : 0u;
      const unsigned kb = __ballot_sync(0xffffffffu, v && (k > T || (k == T && i <= imax)));
      if (lane == 0) bits[wd] = kb;
    }
  }
  __syncthreads();

  RKV_SSTAMP(4);
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
      if (pos < budget) out[pos] = m + q * 32 + b - delta;
      ++pos;
    }
  }
  RKV_SSTAMP(5);
}

// Bytes of the kept bitmap for units of up to c candidates: positions c + 3
// rounded up to whole runs of 128, one bit each.
size_t bitmap_bytes(int c) { return static_cast<size_t>((c + 3 + 127) / 128) * 16 + 16; }

}  // namespace

cudaError_t select_configure() {
  return cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bitmap_bytes(kMaxTokensPerUnit)));
}

cudaError_t launch_select(const int64_t* tok_off, int U, int64_t Ttot, int w, int cmax,
                          const float* a,
                          const float* r, float lam, int budget, const int32_t* budgets,
                          int sinks, int W, int32_t* idx, int32_t* n_kept, cudaStream_t st) {
  // the kept bitmap: every position of the longest unit, in whole runs of 128
  const size_t smem = bitmap_bytes(cmax > 0 ? cmax : 0);
  select_kernel<<<U, kSelThreads, smem, st>>>(tok_off, U, Ttot, w, a, r, lam, budget, budgets,
                                              sinks, W, idx, n_kept);
  return cudaGetLastError();
}

}  // namespace rkv

#ifdef RKV_TRACE
extern "C" int rkv_debug_select_trace(void* dst, size_t bytes) {
  return static_cast<int>(cudaMemcpyFromSymbol(dst, rkv::g_sel_trace, bytes));
}
#endif
