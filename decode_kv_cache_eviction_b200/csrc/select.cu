// Joint eviction (R-KV 联合淘汰): s_i = lambda * a_i - (1 - lambda) * r_i and a
// deterministic top-B of the candidates: the B largest by (s descending, index
// ascending), written in ascending index order.  A NaN score ranks below every
// number (ties among NaNs by index, like the other ties).
//
// One CTA per unit: 128 threads (seven per SM) when the longest unit has more
// than kShortMaxCand candidates, else 64 threads with half the sample and list
// capacity (fourteen per SM).  s is mapped to an order-preserving uint32 key
// where a key is needed; a unit of any length needs no shared-memory copy of
// its scores.
//   1. Sample: the keys of S candidates in evenly spaced blocks of 16 (whole
//      64-byte segments of a and of r).  Two order statistics of the sample,
//      about four standard deviations of the sampling error above and below the
//      budget's rank, give splitters hi >= lo (as keys and as floats).
//   2. Classify (the one pass that reads a and r from HBM): every candidate is
//      above the bracket (s > hi, kept for sure), inside it (lo <= s <= hi,
//      appended with its index to a short list) or below.  A warp takes runs of
//      128 positions, lane l the aligned float4 of positions 4l .. 4l+3 of a
//      and of r, four runs' loads in flight.  Plain float compares against the
//      splitters decide (the key order is the float order); only list entries
//      get a key.  List slots come from four ballots per run and one shared
//      atomic per warp and run.
//   3. If the budget's rank falls inside the bracket and the list fits, the
//      exact threshold key T and the tie cut (keys equal to T are taken lowest
//      index first) are found by radix selection on the list alone, and the
//      kept list entries are added to the bitmap.  Otherwise (rare: many equal
//      keys, or a sample far from the data) the same selection runs over all
//      candidates, reading a and r again.
//   4. The bitmap is turned into ascending indices: each warp takes a
//      contiguous share of the words, one word per lane at a time.
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
// first kStCtas units' phases (slot 6: the SM, slot 7: kernel entry).
constexpr int kStCtas = 1024, kStSlots = 8;
__device__ unsigned long long g_sel_trace[kStCtas * kStSlots];
#define RKV_SSTAMP(slot)                                                                  \
  do {                                                                                    \
    if (threadIdx.x == 0 && blockIdx.x < kStCtas)                                         \
      g_sel_trace[blockIdx.x * kStSlots + (slot)] = globaltimer_ns();                     \
  } while (0)
#else
#define RKV_SSTAMP(slot) do { } while (0)
#endif

// Launch shape and on-chip capacities: threads, sample size (at most the
// candidate count), bracket entries kept on chip.  Units of at most
// kShortMaxCand candidates take the short shape, so that twice as many units
// (and their latency-bound phases) share an SM.
template <int NT, int SMP, int LC, int MINB>
struct SelCfg {
  static constexpr int kThreads = NT, kWarps = NT / 32, kSample = SMP, kListCap = LC,
                       kMinBlocks = MINB;
};
using LongSel = SelCfg<128, 2048, 3072, 7>;
using ShortSel = SelCfg<64, 1024, 1536, 14>;
constexpr int kShortMaxCand = 8192;
constexpr float kSpread = 4.f;    // bracket half-width in sampling standard deviations

// Order-preserving key of a score: -0 and +0 get the key of +0, a NaN key 0
// (below every number's key, which is at least that of -inf, 0x007fffff).
__device__ __forceinline__ uint32_t order_key(float s) {
  const uint32_t b = __float_as_uint(__fadd_rn(s, 0.f));   // -0 + 0 = +0
  const uint32_t k = b ^ (static_cast<uint32_t>(static_cast<int32_t>(b) >> 31) | 0x80000000u);
  return s == s ? k : 0u;
}
// The float whose key is k (k = 0 gives a NaN, which no compare accepts).
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

template <class C>
struct SelShared {
  uint32_t hist[512];
  union {                        // the sample is done with before the list fills
    uint32_t sample[C::kSample];
    uint2 list[C::kListCap];        // bracket entries: (score bits, candidate index)
  };
  int nlist;
  int cnt_above;
  int sh[8];
  uint32_t wred[C::kWarps];
  uint32_t wred2[C::kWarps];
};

// Block-wide: the k-th largest (1 <= k <= number of matches) of the values
// get(i) over i in [0, n) for which get returns valid, radix-selected most
// significant digit first.  `lo_bits` is the number of low bits in which the
// values may differ (bits above are common to all: `prefix`).  Returns the
// value; *above receives the number of matching values strictly greater.
template <class C, class Get>
__device__ uint32_t kth_largest(SelShared<C>& s, Get get, int n, int k, uint32_t prefix,
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
    for (int b = tid; b < 256; b += C::kThreads) s.hist[b] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += C::kThreads) {
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
template <class C>
__device__ void two_kth_largest(SelShared<C>& s, const uint32_t* vals, int n, int k1, int k2,
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
    for (int b = tid; b < 512; b += C::kThreads) s.hist[b] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += C::kThreads) {
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
template <class C, class Get>
__device__ void min_max(SelShared<C>& s, Get get, int n, uint32_t* mn, uint32_t* mx) {
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  uint32_t a = 0xffffffffu, b = 0u;
  for (int i = tid; i < n; i += C::kThreads) {
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
  for (int q = 0; q < C::kWarps; ++q) {
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

template <class C>
__global__ void __launch_bounds__(C::kThreads, C::kMinBlocks)
    select_kernel(const int64_t* __restrict__ tok_off, int U, int64_t Ttot, int w,
                  const float* __restrict__ a,
                  const float* __restrict__ r, float lam, int max_budget,
                  const int32_t* __restrict__ budgets, int sinks, int W,
                  int32_t* __restrict__ idx, int32_t* __restrict__ n_kept) {
  __shared__ SelShared<C> s;
  extern __shared__ uint32_t bits[];   // kept bitmap, ceil(c / 32) words
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const float lw = lam, rw = 1.f - lam;
  const int u = blockIdx.x;
  if (u >= U) return;
#ifdef RKV_TRACE
  if (threadIdx.x == 0 && blockIdx.x < kStCtas) {
    g_sel_trace[blockIdx.x * kStSlots + 7] = globaltimer_ns();
    unsigned smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    g_sel_trace[blockIdx.x * kStSlots + 6] = smid;
  }
#endif

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
    for (int i = tid; i < W; i += C::kThreads) out[i] = i < N ? i : -1;
    if (tid == 0) n_kept[u] = N;
    return;
  }
  // sinks, the window after the selected candidates, and the unused tail
  for (int t = tid; t < W - budget; t += C::kThreads) {
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

  // runs [run_lo, run_hi) take 128-bit loads: every element they touch lies in
  // [0, T) (p0 >= -3, so only run 0 can start before the array)
  int run_lo = 0, run_hi = 0;
  if (vec_ok) {
    run_lo = p0 >= 0 ? 0 : 1;
    run_hi = static_cast<int>(min(static_cast<int64_t>(nruns), (Ttot - p0) / 128));
  }
  // lane's float4 of run run_lo (in bounds whenever run_lo < run_hi)
  const int64_t g_lo = p0 + static_cast<int64_t>(run_lo) * 128 + 4 * lane;
  const float4* a4 = reinterpret_cast<const float4*>(a + (run_lo < run_hi ? g_lo : 0));
  const float4* r4 = reinterpret_cast<const float4*>(r + (run_lo < run_hi ? g_lo : 0));
  constexpr int kRuns = 4;   // runs per warp and iteration of the classification
  // the warp's first classification iteration into L2 while the sample and
  // the splitters are worked out
  if ((lane & 7) == 0) {
#pragma unroll
    for (int x = 0; x < kRuns; ++x) {
      const int run = wp * kRuns + x;
      if (run >= run_lo && run < run_hi) {
        prefetch_l2(a4 + 32 * (run - run_lo));
        prefetch_l2(r4 + 32 * (run - run_lo));
      }
    }
  }

  // ---- 1. sample and splitters: S / 16 evenly spaced blocks of 16 consecutive
  // candidates (64-byte segments of a and r), S about c / 8 within
  // [256, C::kSample]; every candidate when S = c
  const int S = min(c, min(C::kSample, max(256, ((c / 8) + 15) & ~15)));
  {
    const int nblk = S >> 4;
    const float step = nblk > 1 ? static_cast<float>(c - 16) / static_cast<float>(nblk - 1) : 0.f;
    constexpr int kPer = C::kSample / C::kThreads;   // sample keys per thread (at most)
    float sa[kPer], sr[kPer];
#pragma unroll
    for (int x = 0; x < kPer; ++x) {   // every load first, then the keys
      const int j = tid + x * C::kThreads;
      int i = j;   // all candidates, or fewer than 16 in a block's place: take them
      if (S < c && j < nblk * 16) i = static_cast<int>(static_cast<float>(j >> 4) * step) + (j & 15);
      i = min(i, c - 1);
      sa[x] = j < S ? __ldg(au + i) : 0.f;
      sr[x] = j < S ? __ldg(ru + i) : 0.f;
    }
#pragma unroll
    for (int x = 0; x < kPer; ++x) {
      const int j = tid + x * C::kThreads;
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
  // would read outside [0, T) take bounds-checked scalar loads.  s > f_hi and
  // lo <= key(s) <= hi are float compares (false for a NaN, whose key is the
  // lowest); only the list entries' keys are formed.
  const float f_hi = key_float(hi), f_lo = key_float(lo);
  int above = 0;
  for (int r0 = wp * kRuns; r0 < nruns; r0 += C::kWarps * kRuns) {
    float4 A[kRuns], R[kRuns];
#pragma unroll
    for (int x = 0; x < kRuns; ++x) {
      const int run = r0 + x;
      if (run >= run_lo && run < run_hi) {
        A[x] = __ldg(a4 + 32 * (run - run_lo));
        R[x] = __ldg(r4 + 32 * (run - run_lo));
      } else if (run < nruns) {
        float ta[4], tr[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = run * 128 + 4 * lane + e - delta;
          ta[e] = (i >= 0 && i < c) ? __ldg(au + i) : 0.f;
          tr[e] = (i >= 0 && i < c) ? __ldg(ru + i) : 0.f;
        }
        A[x] = make_float4(ta[0], ta[1], ta[2], ta[3]);
        R[x] = make_float4(tr[0], tr[1], tr[2], tr[3]);
      }
    }
    // the warp's next iteration into L2 while this one is processed (one
    // prefetch per 128-byte line)
    if ((lane & 7) == 0) {
#pragma unroll
      for (int x = 0; x < kRuns; ++x) {
        const int run = r0 + C::kWarps * kRuns + x;
        if (run >= run_lo && run < run_hi) {
          prefetch_l2(a4 + 32 * (run - run_lo));
          prefetch_l2(r4 + 32 * (run - run_lo));
        }
      }
    }
#pragma unroll
    for (int x = 0; x < kRuns; ++x) {
      const int run = r0 + x;
      if (run >= nruns) break;
      const float av[4] = {A[x].x, A[x].y, A[x].z, A[x].w};
      const float rv[4] = {R[x].x, R[x].y, R[x].z, R[x].w};
      const int i0 = run * 128 + 4 * lane - delta;
      float sv[4];
      uint32_t nab = 0, nin = 0;
      if (run * 128 >= delta && run * 128 + 128 - delta <= c) {
        // every position of the run holds a candidate
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          sv[e] = __fsub_rn(__fmul_rn(lw, av[e]), __fmul_rn(rw, rv[e]));
          const bool g = sv[e] > f_hi;
          nab |= g ? (1u << e) : 0u;
          nin |= (!g && sv[e] >= f_lo) ? (1u << e) : 0u;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          sv[e] = __fsub_rn(__fmul_rn(lw, av[e]), __fmul_rn(rw, rv[e]));
          const bool v = i0 + e >= 0 && i0 + e < c;
          const bool g = sv[e] > f_hi;
          nab |= (v && g) ? (1u << e) : 0u;
          nin |= (v && !g && sv[e] >= f_lo) ? (1u << e) : 0u;
        }
      }
      // bitmap word 4 run + l / 8 holds the nibbles of lanes 8 (l / 8) ..
      uint32_t wv = nab << (4 * (lane & 7));
      wv |= __shfl_xor_sync(0xffffffffu, wv, 1);
      wv |= __shfl_xor_sync(0xffffffffu, wv, 2);
      wv |= __shfl_xor_sync(0xffffffffu, wv, 4);
      if ((lane & 7) == 0) bits[run * 4 + (lane >> 3)] = wv;
      above += __popc(nab);
      // bracket entries (score bits, index): the lanes that have some take
      // their slots with one shared atomic each
      if (nin) {
        int q = atomicAdd(&s.nlist, __popc(nin));
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if ((nin >> e) & 1u) {
            if (q < C::kListCap)
              s.list[q] = make_uint2(__float_as_uint(sv[e]), static_cast<uint32_t>(i0 + e));
            ++q;
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

  if (want >= 1 && want <= nl && nl <= C::kListCap) {
    // ---- 3. exact threshold inside the bracket
    auto get_list = [&](int i, uint32_t& v) {
      v = order_key(__uint_as_float(s.list[i].x));
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
        const uint2 en = s.list[i];
        v = ~en.y;
        return order_key(__uint_as_float(en.x)) == T;
      };
      int dummy2;
      imax = static_cast<int>(~kth_largest(s, get_tied, nl, take_eq, 0u, 32, &dummy2));
    }
    for (int i = tid; i < nl; i += C::kThreads) {
      const uint2 en = s.list[i];
      const uint32_t k = order_key(__uint_as_float(en.x));
      const int ii = static_cast<int>(en.y);
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
    for (int wd = wp; wd < nwords; wd += C::kWarps) {
      const int i = wd * 32 + lane - delta;
      const bool v = i >= 0 && i < c;
      const uint32_t k = v ? key_at(i) : 0u;
      const unsigned kb = __ballot_sync(0xffffffffu, v && (k > T || (k == T && i <= imax)));
      if (lane == 0) bits[wd] = kb;
    }
  }
  __syncthreads();

  RKV_SSTAMP(4);
  // ---- 4. bitmap -> ascending indices: warp wp takes a contiguous share of
  // the words, one word per lane at a time
  const int perw = (nwords + C::kWarps - 1) / C::kWarps;
  const int w0 = min(nwords, wp * perw), w1 = min(nwords, w0 + perw);
  int cnt = 0;
  for (int q = w0 + lane; q < w1; q += 32) cnt += __popc(bits[q]);
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  if (lane == 0) s.wred[wp] = static_cast<uint32_t>(cnt);
  __syncthreads();
  int pos = 0;
  for (int q = 0; q < wp; ++q) pos += static_cast<int>(s.wred[q]);
  for (int q0 = w0; q0 < w1; q0 += 32) {
    const int q = q0 + lane;
    uint32_t x = q < w1 ? bits[q] : 0u;
    const int n = __popc(x);
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int my = pos + incl - n;
    pos += __shfl_sync(0xffffffffu, incl, 31);
    const int ob = m + q * 32 - delta;   // index of bit 0 of the word
    while (x) {   // two set bits per step
      const int b0 = __ffs(x) - 1;
      x &= x - 1;
      const int b1 = __ffs(x) - 1;   // -1: no second bit
      x &= x - 1;
      if (my < budget) out[my] = ob + b0;
      if (b1 >= 0 && my + 1 < budget) out[my + 1] = ob + b1;
      my += 2;
    }
  }
  RKV_SSTAMP(5);
}

// Bytes of the kept bitmap for units of up to c candidates: positions c + 3
// rounded up to whole runs of 128, one bit each.
size_t bitmap_bytes(int c) { return static_cast<size_t>((c + 3 + 127) / 128) * 16 + 16; }

}  // namespace

cudaError_t select_configure() {
  cudaError_t e = cudaFuncSetAttribute(select_kernel<LongSel>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(bitmap_bytes(kMaxTokensPerUnit)));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(select_kernel<ShortSel>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              static_cast<int>(bitmap_bytes(kShortMaxCand)));
}

cudaError_t launch_select(const int64_t* tok_off, int U, int64_t Ttot, int w, int cmax,
                          const float* a,
                          const float* r, float lam, int budget, const int32_t* budgets,
                          int sinks, int W, int32_t* idx, int32_t* n_kept, cudaStream_t st) {
  // the kept bitmap: every position of the longest unit, in whole runs of 128
  const int c = cmax > 0 ? cmax : 0;
  const size_t smem = bitmap_bytes(c);
  if (c <= kShortMaxCand)
    select_kernel<ShortSel><<<U, ShortSel::kThreads, smem, st>>>(
        tok_off, U, Ttot, w, a, r, lam, budget, budgets, sinks, W, idx, n_kept);
  else
    select_kernel<LongSel><<<U, LongSel::kThreads, smem, st>>>(
        tok_off, U, Ttot, w, a, r, lam, budget, budgets, sinks, W, idx, n_kept);
  return cudaGetLastError();
}

}  // namespace rkv

#ifdef RKV_TRACE
extern "C" int rkv_debug_select_trace(void* dst, size_t bytes) {
  return static_cast<int>(cudaMemcpyFromSymbol(dst, rkv::g_sel_trace, bytes));
}
#endif
