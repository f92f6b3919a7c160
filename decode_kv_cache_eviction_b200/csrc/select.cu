// Joint eviction (R-KV 联合淘汰): s_i = lambda * a_i - (1 - lambda) * r_i and a
// deterministic top-B of the candidates, one CTA per unit.
//
// The fp32 scores are mapped to order-preserving uint32 keys and kept in shared
// memory (one HBM read of a and r).  A 4-pass radix select (8-bit digits, most
// significant first) finds the exact key T of the B-th largest score and how
// many keys equal to T must be taken; equal keys are taken lowest index first.
// The kept set is then written in ascending index order: each warp owns a
// contiguous segment of the candidates, counts its "greater" and "equal" keys,
// and after one block-level prefix over the warps it writes its positions with
// ballots, with no further block synchronisation.
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

__device__ __forceinline__ uint32_t order_key(float s) {
  uint32_t b = __float_as_uint(s);
  if ((b << 1) == 0) b = 0;  // -0 and +0 compare equal
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

template <int NT>
__global__ void __launch_bounds__(NT) select_kernel(const int64_t* __restrict__ tok_off, int w,
                                                    const float* __restrict__ a,
                                                    const float* __restrict__ r, float lam,
                                                    int budget, int32_t* __restrict__ idx,
                                                    int32_t* __restrict__ n_kept) {
  constexpr int NW = NT / 32;
  extern __shared__ uint32_t keys[];
  __shared__ int hist[257];
  __shared__ int sh[2];
  __shared__ int wgt[NW], weq[NW], eqb[NW], outb[NW];
  const int u = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const int64_t base = tok_off[u];
  const int N = static_cast<int>(tok_off[u + 1] - base);
  const int c = N - w;
  const int W = budget + w;
  int32_t* out = idx + static_cast<int64_t>(u) * W;

  if (c <= budget) {  // every token is kept
    for (int i = tid; i < W; i += NT) out[i] = i < N ? i : -1;
    if (tid == 0) n_kept[u] = N;
    return;
  }
  const float lw = lam, rw = 1.f - lam;
  for (int i = tid; i < c; i += NT) {
    const float s = __fsub_rn(__fmul_rn(lw, a[base + i]), __fmul_rn(rw, r[base + i]));
    keys[i] = order_key(s);
  }
  __syncthreads();

  // ---- radix select of the budget-th largest key
  int want = budget;
  uint32_t prefix = 0, pmask = 0;
  const int cround = (c + 31) & ~31;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int b = tid; b < 257; b += NT) hist[b] = 0;
    __syncthreads();
    for (int i = tid; i < cround; i += NT) {
      uint32_t bin = 256;
      if (i < c) {
        const uint32_t k = keys[i];
        if ((k & pmask) == prefix) bin = (k >> shift) & 255u;
      }
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin < 256 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
    }
    __syncthreads();
    if (wp == 0) {
      int cnt[8], tot = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        cnt[k] = hist[255 - 8 * lane - k];
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
            break;
          }
          run += cnt[k];
        }
      }
    }
    __syncthreads();
    want -= sh[1];
    prefix |= static_cast<uint32_t>(sh[0]) << shift;
    pmask |= 255u << shift;
    __syncthreads();
  }
  const uint32_t T = prefix;  // key of the budget-th largest score
  const int take_eq = want;   // keys equal to T that are kept (lowest indices)

  // ---- per-warp segments, counts, then ordered output
  const int seg = (((c + NW - 1) / NW) + 31) & ~31;
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
    for (int x = 0; x < NW; ++x) {
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
    if (f) out[oseen + __popc(bf & lt)] = i;
    eseen += __popc(be);
    oseen += __popc(bf);
  }
  for (int t = tid; t < w; t += NT) out[budget + t] = c + t;
  if (tid == 0) n_kept[u] = budget + w;
}

}  // namespace

cudaError_t select_configure() {
  const int smem = kMaxTokensPerUnit * 4;
  cudaError_t e;
  e = cudaFuncSetAttribute(select_kernel<1024>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(select_kernel<512>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(select_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

cudaError_t launch_select(const int64_t* tok_off, int U, int w, int cmax, const float* a,
                          const float* r, float lam, int budget, int32_t* idx, int32_t* n_kept,
                          cudaStream_t st) {
  const size_t smem = cmax > budget ? static_cast<size_t>(cmax) * 4 : 0;
  if (cmax > 16384)
    select_kernel<1024><<<U, 1024, smem, st>>>(tok_off, w, a, r, lam, budget, idx, n_kept);
  else if (cmax > 4096)
    select_kernel<512><<<U, 512, smem, st>>>(tok_off, w, a, r, lam, budget, idx, n_kept);
  else
    select_kernel<256><<<U, 256, smem, st>>>(tok_off, w, a, r, lam, budget, idx, n_kept);
  return cudaGetLastError();
}

}  // namespace rkv
