// Adaptive budget from the ReFreeKV review: one row of the attention matrix
// (k = 1, the newest query) stands for all of it, tokens are ranked as the
// first m sinks then newest to oldest, and the kept prefix stops where the
// Frobenius norm of the kept entries reaches (1 - T) of the row's norm.
//
// Per unit (one 256-thread CTA, persistent over units):
//   pass 1  logits z_g(j) = q_g . k_j / sqrt(d) of the G newest queries for
//           every key j, online max / sum per head g; the logits go to a
//           scratch array (GP floats per token, one coalesced store per warp
//           step), so K is read once;
//   pass 2  the logits back from the scratch (mostly from L2), p(j) =
//           mean_g exp(z_g(j) - M_g) / S_g, written to p_last, and e(j) =
//           p(j)^2 summed;
//   pass 3  the stopping point: the sinks' energy, then the suffix sums from
//           the newest token down until (1 - T)^2 of the total is reached.
//
// Logits on CUDA cores: lane l holds dimensions 4l .. 4l+3 of the (padded)
// GP queries; a warp takes 32 / GP tokens at a time (each token's K row is one
// coalesced 256-byte read), forms 32 partial dot products per lane and
// finishes them with a 31-shuffle transposed reduction, after which lane l
// holds the complete logit of token l / GP, head l % GP.
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

constexpr int kRfThreads = 256;
constexpr int kRfWarps = kRfThreads / 32;

// On return v[0] of lane l holds the sum over the warp's lanes of their v[l].
__device__ __forceinline__ float transpose_reduce(float (&v)[32], int lane) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool up = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = up ? v[i] : v[i + s];
      const float keep = up ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

template <int GP>
__global__ void __launch_bounds__(kRfThreads)
    refree_kernel(const int64_t* __restrict__ tok_off, int U, int G, int w,
                  const uint16_t* __restrict__ Q, const uint2* __restrict__ K, float scale_log2,
                  int sinks, float T, int max_budget, float* __restrict__ zbuf,
                  float* __restrict__ p_last, int32_t* __restrict__ budgets,
                  int32_t* __restrict__ keep_count) {
  constexpr int TB = 32 / GP;   // tokens per warp step
  __shared__ float red_m[kRfWarps][32], red_s[kRfWarps][32];
  __shared__ float fin_m[GP], fin_s[GP];
  __shared__ float wsum[kRfWarps];
  __shared__ float sh_e[2];
  __shared__ int sh_k;
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const int gl = lane % GP;          // head of this lane's finished logit
  const int tl = lane / GP;          // token (within the step) of that logit

  for (int u = blockIdx.x; u < U; u += gridDim.x) {
    const int64_t base = tok_off[u];
    const int N = static_cast<int>(tok_off[u + 1] - base);
    // the newest query of every head, dimensions 4 lane .. 4 lane + 3
    float q[GP][4];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      if (g < G) {
        const uint16_t* qp = Q + ((static_cast<int64_t>(u) * G + g) * w + (w - 1)) * 128 + 4 * lane;
        const uint2 qq = *reinterpret_cast<const uint2*>(qp);
        q[g][0] = bf_lo(qq.x); q[g][1] = bf_hi(qq.x);
        q[g][2] = bf_lo(qq.y); q[g][3] = bf_hi(qq.y);
      } else {
        q[g][0] = q[g][1] = q[g][2] = q[g][3] = 0.f;
      }
    }
    auto logit = [&](int j0) -> float {   // logit of (token j0 + tl, head gl), log2 units
      uint2 kk[TB];
#pragma unroll
      for (int t = 0; t < TB; ++t) {
        const int j = j0 + t;
        kk[t] = j < N ? __ldcs(&K[(base + j) * 32 + lane]) : make_uint2(0u, 0u);
      }
      float v[32];
#pragma unroll
      for (int t = 0; t < TB; ++t) {
        const float k0 = bf_lo(kk[t].x), k1 = bf_hi(kk[t].x);
        const float k2 = bf_lo(kk[t].y), k3 = bf_hi(kk[t].y);
#pragma unroll
        for (int g = 0; g < GP; ++g)
          v[t * GP + g] = fmaf(q[g][0], k0, fmaf(q[g][1], k1, fmaf(q[g][2], k2, q[g][3] * k3)));
      }
      return transpose_reduce(v, lane) * scale_log2;
    };
    const bool real = gl < G;

    // ---- pass 1: per-head max and sum of 2^(z - max)
    float rm = -INFINITY, rs = 0.f;
    float* zu = zbuf + base * GP;   // logit of (token j, head g) at zu[j * GP + g]
    for (int j0 = wp * TB; j0 < N; j0 += kRfWarps * TB) {
      const float z = logit(j0);
      if (j0 + tl < N) __stcg(&zu[j0 * GP + lane], z);
      if (real && j0 + tl < N) {
        if (z > rm) {
          rs = rs * ex2(rm - z) + 1.f;
          rm = z;
        } else {
          rs += ex2(z - rm);
        }
      }
    }
    red_m[wp][lane] = rm;
    red_s[wp][lane] = rs;
    __syncthreads();
    if (tid < GP) {
      float M = -INFINITY;
      for (int x = 0; x < kRfWarps; ++x)
        for (int l = tid; l < 32; l += GP) M = fmaxf(M, red_m[x][l]);
      float S = 0.f;
      for (int x = 0; x < kRfWarps; ++x)
        for (int l = tid; l < 32; l += GP)
          if (red_s[x][l] > 0.f) S += red_s[x][l] * ex2(red_m[x][l] - M);
      fin_m[tid] = M;
      fin_s[tid] = S > 0.f ? 1.f / S : 0.f;
    }
    __syncthreads();

    // ---- pass 2: p = mean over heads of the probabilities; energy
    const float Mg = fin_m[gl], invS = fin_s[gl];
    const float invG = 1.f / static_cast<float>(G);
    float esum = 0.f;
    for (int j0 = wp * TB; j0 < N; j0 += kRfWarps * TB) {
      const float z = j0 + tl < N ? __ldcg(&zu[j0 * GP + lane]) : 0.f;
      float pr = real ? ex2(z - Mg) * invS : 0.f;
#pragma unroll
      for (int o = 1; o < GP; o <<= 1) pr += __shfl_xor_sync(0xffffffffu, pr, o);
      const int j = j0 + tl;
      if (gl == 0 && j < N) {
        const float pj = pr * invG;
        p_last[base + j] = pj;
        esum = fmaf(pj, pj, esum);
      }
    }
    esum = warp_reduce_sum(esum);
    if (lane == 0) wsum[wp] = esum;
    __syncthreads();   // also orders the p_last writes before pass 3 reads them
    if (tid == 0) {
      float e = 0.f;
      for (int x = 0; x < kRfWarps; ++x) e += wsum[x];
      sh_e[0] = e;
    }
    __syncthreads();
    const float need = (1.f - T) * (1.f - T) * sh_e[0];

    // ---- pass 3: smallest prefix of (sinks, newest .. oldest) reaching `need`
    const int m = min(sinks, N);
    if (tid == 0) {
      float acc = 0.f;
      int k = 0;
      while (k < m) {
        const float pj = __ldcg(&p_last[base + k]);
        acc = fmaf(pj, pj, acc);
        ++k;
        if (acc >= need) break;
      }
      sh_e[1] = acc;
      sh_k = (acc >= need) ? k : -1;
    }
    __syncthreads();
    if (sh_k < 0) {
      // suffix sums from the newest token down, kRfThreads tokens per round;
      // thread t takes token N - 1 - (r0 + t)
      float run = sh_e[1];
      int found = -1;
      for (int r0 = 0; r0 < N - m && found < 0; r0 += kRfThreads) {
        const int r = r0 + tid;
        const int j = N - 1 - r;
        float e = 0.f;
        if (r < N - m) {
          const float pj = __ldcg(&p_last[base + j]);
          e = pj * pj;
        }
        // inclusive prefix over the block, in thread order
        float x = e;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (lane == 31) wsum[wp] = x;
        __syncthreads();
        float before = run;
        for (int y = 0; y < wp; ++y) before += wsum[y];
        const bool hit = r < N - m && before + x >= need;
        const unsigned bal = __ballot_sync(0xffffffffu, hit);
        if (lane == 0) red_m[wp][0] = bal ? static_cast<float>(wp * 32 + __ffs(bal) - 1) : -1.f;
        __syncthreads();
        if (tid == 0) {
          int f = -1;
          for (int y = 0; y < kRfWarps && f < 0; ++y)
            if (red_m[y][0] >= 0.f) f = static_cast<int>(red_m[y][0]);
          float tot = run;
          for (int y = 0; y < kRfWarps; ++y) tot += wsum[y];
          sh_e[1] = tot;
          sh_k = f >= 0 ? m + r0 + f + 1 : -1;
        }
        __syncthreads();
        run = sh_e[1];
        found = sh_k;
      }
      if (found < 0 && tid == 0) sh_k = N;   // rounding: keep everything
      __syncthreads();
    }
    if (tid == 0) {
      const int k = sh_k;
      const int c = N - w;
      const int mc = min(sinks, c);
      int b = k - mc - w;
      b = b < 0 ? 0 : (b > max_budget ? max_budget : b);
      budgets[u] = b;
      if (keep_count) keep_count[u] = k;
    }
    __syncthreads();   // shared state is reused by the next unit
  }
}

template <int GP>
cudaError_t launch_rf(const int64_t* tok_off, int U, int G, int w, const void* Q, const void* K,
                      int sinks, float T, int max_budget, float* zbuf, float* p_last,
                      int32_t* budgets, int32_t* keep_count, int nsm, cudaStream_t st) {
  int grid = nsm * 4;
  if (grid > U) grid = U;
  const float scale_log2 = kLog2e / sqrtf(static_cast<float>(kHeadDim));
  refree_kernel<GP><<<grid, kRfThreads, 0, st>>>(
      tok_off, U, G, w, static_cast<const uint16_t*>(Q), static_cast<const uint2*>(K), scale_log2,
      sinks, T, max_budget, zbuf, p_last, budgets, keep_count);
  return cudaGetLastError();
}

}  // namespace

int refree_padded_group(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }

cudaError_t launch_refree(const int64_t* tok_off, int U, int G, int w, const void* Q,
                          const void* K, int sinks, float T, int max_budget, float* zbuf,
                          float* p_last, int32_t* budgets, int32_t* keep_count, int nsm,
                          cudaStream_t st) {
  switch (refree_padded_group(G)) {
    case 1: return launch_rf<1>(tok_off, U, G, w, Q, K, sinks, T, max_budget, zbuf, p_last,
                                budgets, keep_count, nsm, st);
    case 2: return launch_rf<2>(tok_off, U, G, w, Q, K, sinks, T, max_budget, zbuf, p_last,
                                budgets, keep_count, nsm, st);
    case 4: return launch_rf<4>(tok_off, U, G, w, Q, K, sinks, T, max_budget, zbuf, p_last,
                                budgets, keep_count, nsm, st);
    default: return launch_rf<8>(tok_off, U, G, w, Q, K, sinks, T, max_budget, zbuf, p_last,
                                 budgets, keep_count, nsm, st);
  }
}

}  // namespace rkv
