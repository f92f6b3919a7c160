// Adaptive budget from the ReFreeKV review: one row of the attention matrix
// (k = 1, the newest query) stands for all of it, tokens are ranked as the
// first m sinks then newest to oldest, and the kept prefix stops where the
// Frobenius norm of the kept entries reaches (1 - T) of the row's norm.
//
// Work is cut into chunks of kRfChunk tokens of one unit, so every SM streams
// K whatever the unit lengths:
//   plan    per-unit chunk offsets (one block, prefix over the units);
//   logits  per chunk: z_g(j) = q_g . k_j / sqrt(d) (log2 units) of the G
//           newest queries for the chunk's keys into a scratch (GP floats per
//           token), and per head the chunk's (max, sum of 2^(z - max));
//   probs   per chunk: the unit's per-head (M, S) merged from its chunks in
//           chunk order, p(j) = mean_g 2^(z_g(j) - M_g) / S_g from the scratch
//           (mostly L2) to p_last, and the chunk's energy sum p^2;
//   cut     per unit: the row's energy from the chunk energies; the sinks'
//           energy; then chunks from the newest down by their energies until
//           one crosses (1 - T)^2 of the total, and a block-wide scan of that
//           chunk's tokens from its newest down for the stopping token.
// K is read once; the scratch adds 2 GP floats of traffic per token.
//
// The logits are a contraction with G <= 8 columns: a warp runs it on the
// tensor cores with m16n8k16 steps (16 tokens x 8 heads), its A fragments
// loaded straight from K's rows (see rf_logits_kernel), so a token costs a few
// instructions and the kernel stays bound by K's bytes.
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

constexpr int kRfThreads = 256;
constexpr int kRfWarps = kRfThreads / 32;

// Chunk g: its unit (largest u with chunk_off[u] <= g), first token and length.
struct RfChunk {
  int u;
  int64_t base;   // first token of the unit
  int N;          // unit length
  int j0, len;    // the chunk's unit-local tokens j0 .. j0 + len - 1
  int g0, nch;    // the unit's chunks
};
__device__ __forceinline__ RfChunk rf_chunk(const int* chunk_off, const int64_t* tok_off, int U,
                                            int g) {
  int lo = 0, hi = U - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(&chunk_off[mid]) <= g) lo = mid;
    else hi = mid - 1;
  }
  RfChunk c;
  c.u = lo;
  c.base = __ldg(&tok_off[lo]);
  c.N = static_cast<int>(__ldg(&tok_off[lo + 1]) - c.base);
  c.g0 = __ldg(&chunk_off[lo]);
  c.nch = __ldg(&chunk_off[lo + 1]) - c.g0;
  c.j0 = (g - c.g0) * kRfChunk;
  c.len = min(kRfChunk, c.N - c.j0);
  return c;
}

// chunk_off[u] = sum over units before u of ceil(N / kRfChunk) (one block)
__global__ void __launch_bounds__(1024) rf_plan_kernel(const int64_t* __restrict__ tok_off,
                                                       int U, int* __restrict__ chunk_off) {
  __shared__ int wsum[32];
  __shared__ int carry;
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  if (tid == 0) carry = 0;
  __syncthreads();
  for (int u0 = 0; u0 < U; u0 += 1024) {
    const int u = u0 + tid;
    const int n = u < U ? static_cast<int>((tok_off[u + 1] - tok_off[u] + kRfChunk - 1) / kRfChunk)
                        : 0;
    int x = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) wsum[wp] = x;
    __syncthreads();
    if (wp == 0) {
      int s = wsum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      wsum[lane] = s;   // inclusive over warps
    }
    __syncthreads();
    const int excl = carry + (wp > 0 ? wsum[wp - 1] : 0) + x - n;
    if (u < U) chunk_off[u] = excl;
    __syncthreads();
    if (tid == 1023) carry = excl + n;
    __syncthreads();
  }
  if (tid == 0) chunk_off[U] = carry;
}

// D (16 x 8, fp32) = A (16 x 16, bf16, row-major) . B (16 x 8, bf16) + C, one warp.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4],
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Logits on the tensor cores: per 16 tokens, D[token][head] = K (16 x 128) .
// Qlast^T (128 x 8 heads, zero past G) as eight m16n8k16 steps.  The head
// dimension is visited in a permuted order (any order gives the same dot
// product): k-step 2s' + h of lane (gid, tid4) takes dimensions
// 32 s' + 8 tid4 + 4 h + {0, 1, 2, 3} for its A columns {2 tid4, 2 tid4 + 1,
// 2 tid4 + 8, 2 tid4 + 9} and B rows alike, so one 16-byte load of a row gives
// a lane its A fragments of two k-steps.  Lane (gid, tid4) ends with the
// logits of tokens gid and gid + 8, heads 2 tid4 and 2 tid4 + 1.
template <int GP>
__global__ void __launch_bounds__(kRfThreads, 4)
    rf_logits_kernel(const int64_t* __restrict__ tok_off, const int* __restrict__ chunk_off,
                     int U, int nchunks, int G, int w, const uint4* __restrict__ Q,
                     const uint4* __restrict__ K, float scale_log2, float* __restrict__ zbuf,
                     float2* __restrict__ cstat) {
  __shared__ float2 red[kRfWarps][32][2];
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const int gid = lane >> 2, t4 = lane & 3;
  const int h0 = 2 * t4;   // this lane's heads h0, h0 + 1
  for (int g = blockIdx.x; g < nchunks; g += gridDim.x) {
    const RfChunk ch = rf_chunk(chunk_off, tok_off, U, g);
    // B fragments: the newest query of head gid (zero past G), four 16-byte
    // pieces covering the eight k-steps
    uint4 qb[4];
#pragma unroll
    for (int sp = 0; sp < 4; ++sp) {
      qb[sp] = gid < G ? __ldg(&Q[((static_cast<int64_t>(ch.u) * G + gid) * w + (w - 1)) * 16 +
                                  4 * sp + t4])
                       : make_uint4(0u, 0u, 0u, 0u);
    }
    const int jend = ch.j0 + ch.len;
    float* zu = zbuf + ch.base * GP;   // logit of (token j, head h) at zu[j * GP + h]
    float m0 = -INFINITY, s0 = 0.f, m1 = -INFINITY, s1 = 0.f;   // heads h0, h0 + 1
    for (int j0 = ch.j0 + 16 * wp; j0 < jend; j0 += 16 * kRfWarps) {
      const int ja = j0 + gid, jb = ja + 8;   // this lane's two tokens
      uint4 ka[4], kb[4];
#pragma unroll
      for (int sp = 0; sp < 4; ++sp) {
        ka[sp] = ja < jend ? __ldcs(&K[(ch.base + ja) * 16 + 4 * sp + t4]) : make_uint4(0u, 0u, 0u, 0u);
        kb[sp] = jb < jend ? __ldcs(&K[(ch.base + jb) * 16 + 4 * sp + t4]) : make_uint4(0u, 0u, 0u, 0u);
      }
      // the warp's next rows into L2 while these are multiplied (lane t4 = 0
      // of each row: the row's two 128-byte lines)
      if (t4 == 0) {
        const int na = ja + 16 * kRfWarps, nb = jb + 16 * kRfWarps;
        if (na < jend) {
          prefetch_l2(&K[(ch.base + na) * 16]);
          prefetch_l2(&K[(ch.base + na) * 16 + 8]);
        }
        if (nb < jend) {
          prefetch_l2(&K[(ch.base + nb) * 16]);
          prefetch_l2(&K[(ch.base + nb) * 16 + 8]);
        }
      }
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int sp = 0; sp < 4; ++sp) {
        const uint32_t a0[4] = {ka[sp].x, kb[sp].x, ka[sp].y, kb[sp].y};
        mma_16816(d, a0, qb[sp].x, qb[sp].y);
        const uint32_t a1[4] = {ka[sp].z, kb[sp].z, ka[sp].w, kb[sp].w};
        mma_16816(d, a1, qb[sp].z, qb[sp].w);
      }
      // d: (token ja, heads h0, h0+1), (token jb, heads h0, h0+1)
      const float za0 = d[0] * scale_log2, za1 = d[1] * scale_log2;
      const float zb0 = d[2] * scale_log2, zb1 = d[3] * scale_log2;
      if (h0 < GP) {
        if constexpr (GP == 1) {
          if (ja < jend) zu[ja] = za0;
          if (jb < jend) zu[jb] = zb0;
        } else {
          if (ja < jend) __stcg(reinterpret_cast<float2*>(&zu[static_cast<int64_t>(ja) * GP + h0]),
                                make_float2(za0, za1));
          if (jb < jend) __stcg(reinterpret_cast<float2*>(&zu[static_cast<int64_t>(jb) * GP + h0]),
                                make_float2(zb0, zb1));
        }
      }
      // running (max, sum of 2^(z - max)) of the lane's two heads
      const float xa0 = ja < jend ? za0 : -INFINITY, xb0 = jb < jend ? zb0 : -INFINITY;
      const float xa1 = ja < jend ? za1 : -INFINITY, xb1 = jb < jend ? zb1 : -INFINITY;
      const float n0 = fmaxf(m0, fmaxf(xa0, xb0)), n1 = fmaxf(m1, fmaxf(xa1, xb1));
      if (n0 > -INFINITY) {
        s0 = s0 * ex2(m0 - n0) + ex2(xa0 - n0) + ex2(xb0 - n0);
        m0 = n0;
      }
      if (n1 > -INFINITY) {
        s1 = s1 * ex2(m1 - n1) + ex2(xa1 - n1) + ex2(xb1 - n1);
        m1 = n1;
      }
    }
    red[wp][lane][0] = make_float2(m0, s0);
    red[wp][lane][1] = make_float2(m1, s1);
    __syncthreads();
    if (tid < GP) {   // head tid: lanes with h0 = tid & ~1, entry tid & 1
      const int t = tid >> 1, e = tid & 1;
      float M = -INFINITY;
      for (int x = 0; x < kRfWarps; ++x)
        for (int gg = 0; gg < 8; ++gg) M = fmaxf(M, red[x][4 * gg + t][e].x);
      float S = 0.f;
      if (tid < G) {
        for (int x = 0; x < kRfWarps; ++x)
          for (int gg = 0; gg < 8; ++gg) {
            const float2 v = red[x][4 * gg + t][e];
            if (v.y > 0.f) S += v.y * ex2(v.x - M);
          }
      }
      cstat[static_cast<int64_t>(g) * GP + tid] = make_float2(M, S);
    }
    __syncthreads();   // red is reused by the next chunk
  }
}

template <int GP>
__global__ void __launch_bounds__(kRfThreads)
    rf_probs_kernel(const int64_t* __restrict__ tok_off, const int* __restrict__ chunk_off, int U,
                    int nchunks, int G, const float* __restrict__ zbuf,
                    const float2* __restrict__ cstat, float* __restrict__ p_last,
                    float* __restrict__ cenergy) {
  __shared__ float fin_m[GP], fin_is[GP];
  __shared__ float wsum[kRfWarps];
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const float invG = 1.f / static_cast<float>(G);
  for (int g = blockIdx.x; g < nchunks; g += gridDim.x) {
    const RfChunk ch = rf_chunk(chunk_off, tok_off, U, g);
    if (wp < GP) {
      // head wp: the unit's chunk statistics, lane-strided, then a warp merge
      float m = -INFINITY, s = 0.f;
      for (int x = lane; x < ch.nch; x += 32) {
        const float2 cs = __ldcg(&cstat[static_cast<int64_t>(ch.g0 + x) * GP + wp]);
        if (cs.y > 0.f) {
          const float mn = fmaxf(m, cs.x);
          s = s * ex2(m - mn) + cs.y * ex2(cs.x - mn);
          m = mn;
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) {
        const float om = __shfl_xor_sync(0xffffffffu, m, o);
        const float os = __shfl_xor_sync(0xffffffffu, s, o);
        const float mn = fmaxf(m, om);
        const float a = s > 0.f ? s * ex2(m - mn) : 0.f;
        const float b = os > 0.f ? os * ex2(om - mn) : 0.f;
        m = mn;
        s = a + b;
      }
      if (lane == 0) {
        fin_m[wp] = m;
        fin_is[wp] = s > 0.f ? 1.f / s : 0.f;
      }
    }
    __syncthreads();
    float Mh[GP], iSh[GP];
#pragma unroll
    for (int h = 0; h < GP; ++h) {
      // padding heads: 2^(z - inf) = 0, times a zero weight
      Mh[h] = h < G ? fin_m[h] : INFINITY;
      iSh[h] = h < G ? fin_is[h] * invG : 0.f;   // the mean over heads folded in
    }
    const int jend = ch.j0 + ch.len;
    const float* zu = zbuf + ch.base * GP;
    float esum = 0.f;
    // thread = token, its GP logits in one or two vector loads; four tokens'
    // loads in flight per thread
    constexpr int kU = 4;
    for (int jb = ch.j0 + tid; jb < jend; jb += kU * kRfThreads) {
      float z[kU][GP];
#pragma unroll
      for (int x = 0; x < kU; ++x) {
        const int j = jb + x * kRfThreads;
        const float* zp = zu + static_cast<int64_t>(j) * GP;
        if (j < jend) {
          if constexpr (GP == 8) {
            const float4 v0 = __ldcg(reinterpret_cast<const float4*>(zp));
            const float4 v1 = __ldcg(reinterpret_cast<const float4*>(zp) + 1);
            z[x][0] = v0.x; z[x][1] = v0.y; z[x][2] = v0.z; z[x][3] = v0.w;
            z[x][4] = v1.x; z[x][5] = v1.y; z[x][6] = v1.z; z[x][7] = v1.w;
          } else if constexpr (GP == 4) {
            const float4 v0 = __ldcg(reinterpret_cast<const float4*>(zp));
            z[x][0] = v0.x; z[x][1] = v0.y; z[x][2] = v0.z; z[x][3] = v0.w;
          } else if constexpr (GP == 2) {
            const float2 v0 = __ldcg(reinterpret_cast<const float2*>(zp));
            z[x][0] = v0.x; z[x][1] = v0.y;
          } else {
            z[x][0] = __ldcg(zp);
          }
        } else {
#pragma unroll
          for (int h = 0; h < GP; ++h) z[x][h] = -INFINITY;
        }
      }
#pragma unroll
      for (int x = 0; x < kU; ++x) {
        const int j = jb + x * kRfThreads;
        float pj = 0.f;
#pragma unroll
        for (int h = 0; h < GP; ++h) pj = fmaf(ex2(z[x][h] - Mh[h]), iSh[h], pj);
        if (j < jend) {
          p_last[ch.base + j] = pj;
          esum = fmaf(pj, pj, esum);
        }
      }
    }
    esum = warp_reduce_sum(esum);
    if (lane == 0) wsum[wp] = esum;
    __syncthreads();
    if (tid == 0) {
      float e = 0.f;
      for (int x = 0; x < kRfWarps; ++x) e += wsum[x];
      cenergy[g] = e;
    }
    __syncthreads();   // fin_* and wsum are reused by the next chunk
  }
}

// One CTA per unit: the stopping point of the ranking (sinks, newest .. oldest).
__global__ void __launch_bounds__(kRfThreads)
    rf_cut_kernel(const int64_t* __restrict__ tok_off, const int* __restrict__ chunk_off, int w,
                  int sinks, float T, int max_budget, const float* __restrict__ p_last,
                  const float* __restrict__ cenergy, int32_t* __restrict__ budgets,
                  int32_t* __restrict__ keep_count) {
  __shared__ float wsum[kRfWarps];
  __shared__ int whit[kRfWarps];
  __shared__ float sh_acc, sh_need;
  __shared__ int sh_k;
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  const int u = blockIdx.x;
  const int64_t base = tok_off[u];
  const int N = static_cast<int>(tok_off[u + 1] - base);
  const int g0 = chunk_off[u], nch = chunk_off[u + 1] - g0;
  const float* p = p_last + base;
  const int m = min(sinks, N);
  if (tid == 0) {
    // the row's energy from the chunk energies, in chunk order
    float E = 0.f;
    for (int x = 0; x < nch; ++x) E += __ldcg(&cenergy[g0 + x]);
    const float need = (1.f - T) * (1.f - T) * E;
    float acc = 0.f;
    int k = -1;
    for (int j = 0; j < m; ++j) {
      const float pj = __ldcg(&p[j]);
      acc = fmaf(pj, pj, acc);
      if (acc >= need) {
        k = j + 1;
        break;
      }
    }
    sh_need = need;
    sh_acc = acc;
    sh_k = k;
  }
  __syncthreads();
  int k = sh_k;
  const float need = sh_need;
  // chunks from the newest down; a chunk's suffix tokens are those >= m
  for (int x = nch - 1; x >= 0 && k < 0; --x) {
    const int cs = x * kRfChunk, ce = min(N, cs + kRfChunk);
    const int lo = max(cs, m);   // the chunk's tokens lo .. ce - 1 are ranked
    if (lo >= ce) break;         // only sinks left
    bool scan = true;
    if (cs >= m) {   // whole chunk ranked: skip it if its energy does not cross
      const float ec = __ldcg(&cenergy[g0 + x]);
      if (sh_acc + ec < need) {
        __syncthreads();
        if (tid == 0) sh_acc += ec;
        __syncthreads();
        scan = false;
      }
    }
    if (!scan) continue;
    // block scan of the chunk's ranked tokens from ce - 1 down, 256 per round
    for (int r0 = 0; r0 < ce - lo && k < 0; r0 += kRfThreads) {
      const int r = r0 + tid;
      const int j = ce - 1 - r;
      float e = 0.f;
      if (j >= lo) {
        const float pj = __ldcg(&p[j]);
        e = pj * pj;
      }
      float xin = e;   // inclusive prefix in thread order
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, xin, o);
        if (lane >= o) xin += y;
      }
      if (lane == 31) wsum[wp] = xin;
      __syncthreads();
      float before = sh_acc;
      for (int y = 0; y < wp; ++y) before += wsum[y];
      const bool hit = j >= lo && before + xin >= need;
      const unsigned bal = __ballot_sync(0xffffffffu, hit);
      if (lane == 0) whit[wp] = bal ? wp * 32 + __ffs(bal) - 1 : -1;
      __syncthreads();
      if (tid == 0) {
        int f = -1;
        for (int y = 0; y < kRfWarps && f < 0; ++y) f = whit[y];
        float tot = sh_acc;
        for (int y = 0; y < kRfWarps; ++y) tot += wsum[y];
        sh_acc = tot;
        if (f >= 0) sh_k = m + (N - (ce - 1 - (r0 + f)));   // sinks + suffix from that token
      }
      __syncthreads();
      k = sh_k;
    }
  }
  if (tid == 0) {
    if (k < 0) k = N;   // rounding: keep everything
    const int c = N - w;
    const int mc = min(sinks, c);
    int b = k - mc - w;
    b = b < 0 ? 0 : (b > max_budget ? max_budget : b);
    budgets[u] = b;
    if (keep_count) keep_count[u] = k;
  }
}

template <int GP>
cudaError_t launch_rf(const RefreeArgs& a, cudaStream_t st) {
  rf_plan_kernel<<<1, 1024, 0, st>>>(a.tok_off, a.U, a.chunk_off);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess || a.nchunks == 0) return err;
  const int64_t cap = static_cast<int64_t>(a.nsm) * 8;
  const int grid = static_cast<int>(a.nchunks < cap ? a.nchunks : cap);
  const float scale_log2 = kLog2e / sqrtf(static_cast<float>(kHeadDim));
  rf_logits_kernel<GP><<<grid, kRfThreads, 0, st>>>(
      a.tok_off, a.chunk_off, a.U, a.nchunks, a.G, a.w, static_cast<const uint4*>(a.Q),
      static_cast<const uint4*>(a.K), scale_log2, a.zbuf, a.cstat);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  rf_probs_kernel<GP><<<grid, kRfThreads, 0, st>>>(a.tok_off, a.chunk_off, a.U, a.nchunks, a.G,
                                                   a.zbuf, a.cstat, a.p_last, a.cenergy);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  rf_cut_kernel<<<a.U, kRfThreads, 0, st>>>(a.tok_off, a.chunk_off, a.w, a.sinks, a.T,
                                            a.max_budget, a.p_last, a.cenergy, a.budgets,
                                            a.keep_count);
  return cudaGetLastError();
}

}  // namespace

int refree_padded_group(int G) { return G <= 1 ? 1 : G <= 2 ? 2 : G <= 4 ? 4 : 8; }

int64_t refree_max_chunks(int64_t max_tokens, int max_units) {
  return max_tokens / kRfChunk + max_units;
}

cudaError_t launch_refree(const RefreeArgs& a, cudaStream_t st) {
  switch (refree_padded_group(a.G)) {
    case 1: return launch_rf<1>(a, st);
    case 2: return launch_rf<2>(a, st);
    case 4: return launch_rf<4>(a, st);
    default: return launch_rf<8>(a, st);
  }
}

}  // namespace rkv
