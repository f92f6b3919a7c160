// Score kernel: importance (R-KV 重要性打分) and, in closed-form mode, the
// redundancy row mean (R-KV 冗余打分) for every unit, with K read from HBM once.
//
// One thread-block cluster of `cs` CTAs owns one unit at a time; CTA `rank`
// owns the contiguous token chunk [rank*L, rank*L + L) (L a multiple of 128,
// at most 512 / RP tiles).  Per unit:
//
//   pass 1 (K tiles streamed by TMA; in closed form left in L2 for pass 2):
//     - logits z = K_tile . Q^T on tcgen05 (M = 128 tokens, N = RP padded
//       query rows, fp32 accumulator).  Tile k's logits stay in TMEM columns
//       [k*RP, (k+1)*RP) for the whole unit, so pass 2 needs no second MMA;
//     - per-thread online softmax statistics (running max, sum of
//       2^(y - max), y = z * log2(e) / sqrt(d)) with a lazy max;
//     - key norms on CUDA cores -> rho = 1/||k||; (closed form) U = sum rho_j k_j.
//   cluster exchange #1: every CTA pushes its (max, sum) per query row [and
//     partial U] into every CTA's inbox with st.async (completing bytes on the
//     receiver's mbarrier); each CTA merges the inbox in rank order, so every
//     CTA holds identical values.
//   pass 2:
//     - abar_j = (1/(G w)) sum_rows 2^(y - M_row) / L_row from the TMEM logits;
//     - (closed form) K tiles again, most recent first (likely still in L2):
//       m_j = (rho_j k_j . U - khat_j . khat_j) / (N - 1) on CUDA cores.
//   cluster exchange #2: sums of abar and of exp(m) over the candidates.
//   write a = abar / sum, r = exp(m) / sum (window rows get 0).
//
// Warp roles (512 threads): warp 0 TMA producer, warp 1 MMA issuer and TMEM
// owner, warps 4-11 softmax (thread = token row of a tile; TMEM lane quarter =
// warp % 4; warps 4-7 take the first half of the query rows, 8-11 the second),
// warps 12-15 norms and U (thread = token row).
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

constexpr float kNegBig = -1e30f;  // initial running max (finite: no inf - inf)
constexpr float kLazy = 8.f;       // log2 headroom before the running max moves

#ifdef RKV_TRACE
// Optional phase trace (build with -DRKV_TRACE): globaltimer stamps per CTA for
// the first kTraceUnits units it processes, kTraceSlots stamps each.
constexpr int kTraceCtas = 256, kTraceUnits = 8, kTraceSlots = 8;
__device__ unsigned long long g_score_trace[kTraceCtas * kTraceUnits * kTraceSlots];
#define RKV_STAMP(it, slot)                                                              \
  do {                                                                                   \
    if ((it) < kTraceUnits && blockIdx.x < kTraceCtas)                                   \
      g_score_trace[(blockIdx.x * kTraceUnits + (it)) * kTraceSlots + (slot)] =          \
          globaltimer_ns();                                                              \
  } while (0)
#else
#define RKV_STAMP(it, slot) do { } while (0)
#endif

struct UnitSched {
  int64_t base;  // first row of the unit in K
  int n;         // N
  int c;         // N - w
  int start;     // first token of this CTA's chunk
  int len;       // tokens in the chunk
  int nt;        // tiles in the chunk
};

__device__ __forceinline__ UnitSched unit_sched(const ScoreParams& p, int u, int rank) {
  UnitSched s;
  s.base = p.tok_off[u];
  s.n = static_cast<int>(p.tok_off[u + 1] - s.base);
  s.c = s.n - p.w;
  int per = (s.n + p.cs - 1) / p.cs;
  per = ((per + kTile - 1) / kTile) * kTile;
  s.start = rank * per;
  s.len = max(0, min(per, s.n - s.start));
  s.nt = (s.len + kTile - 1) / kTile;
  return s;
}

constexpr int kConsumers = 384;   // softmax + norm threads

template <int RH>
__device__ __forceinline__ void tmem_ld_rows(uint32_t taddr, uint32_t (&v)[RH]) {
  if constexpr (RH == 8) tmem_ld8(taddr, v);
  else tmem_ld16(taddr, v);
}

// Merge two (max, sum) softmax statistics in the log2 domain.
__device__ __forceinline__ void merge_stat(float& m, float& s, float om, float os) {
  const float M = fmaxf(m, om);
  s = s * ex2(m - M) + os * ex2(om - M);
  m = M;
}

// Push this CTA's n4 16-byte chunks at `src` into slot `rank` of the inbox
// (same offset) of every CTA of the cluster with st.async; each store
// completes its bytes on the receiving CTA's barrier `bar`, which expects
// cs * n4 * 16 bytes per round.  No fence is needed: the receiver sees the
// data once its barrier phase completes.
__device__ __forceinline__ void cluster_push(const float* src, float* inbox, int n4, int cs,
                                             int rank, uint64_t* bar, int ctid) {
  const uint32_t inbox_base = smem_u32(inbox) + static_cast<uint32_t>(rank * n4 * 16);
  const uint32_t bar_local = smem_u32(bar);
  for (int e = ctid; e < n4 * cs; e += kConsumers) {
    const int dst = e / n4, ch = e - dst * n4;
    const float4 v = reinterpret_cast<const float4*>(src)[ch];
    st_async_v4(mapa(inbox_base + ch * 16, dst), mapa(bar_local, dst), v);
  }
}

// Load the 16 swizzled 16-byte chunks of K-tile row `row` (128 bf16).
__device__ __forceinline__ void load_row(uint32_t sb, int row, uint4 (&xs)[16]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      const uint32_t ad = sb + h * (kTileBytes / 2) + row * 128 + ((cc ^ (row & 7)) << 4);
      asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                   : "=r"(xs[h * 8 + cc].x), "=r"(xs[h * 8 + cc].y), "=r"(xs[h * 8 + cc].z),
                     "=r"(xs[h * 8 + cc].w)
                   : "r"(ad));
    }
  }
}

template <int RP, bool CLOSED>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                 const ScoreParams p) {
  constexpr int XB = 2 * RP + (CLOSED ? 128 : 0);   // round-1 partial floats per CTA
  constexpr int RH = RP / 2;                         // query rows per softmax warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const int NS = p.nstages;
  const ScoreLayout L = score_layout(RP, CLOSED, NS);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const int cid = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(cluster_count_x());
  const int cs = p.cs;

  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* empty = full + NS;
  uint64_t* tready = empty + NS;   // [32] logits of tile k are in TMEM
  uint64_t* tfree = tready + 32;   // softmax warps are done with the unit's TMEM
  uint64_t* qfull = tfree + 1;
  uint64_t* qempty = qfull + 2;
  uint64_t* redbar = qempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L.slot);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + L.flags);
  float* rsum = reinterpret_cast<float*>(sm + L.rsum);
  float* xbuf = reinterpret_cast<float*>(sm + L.xbuf);
  float* gath = reinterpret_cast<float*>(sm + L.gath);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);  // MMA thread + 4 norm warps
    }
    for (int k = 0; k < 32; ++k) mbar_init(&tready[k], 1);
    mbar_init(tfree, 8);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&qfull[b], 1);
      mbar_init(&qempty[b], 1);
      mbar_init(&redbar[b], 1);   // local arrive.expect_tx; bytes from every CTA
    }
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc<1>(tmem_slot, kTmemColsTotal);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&qmap);
      const uint64_t keep = policy_evict_normal(), drop = policy_evict_first();
      int stage = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int u = cid; u < p.num_units; u += ncl, ++it) {
        const UnitSched s = unit_sched(p, u, rank);
        const int qb = it & 1;
        if (mbar_wait(&qempty[qb], ((it >> 1) & 1) ^ 1, abort, p.status)) {
          uint8_t* qd = sm + L.q + qb * RP * 256;
          mbar_arrive_expect_tx(&qfull[qb], RP * 256);
          tma_load_2d(qd, &qmap, &qfull[qb], 0, u * p.R, keep);
          tma_load_2d(qd + RP * 128, &qmap, &qfull[qb], 64, u * p.R, keep);
        }
        for (int pass = 0; pass < (CLOSED ? 2 : 1); ++pass) {
          for (int kk = 0; kk < s.nt; ++kk) {
            const int k = pass ? s.nt - 1 - kk : kk;
            if (mbar_wait(&empty[stage], ph ^ 1, abort, p.status)) {
              uint8_t* dst = sm + L.stages + stage * kTileBytes;
              const int y = static_cast<int>(s.base + s.start + kTile * k);
              // read once (GEMM form), or kept for the pass-2 re-read (closed form)
              const uint64_t pol = (CLOSED && pass == 0) ? keep : drop;
              mbar_arrive_expect_tx(&full[stage], kTileBytes);
              tma_load_2d(dst, &kmap, &full[stage], 0, y, pol);
              tma_load_2d(dst + kTileBytes / 2, &kmap, &full[stage], 64, y, pol);
            }
            if (++stage == NS) { stage = 0; ph ^= 1; }
          }
          if (pass == 0) RKV_STAMP(it, 7);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, RP);
      int stage = 0;
      uint32_t ph = 0;
      int it = 0;
      for (int u = cid; u < p.num_units; u += ncl, ++it) {
        const UnitSched s = unit_sched(p, u, rank);
        const int qb = it & 1;
        bool ok = mbar_wait(&qfull[qb], (it >> 1) & 1, abort, p.status);
        // the previous unit's logits must have been read out of TMEM
        ok = mbar_wait(tfree, (it & 1) ^ 1, abort, p.status) && ok;
        const uint32_t qaddr = smem_u32(sm + L.q + qb * RP * 256);
        for (int k = 0; k < s.nt; ++k) {
          const bool go = mbar_wait(&full[stage], ph, abort, p.status) && ok;
          tc_fence_after();
          if (go) {
            const uint32_t kaddr = smem_u32(sm + L.stages + stage * kTileBytes);
            const uint32_t d = tmem + k * RP;
#pragma unroll
            for (int kq = 0; kq < 8; ++kq) {
              const uint32_t ko = (kq >> 2) * (kTileBytes / 2) + (kq & 3) * 32;
              const uint32_t qo = (kq >> 2) * (RP * 128) + (kq & 3) * 32;
              mma_bf16<1>(d, desc_kmajor_sw128(kaddr + ko), desc_kmajor_sw128(qaddr + qo),
                          idesc, kq > 0);
            }
            mma_commit(&empty[stage]);
            mma_commit(&tready[k]);
          } else {
            mbar_arrive(&empty[stage]);
          }
          if (++stage == NS) { stage = 0; ph ^= 1; }
        }
        if (ok) mma_commit(&qempty[qb]);
        else mbar_arrive(&qempty[qb]);
        if constexpr (CLOSED) {
          // pass-2 tiles feed only the norm warps: keep the ring's arrival count
          for (int k = 0; k < s.nt; ++k) {
            mbar_wait(&full[stage], ph, abort, p.status);
            mbar_arrive(&empty[stage]);
            if (++stage == NS) { stage = 0; ph ^= 1; }
          }
        }
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ consumers
    const int ctid = threadIdx.x - 128;      // 0..383
    const bool is_soft = warp < 12;          // warps 4-11: softmax
    const int q4 = warp & 3;                 // TMEM lane quarter
    const int row = q4 * 32 + lane;          // token row of the tile
    const int r0 = ((warp - 4) >> 2) * RH;   // first query row of a softmax warp
    float* abar_s = reinterpret_cast<float*>(sm + L.abar);
    float* marr = reinterpret_cast<float*>(sm + L.marr);
    float* rhoc = reinterpret_cast<float*>(sm + L.rhoc);
    float* rhot = reinterpret_cast<float*>(sm + L.rhot);
    float* ufin = reinterpret_cast<float*>(sm + L.ufin);
    float* mrow = reinterpret_cast<float*>(sm + L.mrow);
    float* invl = reinterpret_cast<float*>(sm + L.invl);
    float* red1 = reinterpret_cast<float*>(sm + L.red1);
    float* red2 = reinterpret_cast<float*>(sm + L.red2);
    const float invR = 1.f / static_cast<float>(p.R);
    // bit r set for real query rows; row_t[r] = window step t of query row
    // r = g*w + t (read only for tiles that reach the window)
    const uint32_t rmask = p.R >= 32 ? 0xffffffffu : ((1u << p.R) - 1u);
    const int* row_t = reinterpret_cast<const int*>(sm + L.rowt);
    if (ctid < 32) reinterpret_cast<int*>(sm + L.rowt)[ctid] = ctid % p.w;
    named_bar_sync(1, kConsumers);

    int stage = 0, ntile1 = 0;
    uint32_t ph = 0;
    uint32_t tph = 0;  // phase bit of tready[k]
    int it = 0;
    for (int u = cid; u < p.num_units; u += ncl, ++it) {
      const UnitSched s = unit_sched(p, u, rank);
      const int N = s.n, c = s.c;
      float st_m[RH], st_s[RH];  // pass 1: running stats; pass 2: row max and 1/sum
#pragma unroll
      for (int r = 0; r < RH; ++r) { st_m[r] = kNegBig; st_s[r] = 0.f; }
      for (int i = ctid; i < s.len; i += kConsumers) abar_s[i] = 0.f;
      float U4[4] = {0.f, 0.f, 0.f, 0.f};
      float part = 0.f;  // pass 2: sum of abar (softmax) or of exp(m) (norm warps)
      if (ctid == 0) RKV_STAMP(it, 0);

      // ================================================= pass 1
      for (int k = 0; k < s.nt; ++k) {
        const int t0 = s.start + kTile * k;
        const int j = t0 + row;
        if (is_soft) {
          mbar_wait(&tready[k], (tph >> k) & 1u, abort, p.status);
          tph ^= 1u << k;
          __syncwarp();
          tc_fence_after();
          uint32_t v[RH];
          tmem_ld_rows<RH>(tmem + (static_cast<uint32_t>(q4 * 32) << 16) + k * RP + r0, v);
          tmem_wait_ld();
          // y = log2-scaled logit, -inf where masked (padding row, beyond N,
          // causal); only a tile that reaches the window needs the causal limit
          float y[RH];
          if (t0 + kTile <= c) {
#pragma unroll
            for (int r = 0; r < RH; ++r)
              y[r] = ((rmask >> (r0 + r)) & 1u) ? __uint_as_float(v[r]) * p.scale_log2 : -INFINITY;
          } else {
#pragma unroll
            for (int r = 0; r < RH; ++r) {
              const bool vis = ((rmask >> (r0 + r)) & 1u) && j < N && j <= c + row_t[r0 + r];
              y[r] = vis ? __uint_as_float(v[r]) * p.scale_log2 : -INFINITY;
            }
          }
          // Lazy running max: the reference max only moves when a logit exceeds
          // it by more than 2^kLazy, so terms 2^(y - max) stay below 256 and the
          // common case is branch-free.
          bool need = false;
#pragma unroll
          for (int r = 0; r < RH; ++r) need |= y[r] > st_m[r] + kLazy;
          if (__any_sync(0xffffffffu, need)) {
#pragma unroll
            for (int r = 0; r < RH; ++r) {
              if (y[r] > st_m[r]) {
                st_s[r] = st_s[r] * ex2(st_m[r] - y[r]) + 1.f;
                st_m[r] = y[r];
              } else {
                st_s[r] += ex2(y[r] - st_m[r]);
              }
            }
          } else {
#pragma unroll
            for (int r = 0; r < RH; ++r) st_s[r] += ex2(y[r] - st_m[r]);
          }
        } else {
          // norm warps: ||k|| of row `row`, rho, (closed form) U accumulation
          mbar_wait(&full[stage], ph, abort, p.status);
          __syncwarp();
          const uint32_t sb = smem_u32(sm + L.stages + stage * kTileBytes);
          uint4 xs[16];
          load_row(sb, row, xs);
          float nq[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int k8 = 0; k8 < 16; ++k8) {
            float f;
            f = bf_lo(xs[k8].x); nq[0] = fmaf(f, f, nq[0]);
            f = bf_hi(xs[k8].x); nq[1] = fmaf(f, f, nq[1]);
            f = bf_lo(xs[k8].y); nq[2] = fmaf(f, f, nq[2]);
            f = bf_hi(xs[k8].y); nq[3] = fmaf(f, f, nq[3]);
            f = bf_lo(xs[k8].z); nq[4] = fmaf(f, f, nq[4]);
            f = bf_hi(xs[k8].z); nq[5] = fmaf(f, f, nq[5]);
            f = bf_lo(xs[k8].w); nq[6] = fmaf(f, f, nq[6]);
            f = bf_hi(xs[k8].w); nq[7] = fmaf(f, f, nq[7]);
          }
          const float n2 =
              ((nq[0] + nq[1]) + (nq[2] + nq[3])) + ((nq[4] + nq[5]) + (nq[6] + nq[7]));
          const float rho = (j < N && n2 > 0.f) ? 1.f / sqrtf(n2) : 0.f;
          if constexpr (CLOSED) {
            rhoc[j - s.start] = rho;
            float* rt = rhot + (ntile1 & 1) * 128;
            rt[row] = rho;
            named_bar_sync(2, 128);
            // U += rho_row * k_row over this warp's 32 rows, dims 4*lane .. 4*lane+3
            const int hh = lane >> 4;
            const uint32_t cidx = (lane & 15) >> 1;
            const uint32_t sub = (lane & 1) * 8;
            float U8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
            for (int rr = 0; rr < 32; ++rr) {
              const int rw = q4 * 32 + rr;
              const float rr_rho = rt[rw];
              const uint32_t ad =
                  sb + hh * (kTileBytes / 2) + rw * 128 + ((cidx ^ (rw & 7)) << 4) + sub;
              uint32_t x0, x1;
              asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(x0), "=r"(x1) : "r"(ad));
              float* Ua = U8 + (rr & 1) * 4;
              Ua[0] = fmaf(rr_rho, bf_lo(x0), Ua[0]);
              Ua[1] = fmaf(rr_rho, bf_hi(x0), Ua[1]);
              Ua[2] = fmaf(rr_rho, bf_lo(x1), Ua[2]);
              Ua[3] = fmaf(rr_rho, bf_hi(x1), Ua[3]);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) U4[i] += U8[i] + U8[4 + i];
          } else {
            if (j < N && p.rho_out) p.rho_out[p.rho_off[u] + j] = rho;
          }
          ++ntile1;
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[stage]);
          if (++stage == NS) { stage = 0; ph ^= 1; }
        }
      }

      // ================================================= exchange 1
      if (ctid == 0) RKV_STAMP(it, 1);
      if (ctid == 256) RKV_STAMP(it, 2);
      if (is_soft) {
#pragma unroll
        for (int r = 0; r < RH; ++r) {
#pragma unroll
          for (int o = 16; o; o >>= 1) {
            const float om = __shfl_xor_sync(0xffffffffu, st_m[r], o);
            const float os = __shfl_xor_sync(0xffffffffu, st_s[r], o);
            merge_stat(st_m[r], st_s[r], om, os);
          }
        }
        if (lane == 0) {
#pragma unroll
          for (int r = 0; r < RH; ++r) {
            red1[(q4 * RP + r0 + r) * 2 + 0] = st_m[r];
            red1[(q4 * RP + r0 + r) * 2 + 1] = st_s[r];
          }
        }
      } else if (CLOSED) {
#pragma unroll
        for (int i = 0; i < 4; ++i) red2[q4 * 128 + lane * 4 + i] = U4[i];
      }
      named_bar_sync(1, kConsumers);
      float* xa = xbuf;  // this CTA's round-1 partials
      if (ctid < RP) {
        float m = kNegBig, sacc = 0.f;
        for (int q = 0; q < 4; ++q)
          merge_stat(m, sacc, red1[(q * RP + ctid) * 2], red1[(q * RP + ctid) * 2 + 1]);
        xa[2 * ctid] = m;
        xa[2 * ctid + 1] = sacc;
      }
      if (CLOSED && ctid >= 256) {
        const int e = ctid - 256;
        xa[2 * RP + e] = red2[e] + red2[128 + e] + red2[256 + e] + red2[384 + e];
      }
      if (ctid == 0) mbar_arrive_expect_tx(&redbar[0], cs * XB * 4);
      named_bar_sync(1, kConsumers);
      cluster_push(xa, gath, XB / 4, cs, rank, &redbar[0], ctid);
      mbar_wait<true>(&redbar[0], it & 1, abort, p.status);
      __syncwarp();
      if (ctid < RP) {
        float m = kNegBig;
        for (int rr = 0; rr < cs; ++rr) m = fmaxf(m, gath[rr * XB + 2 * ctid]);
        float sacc = 0.f;
        for (int rr = 0; rr < cs; ++rr)
          sacc = fmaf(gath[rr * XB + 2 * ctid + 1], ex2(gath[rr * XB + 2 * ctid] - m), sacc);
        mrow[ctid] = m;
        invl[ctid] = sacc > 0.f ? 1.f / sacc : 0.f;
      }
      if (CLOSED && ctid >= 256) {
        const int e = ctid - 256;
        float acc = 0.f;
        for (int rr = 0; rr < cs; ++rr) acc += gath[rr * XB + 2 * RP + e];
        ufin[e] = acc;
      }
      named_bar_sync(1, kConsumers);
      if (is_soft) {
#pragma unroll
        for (int r = 0; r < RH; ++r) {
          // padding rows: a huge max and zero weight, so they add exactly 0
          st_m[r] = ((rmask >> (r0 + r)) & 1u) ? mrow[r0 + r] : 1e30f;
          st_s[r] = ((rmask >> (r0 + r)) & 1u) ? invl[r0 + r] : 0.f;
        }
      }
      if (ctid == 0) RKV_STAMP(it, 3);

      // ================================================= pass 2
      const float inv_nm1 = N > 1 ? 1.f / static_cast<float>(N - 1) : 0.f;
      if (is_soft) {
        for (int k = 0; k < s.nt; ++k) {
          const int t0 = s.start + kTile * k;
          const int j = t0 + row;
          uint32_t v[RH];
          tmem_ld_rows<RH>(tmem + (static_cast<uint32_t>(q4 * 32) << 16) + k * RP + r0, v);
          tmem_wait_ld();
          float pq[4] = {0.f, 0.f, 0.f, 0.f};
          if (t0 + kTile <= c) {
#pragma unroll
            for (int r = 0; r < RH; ++r)
              pq[r & 3] = fmaf(ex2(fmaf(__uint_as_float(v[r]), p.scale_log2, -st_m[r])),
                               st_s[r], pq[r & 3]);
          } else {
#pragma unroll
            for (int r = 0; r < RH; ++r)
              if (((rmask >> (r0 + r)) & 1u) && j < N && j <= c + row_t[r0 + r])
                pq[r & 3] = fmaf(ex2(fmaf(__uint_as_float(v[r]), p.scale_log2, -st_m[r])),
                                 st_s[r], pq[r & 3]);
          }
          if (j < c) {
            // two warps (row halves) add into the zeroed slot: a + b either way
            const float ab_ = ((pq[0] + pq[1]) + (pq[2] + pq[3])) * invR;
            atomicAdd(&abar_s[j - s.start], ab_);
            part += ab_;
          }
        }
        // the unit's logits have been read: TMEM may take the next unit
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tfree);
      } else if (CLOSED) {
        for (int kk = 0; kk < s.nt; ++kk) {
          const int k = s.nt - 1 - kk;
          const int j = s.start + kTile * k + row;
          mbar_wait(&full[stage], ph, abort, p.status);
          __syncwarp();
          const uint32_t sb = smem_u32(sm + L.stages + stage * kTileBytes);
          uint4 xs[16];
          load_row(sb, row, xs);
          float dq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int k8 = 0; k8 < 16; ++k8) {
            const float4 ua = *reinterpret_cast<const float4*>(&ufin[k8 * 8]);
            const float4 ub = *reinterpret_cast<const float4*>(&ufin[k8 * 8 + 4]);
            dq[0] = fmaf(bf_lo(xs[k8].x), ua.x, dq[0]);
            dq[1] = fmaf(bf_hi(xs[k8].x), ua.y, dq[1]);
            dq[2] = fmaf(bf_lo(xs[k8].y), ua.z, dq[2]);
            dq[3] = fmaf(bf_hi(xs[k8].y), ua.w, dq[3]);
            dq[0] = fmaf(bf_lo(xs[k8].z), ub.x, dq[0]);
            dq[1] = fmaf(bf_hi(xs[k8].z), ub.y, dq[1]);
            dq[2] = fmaf(bf_lo(xs[k8].w), ub.z, dq[2]);
            dq[3] = fmaf(bf_hi(xs[k8].w), ub.w, dq[3]);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[stage]);
          if (++stage == NS) { stage = 0; ph ^= 1; }
          if (j < c) {
            const float rho = rhoc[j - s.start];
            const float dot = (dq[0] + dq[1]) + (dq[2] + dq[3]);
            const float m = (rho * dot - (rho > 0.f ? 1.f : 0.f)) * inv_nm1;
            marr[j - s.start] = m;
            part += ex2(m * kLog2e);
          }
        }
      }
      if (ctid == 0) RKV_STAMP(it, 4);

      // ================================================= exchange 2 and output
      part = warp_reduce_sum(part);
      if (lane == 0) rsum[warp - 4] = part;
      named_bar_sync(1, kConsumers);
      float* xb2 = xbuf + XB;
      float* g2 = reinterpret_cast<float*>(sm + L.gath2);   // [cs][4] received sums
      if (ctid == 0) {
        xb2[0] = ((rsum[0] + rsum[1]) + (rsum[2] + rsum[3])) +
                 ((rsum[4] + rsum[5]) + (rsum[6] + rsum[7]));
        xb2[1] = (rsum[8] + rsum[9]) + (rsum[10] + rsum[11]);
        xb2[2] = 0.f;
        xb2[3] = 0.f;
        mbar_arrive_expect_tx(&redbar[1], cs * 16);
      }
      named_bar_sync(1, kConsumers);
      cluster_push(xb2, g2, 1, cs, rank, &redbar[1], ctid);
      mbar_wait<true>(&redbar[1], it & 1, abort, p.status);
      __syncwarp();
      if (ctid == 0) {
        float sa = 0.f, se = 0.f;
        for (int rr = 0; rr < cs; ++rr) {
          sa += g2[4 * rr];
          se += g2[4 * rr + 1];
        }
        rsum[16] = sa > 0.f ? 1.f / sa : 0.f;
        rsum[17] = se > 0.f ? 1.f / se : 0.f;
      }
      named_bar_sync(1, kConsumers);
      const float inv_sa = rsum[16], inv_se = rsum[17];
      if (ctid == 0) RKV_STAMP(it, 5);
      for (int i = ctid; i < s.len; i += kConsumers) {
        const int j = s.start + i;
        const int64_t g = s.base + j;
        if (j < c) {
          p.a_out[g] = abar_s[i] * inv_sa;
          if constexpr (CLOSED) {
            const float m = marr[i];
            p.r_out[g] = ex2(m * kLog2e) * inv_se;
            if (p.m_out) p.m_out[g] = m;
          }
        } else {
          p.a_out[g] = 0.f;
          p.r_out[g] = 0.f;
          if (p.m_out) p.m_out[g] = 0.f;
        }
      }
      if (!CLOSED && p.rho_out && rank == 0) {
        const int64_t pe = p.rho_off[u + 1];
        for (int64_t g = p.rho_off[u] + N + ctid; g < pe; g += kConsumers) p.rho_out[g] = 0.f;
      }
      if (ctid == 0) RKV_STAMP(it, 6);
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<1>(tmem, kTmemColsTotal);
  }
}

template <int RP, bool CLOSED>
void* score_fn() {
  return reinterpret_cast<void*>(&score_kernel<RP, CLOSED>);
}

void* pick(int rp, bool closed) {
  if (rp == 16) return closed ? score_fn<16, true>() : score_fn<16, false>();
  return closed ? score_fn<32, true>() : score_fn<32, false>();
}

}  // namespace

#ifdef RKV_TRACE
cudaError_t score_trace_read(void* dst, size_t bytes) {
  return cudaMemcpyFromSymbol(dst, g_score_trace, bytes);
}
#endif

cudaError_t score_configure(int rp, bool closed, int smem_bytes, int cs) {
  void* f = pick(rp, closed);
  cudaError_t e = cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes);
  if (e != cudaSuccess) return e;
  if (cs > 8) e = cudaFuncSetAttribute(f, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

int score_max_clusters(int rp, bool closed, int smem_bytes, int cs) {
  void* f = pick(rp, closed);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(cs * 8, 1, 1);
  cfg.blockDim = dim3(kScoreThreads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = cs;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, f, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t launch_score(const CUtensorMap& kmap, const CUtensorMap& qmap, const ScoreParams& p,
                         int rp, bool closed, int nclusters, cudaStream_t st) {
  const ScoreLayout L = score_layout(rp, closed, p.nstages);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nclusters * p.cs, 1, 1);
  cfg.blockDim = dim3(kScoreThreads, 1, 1);
  cfg.dynamicSmemBytes = L.total + 1024;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = p.cs;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  if (rp == 16) {
    if (closed) return cudaLaunchKernelEx(&cfg, score_kernel<16, true>, kmap, qmap, p);
    return cudaLaunchKernelEx(&cfg, score_kernel<16, false>, kmap, qmap, p);
  }
  if (closed) return cudaLaunchKernelEx(&cfg, score_kernel<32, true>, kmap, qmap, p);
  return cudaLaunchKernelEx(&cfg, score_kernel<32, false>, kmap, qmap, p);
}

}  // namespace rkv
