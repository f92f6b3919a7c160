// Score kernel: importance (R-KV 重要性打分) and, in closed-form mode, the
// redundancy row mean (R-KV 冗余打分) for every unit, in one pass over K.
//
// One thread-block cluster of `cs` CTAs owns one unit at a time; CTA `rank`
// owns the contiguous token chunk [rank*L, rank*L + L) (L a multiple of 128).
// Each chunk is streamed twice as 128-token K tiles through a TMA ring:
//
//   pass 1 (forward order, loads kept in L2 with evict_last):
//     - logits z = K_tile . Q^T on tcgen05 (M = 128 tokens, N = padded G*w,
//       fp32 accumulator in TMEM); per-thread online softmax statistics
//       (running max and sum of 2^(y - max), y = z * log2(e) / sqrt(d));
//     - key norms ||k|| on CUDA cores -> rho = 1/||k||;
//     - (closed form) U = sum_j rho_j k_j.
//   cluster exchange #1: merge (max, sum) per query row and U over the cluster
//     through distributed shared memory.
//   pass 2 (reverse order, so the most recently loaded tiles -- most likely
//     still in L2 -- come first):
//     - logits again; abar_j = (1/(G w)) sum_rows 2^(y - M_row) / L_row;
//     - (closed form) m_j = (rho_j k_j . U - khat_j . khat_j) / (N - 1).
//   cluster exchange #2: sum of abar over candidates and of exp(m).
//   write a = abar / sum, r = exp(m) / sum (window rows get 0).
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 MMA issuer and TMEM
// owner, warps 4-7 logits/softmax (thread = token row of the tile, lane
// quarter = warp % 4), warps 8-11 norms / U / k.U (thread = token row).
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

constexpr int kNAcc = 4;  // TMEM accumulator buffers

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

template <int RP>
__device__ __forceinline__ void tmem_ld_rows(uint32_t taddr, uint32_t (&v)[RP]) {
  if constexpr (RP == 16) tmem_ld16(taddr, v);
  else tmem_ld32(taddr, v);
}

// Merge two (max, sum) softmax statistics in the log2 domain.
__device__ __forceinline__ void merge_stat(float& m, float& s, float om, float os) {
  const float M = fmaxf(m, om);
  if (M == -INFINITY) {
    m = M;
    s = 0.f;
    return;
  }
  s = s * ex2(m - M) + os * ex2(om - M);
  m = M;
}

// Exchange `nvals` floats at `xb` (this CTA's partials) with every CTA of the
// cluster: release-arrive on each CTA's barrier, then wait for all of them.
__device__ __forceinline__ void cluster_exchange(uint64_t* bar, uint32_t parity, int cs,
                                                 int ctid, volatile int* abort, int* status) {
  fence_acq_rel_cluster();
  named_bar_sync(1, 256);
  if (ctid == 0) {
    const uint32_t local = smem_u32(bar);
    for (int rr = 0; rr < cs; ++rr) mbar_arrive_cluster(mapa(local, rr));
  }
  mbar_wait<true>(bar, parity, abort, status);
  __syncwarp();
}

template <int RP, bool CLOSED>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                 const ScoreParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const int NS = p.nstages;
  const ScoreLayout L = score_layout(RP, CLOSED, p.lmax, NS);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_ctarank());
  const int cid = static_cast<int>(cluster_id_x());
  const int ncl = static_cast<int>(cluster_count_x());
  const int cs = p.cs;
  const int XB = score_xb(RP);

  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* empty = full + NS;
  uint64_t* acc_full = empty + NS;
  uint64_t* acc_empty = acc_full + kNAcc;
  uint64_t* qfull = acc_empty + kNAcc;
  uint64_t* qempty = qfull + 2;
  uint64_t* redbar = qempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L.slot);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + L.flags);
  float* rsum = reinterpret_cast<float*>(sm + L.rsum);
  float* xbuf = reinterpret_cast<float*>(sm + L.xbuf);
  constexpr uint32_t kTmemCols = (kNAcc * RP < 32) ? 32 : kNAcc * RP;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);  // MMA commit + 4 norm warps
    }
    for (int b = 0; b < kNAcc; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&qfull[b], 1);
      mbar_init(&qempty[b], 1);
      mbar_init(&redbar[b], cs);
    }
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc<1>(tmem_slot, kTmemCols);
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
      const uint64_t keep = policy_evict_last(), drop = policy_evict_first();
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
        for (int pass = 0; pass < 2; ++pass) {
          for (int kk = 0; kk < s.nt; ++kk) {
            const int k = pass ? s.nt - 1 - kk : kk;
            if (mbar_wait(&empty[stage], ph ^ 1, abort, p.status)) {
              uint8_t* dst = sm + L.stages + stage * kTileBytes;
              const int y = static_cast<int>(s.base + s.start + kTile * k);
              mbar_arrive_expect_tx(&full[stage], kTileBytes);
              tma_load_2d(dst, &kmap, &full[stage], 0, y, pass ? drop : keep);
              tma_load_2d(dst + kTileBytes / 2, &kmap, &full[stage], 64, y, pass ? drop : keep);
            }
            if (++stage == NS) { stage = 0; ph ^= 1; }
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, RP);
      int stage = 0, ab = 0;
      uint32_t ph = 0, aph = 0;
      int it = 0;
      for (int u = cid; u < p.num_units; u += ncl, ++it) {
        const UnitSched s = unit_sched(p, u, rank);
        const int qb = it & 1;
        bool ok = mbar_wait(&qfull[qb], (it >> 1) & 1, abort, p.status);
        const uint32_t qaddr = smem_u32(sm + L.q + qb * RP * 256);
        for (int pass = 0; pass < 2; ++pass) {
          for (int kk = 0; kk < s.nt; ++kk) {
            bool go = mbar_wait(&full[stage], ph, abort, p.status);
            go = mbar_wait(&acc_empty[ab], aph ^ 1, abort, p.status) && go && ok;
            tc_fence_after();
            if (go) {
              const uint32_t kaddr = smem_u32(sm + L.stages + stage * kTileBytes);
              const uint32_t d = tmem + ab * RP;
#pragma unroll
              for (int kq = 0; kq < 8; ++kq) {
                const uint32_t ko = (kq >> 2) * (kTileBytes / 2) + (kq & 3) * 32;
                const uint32_t qo = (kq >> 2) * (RP * 128) + (kq & 3) * 32;
                mma_bf16<1>(d, desc_kmajor_sw128(kaddr + ko), desc_kmajor_sw128(qaddr + qo),
                            idesc, kq > 0);
              }
              mma_commit(&empty[stage]);
              mma_commit(&acc_full[ab]);
            }
            if (++stage == NS) { stage = 0; ph ^= 1; }
            if (++ab == kNAcc) { ab = 0; aph ^= 1; }
          }
        }
        if (ok) mma_commit(&qempty[qb]);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ consumers
    const int ctid = threadIdx.x - 128;      // 0..255
    const bool is_soft = warp < 8;           // warps 4-7: logits / softmax
    const int q4 = warp & 3;                 // TMEM lane quarter
    const int row = q4 * 32 + lane;          // token row of the tile
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

    int stage = 0, ab = 0, ntile1 = 0;
    uint32_t ph = 0, aph = 0;
    int it = 0;
    for (int u = cid; u < p.num_units; u += ncl, ++it) {
      const UnitSched s = unit_sched(p, u, rank);
      const int N = s.n, c = s.c, w = p.w;
      float st_m[RP], st_s[RP];  // pass 1: running stats; pass 2: row max and 1/sum
#pragma unroll
      for (int r = 0; r < RP; ++r) { st_m[r] = -INFINITY; st_s[r] = 0.f; }
      float U4[4] = {0.f, 0.f, 0.f, 0.f};
      float part = 0.f;  // pass 2: sum of abar (softmax warps) or of exp(m) (norm warps)

      // ================================================= pass 1
      for (int k = 0; k < s.nt; ++k) {
        const int t0 = s.start + kTile * k;
        if (is_soft) {
          mbar_wait(&acc_full[ab], aph, abort, p.status);
          __syncwarp();
          tc_fence_after();
          uint32_t v[RP];
          tmem_ld_rows<RP>(tmem + (static_cast<uint32_t>(q4 * 32) << 16) + ab * RP, v);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
          if (++ab == kNAcc) { ab = 0; aph ^= 1; }
          const int j = t0 + row;
          if (t0 + kTile <= c) {
#pragma unroll
            for (int r = 0; r < RP; ++r) {
              if (r < p.R) {
                const float y = __uint_as_float(v[r]) * p.scale_log2;
                if (y > st_m[r]) { st_s[r] = st_s[r] * ex2(st_m[r] - y) + 1.f; st_m[r] = y; }
                else st_s[r] += ex2(y - st_m[r]);
              }
            }
          } else {
#pragma unroll
            for (int r = 0; r < RP; ++r) {
              if (r < p.R && j < N && j <= c + (r % w)) {
                const float y = __uint_as_float(v[r]) * p.scale_log2;
                if (y > st_m[r]) { st_s[r] = st_s[r] * ex2(st_m[r] - y) + 1.f; st_m[r] = y; }
                else st_s[r] += ex2(y - st_m[r]);
              }
            }
          }
        } else {
          // norm warps: ||k|| of row `row`, rho, (closed) U accumulation
          mbar_wait(&full[stage], ph, abort, p.status);
          const uint32_t sb = smem_u32(sm + L.stages + stage * kTileBytes);
          const int j = t0 + row;
          float n2a = 0.f, n2b = 0.f;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
#pragma unroll
            for (int cc = 0; cc < 8; ++cc) {
              uint4 x;
              const uint32_t ad = sb + h * (kTileBytes / 2) + row * 128 + ((cc ^ (row & 7)) << 4);
              asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                           : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w) : "r"(ad));
              float f;
              f = bf_lo(x.x); n2a = fmaf(f, f, n2a); f = bf_hi(x.x); n2b = fmaf(f, f, n2b);
              f = bf_lo(x.y); n2a = fmaf(f, f, n2a); f = bf_hi(x.y); n2b = fmaf(f, f, n2b);
              f = bf_lo(x.z); n2a = fmaf(f, f, n2a); f = bf_hi(x.z); n2b = fmaf(f, f, n2b);
              f = bf_lo(x.w); n2a = fmaf(f, f, n2a); f = bf_hi(x.w); n2b = fmaf(f, f, n2b);
            }
          }
          const float n2 = n2a + n2b;
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
#pragma unroll 8
            for (int rr = 0; rr < 32; ++rr) {
              const int rw = q4 * 32 + rr;
              const float rr_rho = rt[rw];
              const uint32_t ad =
                  sb + hh * (kTileBytes / 2) + rw * 128 + ((cidx ^ (rw & 7)) << 4) + sub;
              uint32_t x0, x1;
              asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(x0), "=r"(x1) : "r"(ad));
              U4[0] = fmaf(rr_rho, bf_lo(x0), U4[0]);
              U4[1] = fmaf(rr_rho, bf_hi(x0), U4[1]);
              U4[2] = fmaf(rr_rho, bf_lo(x1), U4[2]);
              U4[3] = fmaf(rr_rho, bf_hi(x1), U4[3]);
            }
          } else {
            if (j < N && p.rho_out) p.rho_out[s.base + j] = rho;
          }
          ++ntile1;
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[stage]);
          if (++stage == NS) { stage = 0; ph ^= 1; }
        }
      }

      // ================================================= exchange 1
      if (is_soft) {
#pragma unroll
        for (int r = 0; r < RP; ++r) {
#pragma unroll
          for (int o = 16; o; o >>= 1) {
            const float om = __shfl_xor_sync(0xffffffffu, st_m[r], o);
            const float os = __shfl_xor_sync(0xffffffffu, st_s[r], o);
            merge_stat(st_m[r], st_s[r], om, os);
          }
        }
        if (lane == 0) {
#pragma unroll
          for (int r = 0; r < RP; ++r) {
            red1[(q4 * RP + r) * 2 + 0] = st_m[r];
            red1[(q4 * RP + r) * 2 + 1] = st_s[r];
          }
        }
      } else if (CLOSED) {
#pragma unroll
        for (int i = 0; i < 4; ++i) red2[q4 * 128 + lane * 4 + i] = U4[i];
      }
      named_bar_sync(1, 256);
      float* xa = xbuf;  // exchange buffer of round 1
      if (ctid < RP) {
        float m = -INFINITY, sacc = 0.f;
        for (int q = 0; q < 4; ++q) merge_stat(m, sacc, red1[(q * RP + ctid) * 2], red1[(q * RP + ctid) * 2 + 1]);
        xa[2 * ctid] = m;
        xa[2 * ctid + 1] = sacc;
      }
      if (CLOSED && ctid >= 128) {
        const int e = ctid - 128;
        xa[2 * RP + e] = red2[e] + red2[128 + e] + red2[256 + e] + red2[384 + e];
      }
      cluster_exchange(&redbar[0], it & 1, cs, ctid, abort, p.status);
      if (ctid < RP) {
        float m = -INFINITY, sacc = 0.f;
        const uint32_t la = smem_u32(&xa[2 * ctid]);
        for (int rr = 0; rr < cs; ++rr) {
          const uint32_t ra = mapa(la, rr);
          merge_stat(m, sacc, ld_cluster_f32(ra), ld_cluster_f32(ra + 4));
        }
        mrow[ctid] = m;
        invl[ctid] = sacc > 0.f ? 1.f / sacc : 0.f;
      }
      if (CLOSED && ctid >= 128) {
        const int e = ctid - 128;
        const uint32_t la = smem_u32(&xa[2 * RP + e]);
        float acc = 0.f;
        for (int rr = 0; rr < cs; ++rr) acc += ld_cluster_f32(mapa(la, rr));
        ufin[e] = acc;
      }
      named_bar_sync(1, 256);
      if (is_soft) {
#pragma unroll
        for (int r = 0; r < RP; ++r) {
          st_m[r] = (r < p.R) ? mrow[r] : 0.f;
          st_s[r] = (r < p.R) ? invl[r] : 0.f;
        }
      }

      // ================================================= pass 2 (reverse)
      const float inv_nm1 = N > 1 ? 1.f / static_cast<float>(N - 1) : 0.f;
      for (int kk = 0; kk < s.nt; ++kk) {
        const int k = s.nt - 1 - kk;
        const int t0 = s.start + kTile * k;
        const int j = t0 + row;
        if (is_soft) {
          mbar_wait(&acc_full[ab], aph, abort, p.status);
          __syncwarp();
          tc_fence_after();
          uint32_t v[RP];
          tmem_ld_rows<RP>(tmem + (static_cast<uint32_t>(q4 * 32) << 16) + ab * RP, v);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&acc_empty[ab]);
          if (++ab == kNAcc) { ab = 0; aph ^= 1; }
          float pj = 0.f;
          if (t0 + kTile <= c) {
#pragma unroll
            for (int r = 0; r < RP; ++r)
              if (r < p.R) pj = fmaf(ex2(fmaf(__uint_as_float(v[r]), p.scale_log2, -st_m[r])), st_s[r], pj);
          } else {
#pragma unroll
            for (int r = 0; r < RP; ++r)
              if (r < p.R && j < N && j <= c + (r % w))
                pj = fmaf(ex2(fmaf(__uint_as_float(v[r]), p.scale_log2, -st_m[r])), st_s[r], pj);
          }
          if (j < c) {
            const float ab_ = pj * invR;
            abar_s[j - s.start] = ab_;
            part += ab_;
          }
        } else {
          mbar_wait(&full[stage], ph, abort, p.status);
          if constexpr (CLOSED) {
            const uint32_t sb = smem_u32(sm + L.stages + stage * kTileBytes);
            float da = 0.f, db = 0.f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
#pragma unroll
              for (int cc = 0; cc < 8; ++cc) {
                uint4 x;
                const uint32_t ad = sb + h * (kTileBytes / 2) + row * 128 + ((cc ^ (row & 7)) << 4);
                asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                             : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w) : "r"(ad));
                const float4 ua = *reinterpret_cast<const float4*>(&ufin[h * 64 + cc * 8]);
                const float4 ub = *reinterpret_cast<const float4*>(&ufin[h * 64 + cc * 8 + 4]);
                da = fmaf(bf_lo(x.x), ua.x, da); db = fmaf(bf_hi(x.x), ua.y, db);
                da = fmaf(bf_lo(x.y), ua.z, da); db = fmaf(bf_hi(x.y), ua.w, db);
                da = fmaf(bf_lo(x.z), ub.x, da); db = fmaf(bf_hi(x.z), ub.y, db);
                da = fmaf(bf_lo(x.w), ub.z, da); db = fmaf(bf_hi(x.w), ub.w, db);
              }
            }
            if (j < c) {
              const float rho = rhoc[j - s.start];
              const float m = (rho * (da + db) - (rho > 0.f ? 1.f : 0.f)) * inv_nm1;
              marr[j - s.start] = m;
              part += ex2(m * kLog2e);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[stage]);
          if (++stage == NS) { stage = 0; ph ^= 1; }
        }
      }

      // ================================================= exchange 2 and output
      part = warp_reduce_sum(part);
      if (lane == 0) rsum[warp - 4] = part;
      named_bar_sync(1, 256);
      float* xb2 = xbuf + XB;
      if (ctid == 0) {
        xb2[0] = rsum[0] + rsum[1] + rsum[2] + rsum[3];
        xb2[1] = rsum[4] + rsum[5] + rsum[6] + rsum[7];
      }
      cluster_exchange(&redbar[1], it & 1, cs, ctid, abort, p.status);
      if (ctid == 0) {
        float sa = 0.f, se = 0.f;
        const uint32_t la = smem_u32(&xb2[0]);
        for (int rr = 0; rr < cs; ++rr) {
          const uint32_t ra = mapa(la, rr);
          sa += ld_cluster_f32(ra);
          se += ld_cluster_f32(ra + 4);
        }
        rsum[8] = sa > 0.f ? 1.f / sa : 0.f;
        rsum[9] = se > 0.f ? 1.f / se : 0.f;
      }
      named_bar_sync(1, 256);
      const float inv_sa = rsum[8], inv_se = rsum[9];
      for (int i = ctid; i < s.len; i += 256) {
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
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<1>(tmem, kTmemCols);
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
  const ScoreLayout L = score_layout(rp, closed, p.lmax, p.nstages);
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
