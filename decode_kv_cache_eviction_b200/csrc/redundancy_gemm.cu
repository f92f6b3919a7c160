// Redundancy kernel, GEMM form (R-KV 冗余打分: cosine similarity between key
// vectors).  For every unit and candidate row i:
//
//   m_i = rho_i * sum_{j != i, j < N} rho_j * (k_i . k_j) / (N - 1),   rho = 1/||k||
//   r_i = exp(m_i) / sum_{i' in C} exp(m_i')
//
// The products k_i . k_j are tile products on the 5th-generation tensor cores
// (tcgen05.mma, bf16 x bf16 -> fp32 in TMEM; exact products of the raw bf16
// keys, so the unit-norm scaling is applied in fp32 in the epilogue rather than
// by rounding khat to bf16).  The epilogue reads each 128 x 256 accumulator tile
// from TMEM, weights column j by rho_j, drops the diagonal, and folds the tile
// into per-row partial sums, so the N x N similarity matrix never reaches HBM.
// The last CTA to finish a unit (atomic counter) applies the token softmax.
//
// Work item = (unit, block of rows).  In pair mode a cluster of two CTAs runs
// one M = 256 MMA (cta_group::2): each CTA holds 128 A rows and half of each
// 256-key B tile, which halves the shared-memory traffic per SM.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 MMA issuer (leader CTA
// only in pair mode) and TMEM owner, warps 4-11 epilogue (warp % 4 selects the
// TMEM lane quarter, (warp - 4) / 4 the 128-column half of the tile).
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

__device__ __forceinline__ int find_unit(const int* item_off, int U, int item) {
  int lo = 0, hi = U - 1;  // largest u with item_off[u] <= item
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(&item_off[mid]) <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

template <bool kPair>
__global__ void __launch_bounds__(kGemmThreads, 1)
    redundancy_gemm_kernel(const __grid_constant__ CUtensorMap amap,
                           const __grid_constant__ CUtensorMap bmap, const GemmParams p) {
  using C = GemmCfg<kPair>;
  constexpr int NSB = C::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const GemmLayout L = gemm_layout<kPair>();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rank = kPair ? static_cast<int>(cluster_ctarank()) : 0;
  const int group_id = kPair ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int ngroups = kPair ? static_cast<int>(cluster_count_x()) : static_cast<int>(gridDim.x);
  const bool leader = rank == 0;

  uint64_t* a_full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* a_empty = a_full + 1;
  uint64_t* b_full = a_empty + 1;
  uint64_t* b_empty = b_full + NSB;
  uint64_t* acc_full = b_empty + NSB;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* rho_full = acc_empty + 2;      // [kRhoSlots] rho tile landed
  uint64_t* rho_empty = rho_full + kRhoSlots;  // [kRhoSlots] epilogue done with it
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L.slot);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + L.flags);
  volatile int* last_flag = reinterpret_cast<volatile int*>(sm + L.flags + 4);

  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int s = 0; s < NSB; ++s) {
      mbar_init(&b_full[s], 1);
      mbar_init(&b_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kPair ? 16 : 8);
    }
    for (int b = 0; b < kRhoSlots; ++b) {
      mbar_init(&rho_full[b], 1);
      mbar_init(&rho_empty[b], 8);   // this CTA's 8 epilogue warps
    }
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc<C::kCtaGroup>(tmem_slot, 512);
    tmem_relinquish<C::kCtaGroup>();
  }
  tc_fence_before();
  if constexpr (kPair) cluster_sync_all();
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = __ldg(&p.item_off[p.num_units]);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&amap);
      prefetch_tmap(&bmap);
      const uint64_t pol = policy_evict_normal();
      const uint32_t a_full_lead = kPair ? mapa(smem_u32(a_full), 0) : smem_u32(a_full);
      int stage = 0;
      uint32_t ph = 0;
      int ai = 0;
      uint32_t rt = 0;   // rho tiles loaded so far
      float* rho_ring = reinterpret_cast<float*>(sm + L.rho);
      for (int item = group_id; item < n_items; item += ngroups, ++ai) {
        const int u = find_unit(p.item_off, p.num_units, item);
        const int blk = item - __ldg(&p.item_off[u]);
        const float* rho_u = p.rho + __ldg(&p.rho_off[u]);
        const int64_t base = __ldg(&p.tok_off[u]);
        const int N = static_cast<int>(__ldg(&p.tok_off[u + 1]) - base);
        const int ya = static_cast<int>(base + blk * C::kRowsPerItem + rank * 128);
        if (mbar_wait(a_empty, (ai & 1) ^ 1, abort, p.status)) {
          uint8_t* ad = sm + L.a;
          if constexpr (kPair) {
            if (leader) mbar_arrive_expect_tx(a_full, 2 * C::kABytes);
            tma_load_2d_pair(ad, &amap, a_full_lead, 0, ya, pol);
            tma_load_2d_pair(ad + C::kABytes / 2, &amap, a_full_lead, 64, ya, pol);
          } else {
            mbar_arrive_expect_tx(a_full, C::kABytes);
            tma_load_2d(ad, &amap, a_full, 0, ya, pol);
            tma_load_2d(ad + C::kABytes / 2, &amap, a_full, 64, ya, pol);
          }
        }
        const int ntiles = (N + C::kN - 1) / C::kN;
        for (int t = 0; t < ntiles; ++t) {
          if (mbar_wait(&b_empty[stage], ph ^ 1, abort, p.status)) {
            uint8_t* bd = sm + L.b + stage * C::kBBytes;
            const int yb = static_cast<int>(base + t * C::kN + rank * C::kBRows);
            if constexpr (kPair) {
              const uint32_t bf_lead = mapa(smem_u32(&b_full[stage]), 0);
              if (leader) mbar_arrive_expect_tx(&b_full[stage], 2 * C::kBBytes);
              tma_load_2d_pair(bd, &bmap, bf_lead, 0, yb, pol);
              tma_load_2d_pair(bd + C::kBBytes / 2, &bmap, bf_lead, 64, yb, pol);
            } else {
              mbar_arrive_expect_tx(&b_full[stage], C::kBBytes);
              tma_load_2d(bd, &bmap, &b_full[stage], 0, yb, pol);
              tma_load_2d(bd + C::kBBytes / 2, &bmap, &b_full[stage], 64, yb, pol);
            }
          }
          if (++stage == NSB) { stage = 0; ph ^= 1; }
          // the 256 column weights of this tile (every CTA of a pair loads its own)
          const uint32_t rs = rt % kRhoSlots;
          if (mbar_wait(&rho_empty[rs], ((rt / kRhoSlots) & 1) ^ 1, abort, p.status)) {
            mbar_arrive_expect_tx(&rho_full[rs], 256 * 4);
            bulk_load(rho_ring + rs * 256, rho_u + t * C::kN, 256 * 4, &rho_full[rs]);
          }
          ++rt;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      const uint32_t idesc = idesc_bf16_f32(C::kMmaM, C::kN);
      int stage = 0, ab = 0;
      uint32_t ph = 0, aph = 0;
      int ai = 0;
      for (int item = group_id; item < n_items; item += ngroups, ++ai) {
        const int u = find_unit(p.item_off, p.num_units, item);
        const int64_t base = __ldg(&p.tok_off[u]);
        const int N = static_cast<int>(__ldg(&p.tok_off[u + 1]) - base);
        const bool aok = mbar_wait(a_full, ai & 1, abort, p.status);
        const uint32_t aaddr = smem_u32(sm + L.a);
        const int ntiles = (N + C::kN - 1) / C::kN;
        for (int t = 0; t < ntiles; ++t) {
          bool go = mbar_wait(&b_full[stage], ph, abort, p.status);
          go = mbar_wait(&acc_empty[ab], aph ^ 1, abort, p.status) && go && aok;
          tc_fence_after();
          if (go) {
            const uint32_t baddr = smem_u32(sm + L.b + stage * C::kBBytes);
            const uint32_t d = tmem + ab * 256;
#pragma unroll
            for (int kq = 0; kq < 8; ++kq) {
              const uint32_t ao = (kq >> 2) * (C::kABytes / 2) + (kq & 3) * 32;
              const uint32_t bo = (kq >> 2) * (C::kBBytes / 2) + (kq & 3) * 32;
              mma_bf16<C::kCtaGroup>(d, desc_kmajor_sw128(aaddr + ao),
                                     desc_kmajor_sw128(baddr + bo), idesc, kq > 0);
            }
            if constexpr (kPair) {
              mma_commit_pair(&b_empty[stage]);
              mma_commit_pair(&acc_full[ab]);
            } else {
              mma_commit(&b_empty[stage]);
              mma_commit(&acc_full[ab]);
            }
          }
          if (++stage == NSB) { stage = 0; ph ^= 1; }
          if (++ab == 2) { ab = 0; aph ^= 1; }
        }
        if (aok) {
          if constexpr (kPair) mma_commit_pair(a_empty);
          else mma_commit(a_empty);
        }
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int etid = threadIdx.x - 128;   // 0..255
    const int ew = warp - 4;              // epilogue warp 0..7
    const int half = ew >> 2;             // column half of the tile
    const int q = warp & 3;               // TMEM lane quarter
    const int rloc = q * 32 + lane;       // row of this CTA's A block
    const float* rho_ring = reinterpret_cast<const float*>(sm + L.rho);
    float* rowx = reinterpret_cast<float*>(sm + L.rowx);
    float* fin = reinterpret_cast<float*>(sm + L.fin);
    const uint32_t acc_empty_lead = kPair ? mapa(smem_u32(acc_empty), 0) : smem_u32(acc_empty);
    int ab = 0;
    uint32_t aph = 0;
    uint32_t rt = 0;   // rho tiles consumed so far
    for (int item = group_id; item < n_items; item += ngroups) {
      const int u = find_unit(p.item_off, p.num_units, item);
      const int blk = item - __ldg(&p.item_off[u]);
      const int64_t base = __ldg(&p.tok_off[u]);
      const int N = static_cast<int>(__ldg(&p.tok_off[u + 1]) - base);
      const int c = N - p.w;
      const int rbase = blk * C::kRowsPerItem + rank * 128;   // unit-local first row
      const int i = rbase + rloc;
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
      const int ntiles = (N + C::kN - 1) / C::kN;
      for (int t = 0; t < ntiles; ++t, ++rt) {
        const int j0 = t * C::kN;
        const uint32_t rs_slot = rt % kRhoSlots;
        const float* rs = rho_ring + rs_slot * 256 + half * 128;
        mbar_wait(&acc_full[ab], aph, abort, p.status);
        mbar_wait(&rho_full[rs_slot], (rt / kRhoSlots) & 1, abort, p.status);
        __syncwarp();
        tc_fence_after();
        const uint32_t tbase =
            tmem + (static_cast<uint32_t>(q * 32) << 16) + ab * 256 + half * 128;
        uint32_t va[32], vb[32], vc[32], vd[32];
        tmem_ld32(tbase, va);
        tmem_ld32(tbase + 32, vb);
        tmem_ld32(tbase + 64, vc);
        tmem_ld32(tbase + 96, vd);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {   // the accumulator is in registers: hand it back to the MMA
          if constexpr (kPair) mbar_arrive_cluster_relaxed(acc_empty_lead + ab * 8);
          else mbar_arrive(&acc_empty[ab]);
        }
        if (++ab == 2) { ab = 0; aph ^= 1; }
        const int cw0 = j0 + half * 128;             // first column of this warp's half
        const int rw0 = rbase + q * 32;              // first row of this warp
        if (!((rw0 < cw0 + 128) && (cw0 < rw0 + 32))) {
          auto fold = [&](const uint32_t (&v)[32], int off) {
#pragma unroll
            for (int cc = 0; cc < 32; cc += 4) {
              const float4 r4 = *reinterpret_cast<const float4*>(rs + off + cc);
              s0 = fmaf(__uint_as_float(v[cc + 0]), r4.x, s0);
              s1 = fmaf(__uint_as_float(v[cc + 1]), r4.y, s1);
              s2 = fmaf(__uint_as_float(v[cc + 2]), r4.z, s2);
              s3 = fmaf(__uint_as_float(v[cc + 3]), r4.w, s3);
            }
          };
          fold(va, 0); fold(vb, 32); fold(vc, 64); fold(vd, 96);
        } else {
          const int jd = i - cw0;                    // this row's diagonal column in the half
          auto fold = [&](const uint32_t (&v)[32], int off) {
#pragma unroll
            for (int cc = 0; cc < 32; cc += 4) {
              const float4 r4 = *reinterpret_cast<const float4*>(rs + off + cc);
              s0 = fmaf(off + cc + 0 == jd ? 0.f : __uint_as_float(v[cc + 0]), r4.x, s0);
              s1 = fmaf(off + cc + 1 == jd ? 0.f : __uint_as_float(v[cc + 1]), r4.y, s1);
              s2 = fmaf(off + cc + 2 == jd ? 0.f : __uint_as_float(v[cc + 2]), r4.z, s2);
              s3 = fmaf(off + cc + 3 == jd ? 0.f : __uint_as_float(v[cc + 3]), r4.w, s3);
            }
          };
          fold(va, 0); fold(vb, 32); fold(vc, 64); fold(vd, 96);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&rho_empty[rs_slot]);
      }
      // ---- item end: combine halves, write m, count the unit's finished blocks
      float tot = (s0 + s1) + (s2 + s3);
      if (half == 1) rowx[rloc] = tot;
      named_bar_sync(3, 256);
      if (half == 0 && i < c) {
        tot += rowx[rloc];
        const float rho_i = __ldg(&p.rho[__ldg(&p.rho_off[u]) + i]);
        p.m_dst[base + i] = rho_i * tot / static_cast<float>(N - 1);
      }
      __threadfence();
      named_bar_sync(3, 256);
      if (etid == 0) {
        const int nblk = __ldg(&p.item_off[u + 1]) - __ldg(&p.item_off[u]);
        const int done = atomicAdd(&p.unit_cnt[u], 1) + 1;
        *last_flag = done == nblk * (kPair ? 2 : 1);
      }
      named_bar_sync(3, 256);
      if (*last_flag) {
        // ---- token softmax over the unit's candidates (|m| <= 1: no max shift)
        __threadfence();
        float sum = 0.f;
        for (int ii = etid; ii < c; ii += 256) sum += ex2(__ldcg(&p.m_dst[base + ii]) * kLog2e);
        sum = warp_reduce_sum(sum);
        if (lane == 0) fin[warp - 4] = sum;
        named_bar_sync(3, 256);
        float totl = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) totl += fin[k];
        const float inv = 1.f / totl;
        for (int ii = etid; ii < c; ii += 256)
          p.r_dst[base + ii] = ex2(__ldcg(&p.m_dst[base + ii]) * kLog2e) * inv;
        named_bar_sync(3, 256);
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  if constexpr (kPair) cluster_sync_all();
  else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc<C::kCtaGroup>(tmem, 512);
  }
}

// One block: items per unit and their prefix, 256-aligned rho segment
// offsets, and zeroed unit counters.
__global__ void plan_kernel(const int64_t* tok_off, int U, int w, int rows_per_item,
                            int* item_off, int* unit_cnt, int64_t* rho_off) {
  __shared__ long long wsum[2][32];
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (U + nt - 1) / nt;
  const int u0 = min(U, tid * per), u1 = min(U, u0 + per);
  long long li = 0, lr = 0;   // this thread's items and padded rho length
  for (int u = u0; u < u1; ++u) {
    const int64_t n = tok_off[u + 1] - tok_off[u];
    const int64_t c = n - w;
    li += c > 0 ? (c + rows_per_item - 1) / rows_per_item : 0;
    lr += (n + kRhoAlign - 1) / kRhoAlign * kRhoAlign;
    unit_cnt[u] = 0;
  }
  // block exclusive scans of li and lr
  long long ii = li, ir = lr;
  const int lane = tid & 31, wp = tid >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long yi = __shfl_up_sync(0xffffffffu, ii, o);
    const long long yr = __shfl_up_sync(0xffffffffu, ir, o);
    if (lane >= o) { ii += yi; ir += yr; }
  }
  if (lane == 31) { wsum[0][wp] = ii; wsum[1][wp] = ir; }
  __syncthreads();
  if (wp == 0) {
    long long xi = lane < (nt >> 5) ? wsum[0][lane] : 0;
    long long xr = lane < (nt >> 5) ? wsum[1][lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long yi = __shfl_up_sync(0xffffffffu, xi, o);
      const long long yr = __shfl_up_sync(0xffffffffu, xr, o);
      if (lane >= o) { xi += yi; xr += yr; }
    }
    wsum[0][lane] = xi;
    wsum[1][lane] = xr;
  }
  __syncthreads();
  long long ri = ii - li + (wp > 0 ? wsum[0][wp - 1] : 0);
  long long rr = ir - lr + (wp > 0 ? wsum[1][wp - 1] : 0);
  for (int u = u0; u < u1; ++u) {
    item_off[u] = static_cast<int>(ri);
    rho_off[u] = rr;
    const int64_t n = tok_off[u + 1] - tok_off[u];
    const int64_t c = n - w;
    ri += c > 0 ? (c + rows_per_item - 1) / rows_per_item : 0;
    rr += (n + kRhoAlign - 1) / kRhoAlign * kRhoAlign;
  }
  if (u1 == U && u0 < u1) {
    item_off[U] = static_cast<int>(ri);
    rho_off[U] = rr;
  }
  if (U == 0 && tid == 0) {
    item_off[0] = 0;
    rho_off[0] = 0;
  }
}

}  // namespace

cudaError_t gemm_configure(bool pair) {
  const int smem = (pair ? gemm_layout<true>().total : gemm_layout<false>().total) + 1024;
  void* f = pair ? reinterpret_cast<void*>(&redundancy_gemm_kernel<true>)
                 : reinterpret_cast<void*>(&redundancy_gemm_kernel<false>);
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

int gemm_max_ctas(bool pair) {
  const int smem = (pair ? gemm_layout<true>().total : gemm_layout<false>().total) + 1024;
  void* f = pair ? reinterpret_cast<void*>(&redundancy_gemm_kernel<true>)
                 : reinterpret_cast<void*>(&redundancy_gemm_kernel<false>);
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (!pair) {
    int per = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, f, kGemmThreads, smem) != cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    return per * nsm;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * nsm, 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, f, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return 2 * n;
}

cudaError_t launch_plan(const int64_t* tok_off, int U, int w, int rows_per_item, int* item_off,
                        int* unit_cnt, int64_t* rho_off, cudaStream_t st) {
  plan_kernel<<<1, 1024, 0, st>>>(tok_off, U, w, rows_per_item, item_off, unit_cnt, rho_off);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const CUtensorMap& amap, const CUtensorMap& bmap, const GemmParams& p,
                        bool pair, int nctas, cudaStream_t st) {
  const int smem = (pair ? gemm_layout<true>().total : gemm_layout<false>().total) + 1024;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nctas, 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = pair ? 2 : 1;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = pair ? 1 : 0;
  if (pair) return cudaLaunchKernelEx(&cfg, redundancy_gemm_kernel<true>, amap, bmap, p);
  return cudaLaunchKernelEx(&cfg, redundancy_gemm_kernel<false>, amap, bmap, p);
}

}  // namespace rkv
