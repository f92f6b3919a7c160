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
// Row-max variant (kMax): the same tiles, folded with a max instead of a
// weighted sum, give the nearest-duplicate redundancy
//   m_i = rho_i * max_{j != i, j < N} rho_j * (k_i . k_j)
// (rho_i >= 0, so the row scaling commutes with the max).  Columns past the end
// of the unit are masked explicitly there, since a zero weight is not neutral
// for a max.
//
// Work item = (unit, block of rows).  In pair mode a cluster of two CTAs runs
// one M = 256 MMA (cta_group::2): each CTA holds 128 A rows and half of each
// 256-key B tile, which halves the shared-memory traffic per SM.
//
// Symmetric form (kSym, row mean on CTA pairs): S = khat khat^T is symmetric,
// so only the 256 x 256 tiles (a, b) with a <= b are computed.  A work item is
// (unit, block b): its 256 keys stay in shared memory as the MMA's B operand
// while the row blocks a = 0 .. b stream through as the A operand, so TMEM
// lane = row of block a and column = key of block b.  Per tile the epilogue
//   - adds rho_i-weighted column sums into registers that persist over the
//     whole item (block b's share from rows of blocks 0 .. b; the diagonal
//     tile with its diagonal dropped), reduced across threads once per item;
//   - for a < b, forms the rho_j-weighted row sums of block a's rows over
//     block b's columns (a 4-thread reduction per 128-column half) and puts
//     them in a shared-memory ring; warp 2 adds the two halves and stores
//     the sums to a scratch slot (a, b), so no epilogue warp waits for
//     another.
// The row weights rho_i of block a come from L2, loaded a tile ahead; the
// column weights of block b are held in registers for the item.
// Every slot is written by exactly one plain store, so nothing needs zeroing
// and the result does not depend on timing.  A finish kernel adds, per row,
// the two CTAs' column sums and the slots (a, b > a) in block order, scales by
// rho_i / (N - 1) and applies the token softmax.
//
// Warp roles: warp 0 TMA producer, warp 1 MMA issuer (leader CTA only in pair
// mode; the whole warp runs the loop and elects one lane per instruction) and
// TMEM owner, then the epilogue warps, warp % 4 selecting the TMEM lane
// quarter.  Row-block form (640 threads = 5 warps per SM sub-partition):
// warps 4-19, (warp - 4) / 4 the 64-column quarter of the tile.  Symmetric
// form (384 threads): warp 2 row-sum store, warps 4-11, (warp - 4) / 4 the
// 128-column half of the tile; with 168 registers a thread, a warp keeps two
// TMEM loads' worth of the tile and the column sums of its 32 columns.
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

#ifdef RKV_TRACE
// Optional per-tile trace (build with -DRKV_TRACE): for the first kGT tiles of
// each CTA, globaltimer stamps of the MMA thread and of epilogue warp 4.
constexpr int kGTCtas = 160, kGT = 64;
__device__ unsigned long long g_gemm_trace[kGTCtas * 2 * kGT * 4];
#define RKV_GSTAMP(role, tile, slot)                                                      \
  do {                                                                                   \
    if ((tile) < kGT && blockIdx.x < kGTCtas)                                            \
      g_gemm_trace[((blockIdx.x * 2 + (role)) * kGT + (tile)) * 4 + (slot)] =            \
          globaltimer_ns();                                                              \
  } while (0)
#else
#define RKV_GSTAMP(role, tile, slot) do { } while (0)
#endif

template <bool B>
struct BoolTag {
  static constexpr bool value = B;
};

__device__ __forceinline__ int find_unit(const int* item_off, int U, int item) {
  int lo = 0, hi = U - 1;  // largest u with item_off[u] <= item
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(&item_off[mid]) <= item) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Block of a work item within its unit.  The symmetric form runs a unit's
// items from the last block (the most tiles) down, so long items start first.
template <bool kSym>
__device__ __forceinline__ int item_block(const int* item_off, int u, int item) {
  const int i0 = __ldg(&item_off[u]);
  if constexpr (kSym) return __ldg(&item_off[u + 1]) - 1 - item;
  return item - i0;
}

// MMA and commit issued by the whole (converged) warp, one lane elected inside
// the instruction sequence: the issue loop's values stay warp-uniform.  The
// MMA carries no compiler memory clobber; its operands are ordered by the
// mbarrier waits before it, which do.
template <int kCtaGroup>
__device__ __forceinline__ void mma_bf16_elect(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  if constexpr (kCtaGroup == 1)
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
  else
    asm volatile(
        "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}
__device__ __forceinline__ void commit_elect(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void commit_pair_elect(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
      "h"(static_cast<uint16_t>(3))
      : "memory");
}

template <bool kPair, bool kMax, bool kSym>
__global__ void __launch_bounds__(gemm_threads(kSym), 1)
    redundancy_gemm_kernel(const __grid_constant__ CUtensorMap amap,
                           const __grid_constant__ CUtensorMap bmap, const GemmParams p) {
  using C = GemmCfg<kPair>;
  constexpr int NSB = C::kStages;
  constexpr int kEpiWarps = (gemm_threads(kSym) - 128) / 32;   // per CTA
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
  uint64_t* row_full = rho_empty + kRhoSlots;  // [kRowRing] symmetric form: partials written
  uint64_t* row_empty = row_full + kRowRing;   // [kRowRing] symmetric form: partials stored
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
      mbar_init(&acc_empty[b], kPair ? 2 * kEpiWarps : kEpiWarps);
    }
    for (int b = 0; b < kRhoSlots; ++b) {
      mbar_init(&rho_full[b], 1);
      mbar_init(&rho_empty[b], kEpiWarps);   // this CTA's epilogue warps
    }
    for (int b = 0; b < kRowRing; ++b) {
      mbar_init(&row_full[b], kEpiWarps);   // the epilogue warps
      mbar_init(&row_empty[b], 1);    // the row-store warp
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
        const int blk = item_block<kSym>(p.item_off, u, item);
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
        // symmetric form: the row blocks 0 .. blk against the item's block
        const int ntiles = kSym ? blk + 1 : (N + C::kN - 1) / C::kN;
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
          // the tile's 256 rho values (column weights of the row-block form);
          // every CTA of a pair loads its own
          if constexpr (!kSym) {
            const uint32_t rs = rt % kRhoSlots;
            if (mbar_wait(&rho_empty[rs], ((rt / kRhoSlots) & 1) ^ 1, abort, p.status)) {
              mbar_arrive_expect_tx(&rho_full[rs], 256 * 4);
              bulk_load(rho_ring + rs * 256, rho_u + t * C::kN, 256 * 4, &rho_full[rs]);
            }
            ++rt;
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (leader) {   // the whole warp, converged; one elected lane issues
      const uint32_t idesc = idesc_bf16_f32(C::kMmaM, C::kN);
      int stage = 0, ab = 0;
      uint32_t ph = 0, aph = 0;
      int ai = 0, tcount = 0;
      for (int item = group_id; item < n_items; item += ngroups, ++ai) {
        const int u = find_unit(p.item_off, p.num_units, item);
        const int64_t base = __ldg(&p.tok_off[u]);
        const int N = static_cast<int>(__ldg(&p.tok_off[u + 1]) - base);
        const bool aok = __all_sync(0xffffffffu, mbar_wait(a_full, ai & 1, abort, p.status));
        const uint32_t aaddr = smem_u32(sm + L.a);
        // descriptors of the item's fixed block for the 8 K-steps: the A
        // operand, or in the symmetric form the B operand
        uint64_t fdesc[8];
#pragma unroll
        for (int kq = 0; kq < 8; ++kq)
          fdesc[kq] = desc_kmajor_sw128(aaddr + (kq >> 2) * (C::kABytes / 2) + (kq & 3) * 32);
        const int ntiles =
            kSym ? item_block<kSym>(p.item_off, u, item) + 1 : (N + C::kN - 1) / C::kN;
        for (int t = 0; t < ntiles; ++t, ++tcount) {
          RKV_GSTAMP(0, tcount, 0);
          bool go = mbar_wait(&b_full[stage], ph, abort, p.status);
          RKV_GSTAMP(0, tcount, 1);
          go = mbar_wait(&acc_empty[ab], aph ^ 1, abort, p.status) && go && aok;
          go = __all_sync(0xffffffffu, go);
          RKV_GSTAMP(0, tcount, 2);
          tc_fence_after();
          if (go) {
            // streamed-tile descriptors: the stage's base plus each K-step's
            // offset in 16-byte units (the start-address field cannot carry:
            // smem < 256 KB)
            const uint64_t sdesc0 = desc_kmajor_sw128(smem_u32(sm + L.b + stage * C::kBBytes));
            const uint32_t d = tmem + ab * 256;
#pragma unroll
            for (int kq = 0; kq < 8; ++kq) {
              const uint32_t bo = (kq >> 2) * (C::kBBytes / 2) + (kq & 3) * 32;
              if constexpr (kSym)   // A = row block t (streamed), B = the item's block
                mma_bf16_elect<C::kCtaGroup>(d, sdesc0 + (bo >> 4), fdesc[kq], idesc, kq > 0);
              else
                mma_bf16_elect<C::kCtaGroup>(d, fdesc[kq], sdesc0 + (bo >> 4), idesc, kq > 0);
            }
            if constexpr (kPair) {
              commit_pair_elect(&b_empty[stage]);
              commit_pair_elect(&acc_full[ab]);
            } else {
              commit_elect(&b_empty[stage]);
              commit_elect(&acc_full[ab]);
            }
          }
          RKV_GSTAMP(0, tcount, 3);
          if (++stage == NSB) { stage = 0; ph ^= 1; }
          if (++ab == 2) { ab = 0; aph ^= 1; }
        }
        if (aok) {
          if constexpr (kPair) commit_pair_elect(a_empty);
          else commit_elect(a_empty);
        }
      }
    }
    __syncwarp();
  } else if (warp == 2 && kSym) {
    // ------------------------------------------------ row-sum store (symmetric)
    // Per tile below the item's block: the two column halves' partial row
    // sums of this CTA's 128 rows, added and stored to the tile's scratch slot.
    const float* rr = reinterpret_cast<const float*>(sm + L.rowr);
    uint32_t n = 0;   // row exchanges so far
    for (int item = group_id; item < n_items; item += ngroups) {
      const int u = find_unit(p.item_off, p.num_units, item);
      const int blk = item_block<kSym>(p.item_off, u, item);
      const int nb = __ldg(&p.item_off[u + 1]) - __ldg(&p.item_off[u]);
      float* cs_u = p.cs + __ldg(&p.cs_off[u]);
      for (int t = 0; t < blk; ++t, ++n) {
        const uint32_t s = n % kRowRing;
        mbar_wait(&row_full[s], (n / kRowRing) & 1, abort, p.status);
        const float* x = rr + s * 512;
        float tot[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int rl = lane + 32 * j;
          tot[j] = x[rl] + x[128 + rl];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&row_empty[s]);
        const int64_t seg = 512 * static_cast<int64_t>(nb) +
                            256 * (static_cast<int64_t>(t) * (nb - 1) -
                                   static_cast<int64_t>(t) * (t - 1) / 2);
        float* dst = cs_u + seg + static_cast<int64_t>(blk - t - 1) * 256 + rank * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[lane + 32 * j] = tot[j];
      }
    }
  } else if (warp >= 4 && kSym) {
    // ------------------------------------------------- epilogue, symmetric form
    // 8 warps: warp % 4 selects the TMEM lane quarter, (warp - 4) / 4 the
    // 128-column half of the tile.  Per tile a warp reads four 32-register
    // chunks (16 lanes x 64 columns each), two in flight: the load of the next
    // chunk overlaps the folds of the current one.
    const int ew = warp - 4;              // epilogue warp 0..7
    const int ch = ew >> 2;               // 128-column half of the tile
    const int q = warp & 3;               // TMEM lane quarter
    const int gq = lane >> 2, tq = lane & 3;   // quad and thread within it
    float* rowr = reinterpret_cast<float*>(sm + L.rowr);    // [kRowRing][ch][128]
    float2* colx = reinterpret_cast<float2*>(sm + L.colx);  // [2][cg][q][32] column sums
    const uint32_t acc_empty_lead = mapa(smem_u32(acc_empty), 0);
    const int rq = rank * 128 + q * 32;   // first row of this warp's quarter in a block
    int ab = 0;
    uint32_t aph = 0;
    uint32_t rt = 0;   // rho tiles consumed so far
    uint32_t nx = 0;   // row exchanges so far
    int ib = 0;        // double buffer of the per-item column exchange
    for (int item = group_id; item < n_items; item += ngroups, ib ^= 1) {
      const int u = find_unit(p.item_off, p.num_units, item);
      const int blk = item_block<kSym>(p.item_off, u, item);
      const float* rho_u = p.rho + __ldg(&p.rho_off[u]);
      float* cs_u = p.cs + __ldg(&p.cs_off[u]);
      // weights rho_j of this thread's 32 columns of block blk: column group
      // cg = 2 ch + c, columns 8k + 2tq + {0, 1} of the group
      float2 wt[2][8];
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int k = 0; k < 8; ++k)
          wt[c][k] = __ldg(reinterpret_cast<const float2*>(rho_u + blk * 256 + ch * 128 + c * 64 +
                                                           2 * tq + 8 * k));
      // rho_i-weighted column sums of the item's block over this thread's rows
      float cp[2][16];
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int k = 0; k < 16; ++k) cp[c][k] = 0.f;
      // One tile: the row blocks t < blk, then the diagonal tile t = blk.
      // weights of this thread's 4 rows of block t (gq + 8k of the quarter),
      // loaded one tile ahead
      const float* wrow = rho_u + rq + gq;
      float nw0 = __ldg(wrow), nw1 = __ldg(wrow + 8), nw2 = __ldg(wrow + 16), nw3 = __ldg(wrow + 24);
      auto tile = [&](auto diag_tag, int t) {
        constexpr bool kDiag = decltype(diag_tag)::value;
        const float w0 = nw0, w1 = nw1, w2 = nw2, w3 = nw3;
        if constexpr (!kDiag) {   // the next tile of the item exists
          const float* wn = wrow + (t + 1) * 256;
          nw0 = __ldg(wn);
          nw1 = __ldg(wn + 8);
          nw2 = __ldg(wn + 16);
          nw3 = __ldg(wn + 24);
        }
        if (ew == 0 && lane == 0) RKV_GSTAMP(1, rt, 0);
        mbar_wait(&acc_full[ab], aph, abort, p.status);
        if (ew == 0 && lane == 0) RKV_GSTAMP(1, rt, 1);
        __syncwarp();
        tc_fence_after();
        const uint32_t tbase =
            tmem + (static_cast<uint32_t>(q * 32) << 16) + ab * 256 + ch * 128;
        uint32_t va[32], vb[32];
        // One chunk (16 lanes h of the quarter x 64 columns of group c): the
        // column sums take rows gq + 16h (weight wa) and gq + 16h + 8 (wb);
        // off the diagonal the row sums of those two rows take the chunk's 16
        // columns, two partial values each.  On the diagonal tile (rows and
        // columns of one block) the element column - row == dd, local to the
        // warp's 32 x 64 sub-block, is dropped and the row sums are skipped:
        // block blk's rows get their share from the column sums.
        auto fold = [&](uint32_t (&v)[32], int h, int c, const float2 (&w)[8], float (&cc)[16],
                        float& pa, float& pb, float& qa, float& qb, float wa, float wb) {
          if constexpr (kDiag) {
            const int dd = rq - ch * 128 - 64 * c;
            if (dd > -32 && dd < 64) {
#pragma unroll
              for (int k = 0; k < 8; ++k)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int col = 8 * k + 2 * tq + (e & 1);
                  const int row = 16 * h + gq + ((e >> 1) << 3);
                  if (col - row == dd) v[4 * k + e] = 0u;
                }
            }
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float x0 = __uint_as_float(v[4 * k]), x1 = __uint_as_float(v[4 * k + 1]);
            const float y0 = __uint_as_float(v[4 * k + 2]), y1 = __uint_as_float(v[4 * k + 3]);
            if constexpr (!kDiag) fma2(pa, pb, x0, x1, w[k].x, w[k].y);
            fma2(cc[2 * k], cc[2 * k + 1], x0, x1, wa, wa);
            if constexpr (!kDiag) fma2(qa, qb, y0, y1, w[k].x, w[k].y);
            fma2(cc[2 * k], cc[2 * k + 1], y0, y1, wb, wb);
          }
        };
        float a0 = 0.f, b0 = 0.f, a1 = 0.f, b1 = 0.f, a2 = 0.f, b2 = 0.f, a3 = 0.f, b3 = 0.f;
        // chunk order: (lanes 0-15, group 0), (0-15, 1), (16-31, 0), (16-31, 1)
        tmem_ld16x256b_x8(tbase, va);
        tmem_wait_ld_dep(va);
        tmem_ld16x256b_x8(tbase + 64, vb);
        fold(va, 0, 0, wt[0], cp[0], a0, b0, a1, b1, w0, w1);
        tmem_wait_ld_dep(vb);
        tmem_ld16x256b_x8(tbase + (16u << 16), va);
        fold(vb, 0, 1, wt[1], cp[1], a0, b0, a1, b1, w0, w1);
        tmem_wait_ld_dep(va);
        tmem_ld16x256b_x8(tbase + (16u << 16) + 64, vb);
        fold(va, 1, 0, wt[0], cp[0], a2, b2, a3, b3, w2, w3);
        tmem_wait_ld_dep(vb);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty_lead + ab * 8);
        if (ew == 0 && lane == 0) RKV_GSTAMP(1, rt, 2);
        if (++ab == 2) { ab = 0; aph ^= 1; }
        fold(vb, 1, 1, wt[1], cp[1], a2, b2, a3, b3, w2, w3);
        if (ew == 0 && lane == 0) RKV_GSTAMP(1, rt, 3);
        ++rt;
        if constexpr (!kDiag) {
          // the quad's four threads hold disjoint columns of the same 4 rows:
          // reduce-scatter so that thread tq keeps row gq + 8 tq
          const float t0 = a0 + b0, t1 = a1 + b1, t2 = a2 + b2, t3 = a3 + b3;
          const bool u2 = (lane & 2) != 0, u1 = (lane & 1) != 0;
          const float k0 = (u2 ? t2 : t0) + __shfl_xor_sync(0xffffffffu, u2 ? t0 : t2, 2);
          const float k1 = (u2 ? t3 : t1) + __shfl_xor_sync(0xffffffffu, u2 ? t1 : t3, 2);
          const float rsum = (u1 ? k1 : k0) + __shfl_xor_sync(0xffffffffu, u1 ? k0 : k1, 1);
          // into the ring; the row-store warp adds the two column halves
          const uint32_t s = nx % kRowRing;
          mbar_wait(&row_empty[s], ((nx / kRowRing) & 1) ^ 1, abort, p.status);
          rowr[s * 512 + ch * 128 + q * 32 + gq + 8 * tq] = rsum;
          __syncwarp();
          if (lane == 0) mbar_arrive(&row_full[s]);
          ++nx;
        }
      };
      for (int t = 0; t < blk; ++t) tile(BoolTag<false>{}, t);
      tile(BoolTag<true>{}, blk);
      // ---- item end: column sums of block blk over the quad index gq (lane
      // bits 2-4), reduce-scattered so that lane l keeps columns 2l and 2l + 1
      // of each group, then the four lane quarters through shared memory
#pragma unroll
      for (int c = 0; c < 2; ++c) {
#pragma unroll
        for (int sft = 16, n = 8; sft >= 4; sft >>= 1, n >>= 1) {
          const bool up = (lane & sft) != 0;
#pragma unroll
          for (int k = 0; k < n; ++k) {
            const float send = up ? cp[c][k] : cp[c][k + n];
            const float keep = up ? cp[c][k + n] : cp[c][k];
            cp[c][k] = keep + __shfl_xor_sync(0xffffffffu, send, sft);
          }
        }
        float2* cx = colx + (ib * 4 + 2 * ch + c) * 4 * 32;
        cx[q * 32 + lane] = make_float2(cp[c][0], cp[c][1]);
      }
      named_bar_sync(4 + ch, 128);
      if (q == 0) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const float2* cx = colx + (ib * 4 + 2 * ch + c) * 4 * 32;
          float2 acc = cx[lane];
#pragma unroll
          for (int qq = 1; qq < 4; ++qq) {
            const float2 y = cx[qq * 32 + lane];
            acc.x += y.x;
            acc.y += y.y;
          }
          // this CTA's rows' share; the pair's other CTA writes the other slot
          *reinterpret_cast<float2*>(cs_u + (2 * blk + rank) * 256 + ch * 128 + c * 64 +
                                     2 * lane) = acc;
        }
      }
    }
  } else if (!kSym && warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int etid = threadIdx.x - 128;   // 0..511
    const int ew = warp - 4;              // epilogue warp 0..15
    const int cg = ew >> 2;               // 64-column group of the tile
    const int q = warp & 3;               // TMEM lane quarter
    const int gq = lane >> 2, tq = lane & 3;   // quad and thread within it
    const float* rho_ring = reinterpret_cast<const float*>(sm + L.rho);
    float* rowx = reinterpret_cast<float*>(sm + L.rowx);
    float* fin = reinterpret_cast<float*>(sm + L.fin);
    const uint32_t acc_empty_lead = kPair ? mapa(smem_u32(acc_empty), 0) : smem_u32(acc_empty);
    int ab = 0;
    uint32_t aph = 0;
    uint32_t rt = 0;   // rho tiles consumed so far
    for (int item = group_id; item < n_items; item += ngroups) {
      const int u = find_unit(p.item_off, p.num_units, item);
      const int blk = item_block<kSym>(p.item_off, u, item);
      const int64_t base = __ldg(&p.tok_off[u]);
      const int N = static_cast<int>(__ldg(&p.tok_off[u + 1]) - base);
      const int c = N - p.w;
      const int rbase = blk * C::kRowsPerItem + rank * 128;   // unit-local first row
      // Each thread accumulates 4 rows of its lane quarter (gq, gq + 8, gq + 16,
      // gq + 24) over its 16 columns of each 64-column group (8i + 2tq + {0,1}),
      // two partial values per row.
      constexpr float kInit = kMax ? -INFINITY : 0.f;
      float a0 = kInit, b0 = kInit, a1 = kInit, b1 = kInit;
      float a2 = kInit, b2 = kInit, a3 = kInit, b3 = kInit;
      const int ntiles = (N + C::kN - 1) / C::kN;
      for (int t = 0; t < ntiles; ++t, ++rt) {
        const int j0 = t * C::kN;
        const uint32_t rs_slot = rt % kRhoSlots;
        const float* rs = rho_ring + rs_slot * 256 + cg * 64 + 2 * tq;
        if (etid == 0) RKV_GSTAMP(1, rt, 0);
        mbar_wait(&acc_full[ab], aph, abort, p.status);
        mbar_wait(&rho_full[rs_slot], (rt / kRhoSlots) & 1, abort, p.status);
        if (etid == 0) RKV_GSTAMP(1, rt, 1);
        __syncwarp();
        tc_fence_after();
        // this thread's 16 column weights: 8 shared-memory reads per tile, 4x
        // fewer than one row per thread over all 64 columns would need
        float2 wt[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) wt[k] = *reinterpret_cast<const float2*>(rs + 8 * k);
        const uint32_t tbase =
            tmem + (static_cast<uint32_t>(q * 32) << 16) + ab * 256 + cg * 64;
        const int cw0 = j0 + cg * 64;                // first column of this warp's group
        const int rw0 = rbase + q * 32;              // first row of this warp's quarter
        const bool masked = ((rw0 < cw0 + 64) && (cw0 < rw0 + 32)) || (kMax && cw0 + 64 > N);
        const int dd = rw0 - cw0;                    // diagonal: column - row == dd
        const int jn = kMax ? N - cw0 : 64;          // first column past the unit
        constexpr uint32_t neutral = kMax ? 0xff800000u : 0u;   // -inf, or 0
        uint32_t v[32];
        // Masked groups (rare): the diagonal and, for the row max, the columns
        // past the unit are neutralised (-inf * rho is -inf or NaN, both
        // ignored by fmaxf).  h selects the 16-lane half of the quarter.
        auto patch = [&](int h) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int col = 8 * k + 2 * tq + (e & 1);
              const int row = 16 * h + gq + ((e >> 1) << 3);
              if (col - row == dd || col >= jn) v[4 * k + e] = neutral;
            }
        };
        auto fold = [&](float& pa, float& pb, float& qa, float& qb) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            if constexpr (kMax) {
              float x0, x1, y0, y1;
              mul2(x0, x1, __uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]), wt[k].x,
                   wt[k].y);
              mul2(y0, y1, __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]), wt[k].x,
                   wt[k].y);
              pa = fmaxf(pa, x0); pb = fmaxf(pb, x1); qa = fmaxf(qa, y0); qb = fmaxf(qb, y1);
            } else {
              fma2(pa, pb, __uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]), wt[k].x,
                   wt[k].y);
              fma2(qa, qb, __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]), wt[k].x,
                   wt[k].y);
            }
          }
        };
        tmem_ld16x256b_x8(tbase, v);                 // lanes 0-15 of the quarter
        tmem_wait_ld();
        if (etid == 0) RKV_GSTAMP(1, rt, 2);
        if (masked) patch(0);
        fold(a0, b0, a1, b1);
        tmem_ld16x256b_x8(tbase + (16u << 16), v);   // lanes 16-31
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {   // the accumulator is in registers: hand it back to the MMA
          if constexpr (kPair) mbar_arrive_cluster_relaxed(acc_empty_lead + ab * 8);
          else mbar_arrive(&acc_empty[ab]);
        }
        if (++ab == 2) { ab = 0; aph ^= 1; }
        if (masked) patch(1);
        fold(a2, b2, a3, b3);
        if (etid == 0) RKV_GSTAMP(1, rt, 3);
        __syncwarp();
        if (lane == 0) mbar_arrive(&rho_empty[rs_slot]);
      }
      // ---- item end: finish the rows over the quad (its four threads hold
      // disjoint columns), combine the four column groups, write m
      auto red = [](float x, float y) { return kMax ? fmaxf(x, y) : x + y; };
      float t0 = red(a0, b0), t1 = red(a1, b1), t2 = red(a2, b2), t3 = red(a3, b3);
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        t0 = red(t0, __shfl_xor_sync(0xffffffffu, t0, o));
        t1 = red(t1, __shfl_xor_sync(0xffffffffu, t1, o));
        t2 = red(t2, __shfl_xor_sync(0xffffffffu, t2, o));
        t3 = red(t3, __shfl_xor_sync(0xffffffffu, t3, o));
      }
      // thread tq of the quad owns row gq + 8 tq of the quarter
      float tot = tq == 0 ? t0 : tq == 1 ? t1 : tq == 2 ? t2 : t3;
      const int rl = q * 32 + gq + 8 * tq;           // row of this CTA's A block
      const int i = rbase + rl;
      if (cg > 0) rowx[(cg - 1) * 128 + rl] = tot;
      named_bar_sync(3, 512);
      if (cg == 0 && i < c) {
        const float rho_i = __ldg(&p.rho[__ldg(&p.rho_off[u]) + i]);
        if constexpr (kMax) {
          tot = fmaxf(fmaxf(tot, rowx[rl]), fmaxf(rowx[128 + rl], rowx[256 + rl]));
          p.m_dst[base + i] = rho_i * tot;
        } else {
          tot += (rowx[rl] + rowx[128 + rl]) + rowx[256 + rl];
          p.m_dst[base + i] = rho_i * tot / static_cast<float>(N - 1);
        }
      }
      __threadfence();
      named_bar_sync(3, 512);
      if (etid == 0) {
        const int nblk = __ldg(&p.item_off[u + 1]) - __ldg(&p.item_off[u]);
        const int done = atomicAdd(&p.unit_cnt[u], 1) + 1;
        *last_flag = done == nblk * (kPair ? 2 : 1);
      }
      named_bar_sync(3, 512);
      if (*last_flag) {
        __threadfence();
        // ---- token softmax over the unit's candidates (|m| <= 1: no max shift)
        float sum = 0.f;
        for (int ii = etid; ii < c; ii += 512) sum += ex2(__ldcg(&p.m_dst[base + ii]) * kLog2e);
        sum = warp_reduce_sum(sum);
        if (lane == 0) fin[ew] = sum;
        named_bar_sync(3, 512);
        float totl = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) totl += fin[k];
        const float inv = 1.f / totl;
        for (int ii = etid; ii < c; ii += 512)
          p.r_dst[base + ii] = ex2(__ldcg(&p.m_dst[base + ii]) * kLog2e) * inv;
        named_bar_sync(3, 512);
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

// One block, before the score kernel: the score chunks of every unit and their
// prefix, zeroed exchange counters and, for the GEMM, items per unit and their
// prefix, 256-aligned rho segment offsets, zeroed unit counters and (symmetric
// form, cs_off != null) the offsets of each unit's scratch.  A GEMM item is a
// block of candidate rows, or in the symmetric form any 256-key block of a unit
// that has candidates (its columns reach every candidate row).
__global__ void plan_kernel(const PlanParams pp) {
  __shared__ long long wsum[4][32];
  const int U = pp.U;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (U + nt - 1) / nt;
  const int u0 = min(U, tid * per), u1 = min(U, u0 + per);
  const bool gemm = pp.rows_per_item > 0;
  const bool sym = pp.cs_off != nullptr;
  const int64_t chunk_tok = static_cast<int64_t>(pp.tpc) * kTile;
  if (tid == 0) *pp.score_abort = 0;
  long long lc = 0, li = 0, lr = 0, ls = 0;   // this thread's chunks, items, rho, scratch
  for (int u = u0; u < u1; ++u) {
    const int64_t n = pp.tok_off[u + 1] - pp.tok_off[u];
    lc += (n + chunk_tok - 1) / chunk_tok;
    for (int e = 0; e < kScoreCnt; ++e) pp.score_cnt[u * kScoreCnt + e] = 0;
    if (gemm) {
      li += gemm_unit_items(n, n - pp.w, pp.rows_per_item, sym);
      lr += (n + kRhoAlign - 1) / kRhoAlign * kRhoAlign;
      ls += sym_scratch_floats(n, pp.w);
      pp.unit_cnt[u] = 0;
    }
  }
  // block exclusive scans
  long long x[4] = {lc, li, lr, ls};
  const int lane = tid & 31, wp = tid >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const long long y = __shfl_up_sync(0xffffffffu, x[k], o);
      if (lane >= o) x[k] += y;
    }
  }
  if (lane == 31)
    for (int k = 0; k < 4; ++k) wsum[k][wp] = x[k];
  __syncthreads();
  if (wp == 0) {
    long long z[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) z[k] = lane < (nt >> 5) ? wsum[k][lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const long long y = __shfl_up_sync(0xffffffffu, z[k], o);
        if (lane >= o) z[k] += y;
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) wsum[k][lane] = z[k];
  }
  __syncthreads();
  long long rc = x[0] - lc + (wp > 0 ? wsum[0][wp - 1] : 0);
  long long ri = x[1] - li + (wp > 0 ? wsum[1][wp - 1] : 0);
  long long rr = x[2] - lr + (wp > 0 ? wsum[2][wp - 1] : 0);
  long long rs = x[3] - ls + (wp > 0 ? wsum[3][wp - 1] : 0);
  for (int u = u0; u < u1; ++u) {
    const int64_t n = pp.tok_off[u + 1] - pp.tok_off[u];
    pp.chunk_off[u] = static_cast<int>(rc);
    const long long nc = (n + chunk_tok - 1) / chunk_tok;
    for (long long q = 0; q < nc; ++q) pp.chunk_unit[rc + q] = u;
    rc += nc;
    if (gemm) {
      pp.item_off[u] = static_cast<int>(ri);
      pp.rho_off[u] = rr;
      if (sym) pp.cs_off[u] = rs;
      ri += gemm_unit_items(n, n - pp.w, pp.rows_per_item, sym);
      rr += (n + kRhoAlign - 1) / kRhoAlign * kRhoAlign;
      rs += sym_scratch_floats(n, pp.w);
    }
  }
  if (u1 == U && u0 < u1) {
    pp.chunk_off[U] = static_cast<int>(rc);
    if (gemm) {
      pp.item_off[U] = static_cast<int>(ri);
      pp.rho_off[U] = rr;
      if (sym) pp.cs_off[U] = rs;
    }
  }
  if (U == 0 && tid == 0) {
    pp.chunk_off[0] = 0;
    if (gemm) {
      pp.item_off[0] = 0;
      pp.rho_off[0] = 0;
      if (sym) pp.cs_off[0] = 0;
    }
  }
}

// Symmetric form, after the GEMM: one CTA per unit.  Row i of block a (i < c)
// gets the two CTAs' column sums of block a, then the row sums of the slots
// (a, b) for b = a + 1 .. nb - 1 in block order, is scaled by rho_i / (N - 1),
// and the token softmax follows.  A thread takes 4 consecutive rows (one
// block) and reads one aligned float4 per slot.
constexpr int kFinishThreads = 512;
__global__ void __launch_bounds__(kFinishThreads)
    sym_finish_kernel(const int64_t* __restrict__ tok_off, int U, int w,
                      const float* __restrict__ rho, const int64_t* __restrict__ rho_off,
                      const float* __restrict__ cs, const int64_t* __restrict__ cs_off,
                      float* m_dst, float* r_dst) {
  __shared__ float wred[kFinishThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, wp = tid >> 5;
  for (int u = blockIdx.x; u < U; u += gridDim.x) {
    const int64_t base = tok_off[u];
    const int N = static_cast<int>(tok_off[u + 1] - base);
    const int c = N - w;
    if (c <= 0) continue;
    const int nb = (N + 255) / 256;
    const float* rho_u = rho + rho_off[u];
    const float* cs_u = cs + cs_off[u];
    const float inv_nm1 = 1.f / static_cast<float>(N - 1);
    float esum = 0.f;
    for (int r0 = 4 * tid; r0 < c; r0 += 4 * kFinishThreads) {
      const int a = r0 >> 8, lr = r0 & 255;
      const float4 d0 = __ldcs(reinterpret_cast<const float4*>(cs_u + (2 * a) * 256 + lr));
      const float4 d1 = __ldcs(reinterpret_cast<const float4*>(cs_u + (2 * a + 1) * 256 + lr));
      float4 acc = make_float4(d0.x + d1.x, d0.y + d1.y, d0.z + d1.z, d0.w + d1.w);
      const float* seg = cs_u + 512 * static_cast<int64_t>(nb) +
                         256 * (static_cast<int64_t>(a) * (nb - 1) -
                                static_cast<int64_t>(a) * (a - 1) / 2) + lr;
#pragma unroll 4
      for (int b = a + 1; b < nb; ++b) {
        const float4 y = __ldcs(reinterpret_cast<const float4*>(seg + (b - a - 1) * 256));
        acc.x += y.x;
        acc.y += y.y;
        acc.z += y.z;
        acc.w += y.w;
      }
      const float part[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = r0 + e;
        if (i < c) {
          const float m = rho_u[i] * part[e] * inv_nm1;
          m_dst[base + i] = m;
          esum += ex2(m * kLog2e);
        }
      }
    }
    // token softmax (|m| <= 1: no max shift); each thread rereads its own rows
    esum = warp_reduce_sum(esum);
    if (lane == 0) wred[wp] = esum;
    __syncthreads();
    float tot = 0.f;
#pragma unroll
    for (int k = 0; k < kFinishThreads / 32; ++k) tot += wred[k];
    const float inv = 1.f / tot;
    for (int r0 = 4 * tid; r0 < c; r0 += 4 * kFinishThreads)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = r0 + e;
        if (i < c) r_dst[base + i] = ex2(m_dst[base + i] * kLog2e) * inv;
      }
    __syncthreads();   // wred is reused by the next unit
  }
}

}  // namespace

#ifdef RKV_TRACE
extern "C" int rkv_debug_gemm_trace(void* dst, size_t bytes) {
  return static_cast<int>(cudaMemcpyFromSymbol(dst, g_gemm_trace, bytes));
}
#endif

namespace {
// The symmetric form exists for CTA pairs and the row mean only (its tiles
// are 256 x 256 and the column sums are added linearly).
void* gemm_fn(bool pair, bool rowmax, bool sym) {
  if (sym) return reinterpret_cast<void*>(&redundancy_gemm_kernel<true, false, true>);
  if (pair) return rowmax ? reinterpret_cast<void*>(&redundancy_gemm_kernel<true, true, false>)
                          : reinterpret_cast<void*>(&redundancy_gemm_kernel<true, false, false>);
  return rowmax ? reinterpret_cast<void*>(&redundancy_gemm_kernel<false, true, false>)
                : reinterpret_cast<void*>(&redundancy_gemm_kernel<false, false, false>);
}
}  // namespace

cudaError_t gemm_configure(bool pair, bool rowmax, bool sym) {
  const int smem = (pair ? gemm_layout<true>().total : gemm_layout<false>().total) + 1024;
  return cudaFuncSetAttribute(gemm_fn(pair, rowmax, sym),
                              cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
}

int gemm_max_ctas(bool pair, bool rowmax, bool sym) {
  const int smem = (pair ? gemm_layout<true>().total : gemm_layout<false>().total) + 1024;
  void* f = gemm_fn(pair, rowmax, sym);
  int dev = 0, nsm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  if (!pair) {
    int per = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, f, gemm_threads(sym), smem) !=
        cudaSuccess) {
      cudaGetLastError();
      return 0;
    }
    return per * nsm;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * nsm, 1, 1);
  cfg.blockDim = dim3(gemm_threads(sym), 1, 1);
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

cudaError_t launch_plan(const PlanParams& pp, cudaStream_t st) {
  plan_kernel<<<1, 1024, 0, st>>>(pp);
  return cudaGetLastError();
}

cudaError_t launch_sym_finish(const GemmParams& p, int nsm, cudaStream_t st) {
  int grid = nsm * 4;
  if (grid > p.num_units) grid = p.num_units;
  sym_finish_kernel<<<grid, kFinishThreads, 0, st>>>(p.tok_off, p.num_units, p.w, p.rho,
                                                     p.rho_off, p.cs, p.cs_off, p.m_dst,
                                                     p.r_dst);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const CUtensorMap& amap, const CUtensorMap& bmap, const GemmParams& p,
                        bool pair, bool rowmax, bool sym, int nctas, cudaStream_t st) {
  const int smem = (pair ? gemm_layout<true>().total : gemm_layout<false>().total) + 1024;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nctas, 1, 1);
  cfg.blockDim = dim3(gemm_threads(sym), 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = pair ? 2 : 1;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = pair ? 1 : 0;
  if (sym)
    return cudaLaunchKernelEx(&cfg, redundancy_gemm_kernel<true, false, true>, amap, bmap, p);
  if (pair) {
    if (rowmax)
      return cudaLaunchKernelEx(&cfg, redundancy_gemm_kernel<true, true, false>, amap, bmap, p);
    return cudaLaunchKernelEx(&cfg, redundancy_gemm_kernel<true, false, false>, amap, bmap, p);
  }
  if (rowmax)
    return cudaLaunchKernelEx(&cfg, redundancy_gemm_kernel<false, true, false>, amap, bmap, p);
  return cudaLaunchKernelEx(&cfg, redundancy_gemm_kernel<false, false, false>, amap, bmap, p);
}

}  // namespace rkv
