// Score kernel: importance (R-KV 重要性打分) and, in closed-form mode, the
// redundancy row mean (R-KV 冗余打分) for every unit, with K read from HBM once.
//
// Work split.  Every unit is cut into chunks of `tpc` tiles of 128 tokens;
// chunk g of the whole batch goes to CTA g % P of a persistent grid of P CTAs
// (one per SM, cooperative launch, so all CTAs are resident together).  A CTA
// walks its chunks x_0, x_1, ... (x_k = blockIdx + k P) one step per chunk:
//
//   step k:  P1(x_k)   stream x_k's K tiles (TMA), logits z = K_tile . Q^T on
//                      tcgen05 (M = 128 tokens, N = RP query rows) into tensor
//                      memory buffer k % 2, per-thread online softmax
//                      statistics, key norms (rho = 1/||k||, closed form also
//                      U = sum_j rho_j k_j);
//            pub(x_k)  the chunk's (max, sum) per query row [and U] go to a
//                      global exchange slot; a release increment of the unit's
//                      first counter announces them;
//            W(x_k-1)  wait until every chunk of x_k-1's unit has announced,
//                      merge their statistics in chunk order (identical in every
//                      CTA of the unit);
//            P2(x_k-1) abar_j = sum_rows 2^(y - M_row) / L_row from buffer
//                      (k-1) % 2, which is then released to the MMA; closed form:
//                      m_j from the K tiles read again (L2) and U;
//            pubS(x_k-1) the chunk's sum of abar [and of exp(m)] over the
//                      candidates, announced on the unit's second counter;
//            WS(x_k-2) wait for those sums of x_k-2's unit, and write its a [r, m].
//
// The K stream of x_k therefore overlaps the exchanges of x_k-1 and x_k-2.
// Progress: a CTA announces x_k before it waits for x_k-1.  If a unit spans at
// most 2P chunks, each wait depends only on announcements that come after waits
// of strictly smaller chunk index (pub(x) follows W(x - 2P) and WS(x - 2P) in its
// CTA), so every wait ends; the host keeps units within 2P chunks.  Every wait
// is bounded: on timeout the CTA records it in the status word and in the
// call's abort word, raises its own abort flag and stops working; CTAs waiting
// on other CTAs see the abort word and give up too.
//
// Query rows: RP = 16 or 32 padded rows per launch (G*w real rows).  More than
// 32 rows run as several launches over row groups of 32; each adds its rows'
// probabilities to a, and the last one normalises and computes the redundancy
// part.
//
// Warp roles (512 threads; thread = token row of a tile, tensor-memory lane
// quarter = warp % 4), each group running on its own so that the K stream
// never waits for an exchange:
//   warp 0      TMA producer;
//   warp 1      MMA issuer and tensor-memory owner;
//   warps 4-7   pass 1: online statistics of every query row, announced per
//               chunk (no waits on other CTAs);
//   warps 8-11  W, merge and pass 2 of x_k-1, then a of x_k-2;
//   warps 12-15 norms: rho (GEMM form) or rho and U, then m and r (closed form).
// Only a tensor-memory buffer couples passes 1 and 2: pass 1 of x_k+1 reuses
// the buffer that pass 2 of x_k-1 releases.
#include "ptx.cuh"
#include "rkv_internal.cuh"

namespace rkv {
namespace {

constexpr float kNegBig = -1e30f;  // initial running max (finite: no inf - inf)
constexpr int kBufCols = 256;      // tensor-memory columns per logit buffer
constexpr uint64_t kDrainNs = 200000000ull;   // teardown wait for copies in flight

#ifdef RKV_TRACE
// Optional phase trace (build with -DRKV_TRACE): globaltimer stamps of the
// consumer threads' step phases, for the first kTrSteps steps of each CTA.
constexpr int kTrCtas = 160, kTrSteps = 32, kTrSlots = 16;
__device__ unsigned long long g_score_trace[kTrCtas * kTrSteps * kTrSlots];
#define RKV_STAMP(k, slot)                                                               \
  do {                                                                                   \
    if (ctid == 0 && (k) < kTrSteps && blockIdx.x < kTrCtas)                             \
      g_score_trace[(blockIdx.x * kTrSteps + (k)) * kTrSlots + (slot)] = globaltimer_ns(); \
  } while (0)
constexpr int kTtCtas = 4, kTtSteps = 16;
__device__ unsigned long long g_tile_trace[kTtCtas * kTtSteps * 16 * 4];
#define RKV_TSTAMP(k, t, slot)                                                              \
  do {                                                                                      \
    if (ctid == 0 && (k) < kTtSteps && blockIdx.x < kTtCtas && (t) < 16)                    \
      g_tile_trace[((blockIdx.x * kTtSteps + (k)) * 16 + (t)) * 4 + (slot)] = globaltimer_ns(); \
  } while (0)
#define RKV_CLK_BEGIN(var) const long long var = clock64()
#define RKV_CLK_ADD(acc, var) acc += clock64() - var
#define RKV_STORE(k, slot, val)                                                          \
  do {                                                                                   \
    if (ctid == 0 && (k) < kTrSteps && blockIdx.x < kTrCtas)                             \
      g_score_trace[(blockIdx.x * kTrSteps + (k)) * kTrSlots + (slot)] = (val);          \
  } while (0)
#else
#define RKV_STAMP(k, slot) do { } while (0)
#define RKV_TSTAMP(k, t, slot) do { } while (0)
#define RKV_CLK_BEGIN(var) do { } while (0)
#define RKV_CLK_ADD(acc, var) do { } while (0)
#define RKV_STORE(k, slot, val) do { } while (0)
#endif

struct Chunk {
  int g;          // global chunk index, -1 for none
  int u;          // unit
  int64_t base;   // first row of the unit in K
  int n, c;       // N, N - w
  int start;      // first token of the chunk
  int len;        // tokens in the chunk
  int nt;         // tiles in the chunk
  int g0, nch;    // first chunk of the unit, chunks of the unit
};

__device__ __forceinline__ Chunk chunk_info(const ScoreParams& p, int g) {
  Chunk h;
  h.g = g;
  const int u = __ldg(&p.chunk_unit[g]);
  h.u = u;
  h.g0 = __ldg(&p.chunk_off[u]);
  h.nch = __ldg(&p.chunk_off[u + 1]) - h.g0;
  h.base = __ldg(&p.tok_off[u]);
  h.n = static_cast<int>(__ldg(&p.tok_off[u + 1]) - h.base);
  h.c = h.n - p.w;
  h.start = (g - h.g0) * p.tpc * kTile;
  h.len = min(p.tpc * kTile, h.n - h.start);
  h.nt = (h.len + kTile - 1) / kTile;
  return h;
}

__device__ __forceinline__ Chunk no_chunk() {
  Chunk h = {};
  h.g = -1;
  return h;
}

__device__ __forceinline__ int ld_acquire_gpu(const int* a) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}

// One thread: wait until *cnt >= target.  Gives up at once if this CTA has
// aborted or another CTA of this call has given up (the call's abort word),
// and after `limit` ns itself, recording the timeout in the status word and
// in the abort word.
__device__ bool wait_count(const int* cnt, int target, volatile int* abort, int* status,
                           int* abort_all, uint64_t limit) {
  if (ld_acquire_gpu(cnt) >= target) return true;
  if (*abort) return false;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    __nanosleep(64);
    if (ld_acquire_gpu(cnt) >= target) return true;
    if ((n & 15u) == 0) {
      if (*abort) return false;
      if (*reinterpret_cast<volatile int*>(abort_all) != 0) {
        *abort = 1;
        return false;
      }
      if (globaltimer_ns() - t0 > limit) {
        *abort = 1;
        atomicOr(status, kStatusTimeout);
        atomicExch(abort_all, 1);
        return false;
      }
    }
  }
}

// Teardown: wait (bounded, regardless of an abort) for the phase of parity
// `par` of a barrier whose completion is already under way (a copy or an MMA
// commit issued earlier).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t par) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, par))
    if (globaltimer_ns() - t0 > kDrainNs) return;
}

// Merge two (max, sum) softmax statistics in the log2 domain.
__device__ __forceinline__ void merge_stat(float& m, float& s, float om, float os) {
  const float M = fmaxf(m, om);
  s = __fadd_rn(__fmul_rn(s, ex2(m - M)), __fmul_rn(os, ex2(om - M)));
  m = M;
}

// Merge each of RH per-lane statistics over the 32 lanes of the warp.  A
// transposed butterfly: at each level a lane keeps half of its rows and sends
// the other half to its partner.  Afterwards m[0], s[0] of lane l hold row
// l % RH merged over all lanes.
template <int RH>
__device__ __forceinline__ void lane_merge(float (&m)[RH], float (&s)[RH], int lane) {
#pragma unroll
  for (int sh = RH / 2; sh >= 1; sh >>= 1) {
    const bool up = (lane & sh) != 0;
#pragma unroll
    for (int i = 0; i < sh; ++i) {
      const float sm_ = up ? m[i] : m[i + sh];
      const float ss_ = up ? s[i] : s[i + sh];
      const float km = up ? m[i + sh] : m[i];
      const float ks = up ? s[i + sh] : s[i];
      const float om = __shfl_xor_sync(0xffffffffu, sm_, sh);
      const float os = __shfl_xor_sync(0xffffffffu, ss_, sh);
      m[i] = km;
      s[i] = ks;
      merge_stat(m[i], s[i], om, os);
    }
  }
#pragma unroll
  for (int sh = RH; sh < 32; sh <<= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, m[0], sh);
    const float os = __shfl_xor_sync(0xffffffffu, s[0], sh);
    merge_stat(m[0], s[0], om, os);
  }
}

// Logits of one tile as the 16x256b shape reads them: for lanes 16h .. 16h+15
// of the warp's quarter, thread t gets v[4i + e] = (token t/4, row 8i + 2(t%4) + e)
// and v[4i + 2 + e] = (token t/4 + 8, the same row), i < RP / 8, e < 2.
template <int RP>
__device__ __forceinline__ void tmem_ld_tile(uint32_t taddr, uint32_t (&v)[RP / 2]) {
  if constexpr (RP == 16) tmem_ld16x256b_x2(taddr, v);
  else tmem_ld16x256b_x4(taddr, v);
}

// Merge per-lane statistics of the NR query rows a lane holds over the 8 lanes
// that hold the same rows (lane bits 2, 3, 4) with a transposed butterfly.
// Afterwards slot s (returned) of the lane's rows is merged over all lanes in
// m[0], s[0]; for NR = 4 two lanes (bit 2) end with the same row.
template <int NR>
__device__ __forceinline__ int quad_rows_merge(float (&m)[NR], float (&sx)[NR], int lane) {
  int slot = 0, half = NR / 2, bit = 16;
#pragma unroll
  for (int lv = 0; (NR >> lv) > 1; ++lv, half >>= 1, bit >>= 1) {
    const bool up = (lane & bit) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float sm_ = up ? m[i] : m[i + half];
      const float ss_ = up ? sx[i] : sx[i + half];
      const float km = up ? m[i + half] : m[i];
      const float ks = up ? sx[i + half] : sx[i];
      const float om = __shfl_xor_sync(0xffffffffu, sm_, bit);
      const float os = __shfl_xor_sync(0xffffffffu, ss_, bit);
      m[i] = km;
      sx[i] = ks;
      merge_stat(m[i], sx[i], om, os);
    }
    if (up) slot += half;
  }
#pragma unroll
  for (; bit >= 4; bit >>= 1) {   // lane bits not used by the halving above
    const float om = __shfl_xor_sync(0xffffffffu, m[0], bit);
    const float os = __shfl_xor_sync(0xffffffffu, sx[0], bit);
    merge_stat(m[0], sx[0], om, os);
  }
  return slot;
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

// Squared norm of a row, eight partial sums added in a fixed tree.
__device__ __forceinline__ float row_norm2(const uint4 (&xs)[16]) {
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
  return ((nq[0] + nq[1]) + (nq[2] + nq[3])) + ((nq[4] + nq[5]) + (nq[6] + nq[7]));
}

template <int RP, bool CLOSED>
__global__ void __launch_bounds__(score_threads(CLOSED), 1)
    score_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                 const ScoreParams p) {
  constexpr int XS = score_xs(RP, CLOSED);  // floats of a chunk's exchange slot
  constexpr int CHT = score_chunk_tokens(RP);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  const int NS = p.nstages;
  const ScoreLayout L = score_layout(RP, CLOSED, NS);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = static_cast<int>(gridDim.x);
  const int b0 = static_cast<int>(blockIdx.x);
  // the redundancy side (norms, U, m) runs in the last row-group launch only
  const bool red = p.final_pass != 0;
  // announcements per chunk on each counter: the statistics (and, closed form,
  // the norm warps' U), then the sum of abar (and of exp(m))
  const int nann = (CLOSED && red) ? 2 : 1;

  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* empty = full + NS;
  uint64_t* tready = empty + NS;   // [2][16] logits of tile t of buffer b are in TMEM
  uint64_t* tfree = tready + 32;   // [2] pass-2 warps are done with buffer b
  uint64_t* qfull = tfree + 2;     // [2]
  uint64_t* qempty = qfull + 2;    // [2]
  uint64_t* mdone = qempty + 2;    // teardown: every MMA has completed
  uint64_t* sfull = mdone + 1;     // [2] a smem slot holds a chunk's abar (and m)
  uint64_t* sfree = sfull + 2;     // [2] the output warps are done with a slot
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L.slot);
  volatile int* abort = reinterpret_cast<volatile int*>(sm + L.flags);
  int8_t* lastp = reinterpret_cast<int8_t*>(sm + L.issued);   // [NS + 2] parity of the last copy

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], red ? 1 + 4 : 1);  // MMA thread [+ 4 norm warps]
    }
    for (int k = 0; k < 32; ++k) mbar_init(&tready[k], 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfree[b], score_threads(CLOSED) == 640 ? 8 : 4);   // pass-2 warps
      mbar_init(&qfull[b], 1);
      mbar_init(&qempty[b], 1);
    }
    mbar_init(mdone, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sfull[b], (CLOSED && red) ? 2 : 1);   // pass-2 warps [+ norm warps]
      mbar_init(&sfree[b], 1);
    }
    for (int s = 0; s < NS + 2; ++s) lastp[s] = -1;
    *abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < RP)   // window step t of query row r = g * w + t of the group
    reinterpret_cast<int*>(sm + L.rowt)[threadIdx.x] = (p.row0 + threadIdx.x) % p.w;
  if (warp == 1) {
    tmem_alloc<1>(tmem_slot, kTmemColsTotal);
    tmem_relinquish<1>();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // bit r set for real query rows of this launch's group; window step of a row
  const uint32_t rmask = p.Rg >= 32 ? 0xffffffffu : ((1u << p.Rg) - 1u);
  int* row_t = reinterpret_cast<int*>(sm + L.rowt);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&kmap);
      prefetch_tmap(&qmap);
      const uint64_t keep = policy_evict_normal(), drop = policy_evict_first();
      int stage = 0;
      uint32_t ph = 0;
      Chunk prev = no_chunk();
      auto load_tiles = [&](const Chunk& h, uint64_t pol) {
        for (int t = 0; t < h.nt; ++t) {
          if (mbar_wait(&empty[stage], ph ^ 1, abort, p.status)) {
            uint8_t* dst = sm + L.stages + stage * kTileBytes;
            const int y = static_cast<int>(h.base + h.start + kTile * t);
            mbar_arrive_expect_tx(&full[stage], kTileBytes);
            tma_load_2d(dst, &kmap, &full[stage], 0, y, pol);
            tma_load_2d(dst + kTileBytes / 2, &kmap, &full[stage], 64, y, pol);
            lastp[stage] = static_cast<int8_t>(ph);
          }
          if (++stage == NS) { stage = 0; ph ^= 1; }
        }
      };
      for (int k = 0;; ++k) {
        const int g = b0 + k * P;
        const bool have = g < p.total_chunks;
        Chunk cur = have ? chunk_info(p, g) : no_chunk();
        if (have) {
          const int qb = k & 1;
          if (mbar_wait(&qempty[qb], ((k >> 1) & 1) ^ 1, abort, p.status)) {
            uint8_t* qd = sm + L.q + qb * RP * 256;
            const int yq = cur.u * p.R + p.row0;
            mbar_arrive_expect_tx(&qfull[qb], RP * 256);
            tma_load_2d(qd, &qmap, &qfull[qb], 0, yq, keep);
            tma_load_2d(qd + RP * 128, &qmap, &qfull[qb], 64, yq, keep);
            lastp[NS + qb] = static_cast<int8_t>((k >> 1) & 1);
          }
          // read once, or kept for the closed form's second read
          load_tiles(cur, (CLOSED && red) ? keep : drop);
        }
        if (CLOSED && red && prev.g >= 0) load_tiles(prev, drop);   // pass 2 of x_k-1
        if (!have) break;
        prev = cur;
      }
      // teardown: every copy issued has landed before the CTA exits
      for (int s = 0; s < NS + 2; ++s)
        if (lastp[s] >= 0) drain_wait(s < NS ? &full[s] : &qfull[s - NS], lastp[s]);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, RP);
      int stage = 0;
      uint32_t ph = 0;
      Chunk prev = no_chunk();
      for (int k = 0;; ++k) {
        const int g = b0 + k * P;
        const bool have = g < p.total_chunks;
        Chunk cur = have ? chunk_info(p, g) : no_chunk();
        if (have) {
          const int qb = k & 1, buf = k & 1;
          bool ok = mbar_wait(&qfull[qb], (k >> 1) & 1, abort, p.status);
          // buffer k % 2 was released by pass 2 of x_k-2
          ok = mbar_wait(&tfree[buf], ((k >> 1) & 1) ^ 1, abort, p.status) && ok;
          const uint32_t qaddr = smem_u32(sm + L.q + qb * RP * 256);
          for (int t = 0; t < cur.nt; ++t) {
            const bool go = mbar_wait(&full[stage], ph, abort, p.status) && ok;
            tc_fence_after();
            if (go) {
              const uint32_t kaddr = smem_u32(sm + L.stages + stage * kTileBytes);
              const uint32_t d = tmem + buf * kBufCols + t * RP;
#pragma unroll
              for (int kq = 0; kq < 8; ++kq) {
                const uint32_t ko = (kq >> 2) * (kTileBytes / 2) + (kq & 3) * 32;
                const uint32_t qo = (kq >> 2) * (RP * 128) + (kq & 3) * 32;
                mma_bf16<1>(d, desc_kmajor_sw128(kaddr + ko), desc_kmajor_sw128(qaddr + qo),
                            idesc, kq > 0);
              }
              mma_commit(&empty[stage]);
              mma_commit(&tready[buf * 16 + t]);
            } else {
              mbar_arrive(&empty[stage]);
            }
            if (++stage == NS) { stage = 0; ph ^= 1; }
          }
          if (ok) mma_commit(&qempty[qb]);
          else mbar_arrive(&qempty[qb]);
        }
        if (CLOSED && red && prev.g >= 0) {
          // pass-2 tiles feed only the norm warps: keep the ring's arrival count
          for (int t = 0; t < prev.nt; ++t) {
            mbar_wait(&full[stage], ph, abort, p.status);
            mbar_arrive(&empty[stage]);
            if (++stage == NS) { stage = 0; ph ^= 1; }
          }
        }
        if (!have) break;
        prev = cur;
      }
      // teardown: all MMAs (and their commits) are complete before TMEM is freed
      mma_commit(mdone);
      drain_wait(mdone, 0);
    }
    __syncwarp();
  } else if (warp == 2 || warp == 3) {
    // ---------------------------------------------- output warps (final pass)
    // chunk x_j once its abar (and m) sit in smem slot j % 2: wait for the
    // sums of every chunk of its unit, write a (and r, m), free the slot
    if (red) {
      const int ctid = threadIdx.x - 64;     // 0..63
      float* abuf = reinterpret_cast<float*>(sm + L.abuf);   // [2 slots][CHT]
      float* marr = reinterpret_cast<float*>(sm + L.marr);   // [2 slots][CHT]
      float* osum = reinterpret_cast<float*>(sm + L.osum);   // [2] inverse sums
      for (int k = 0;; ++k) {
        const int g = b0 + k * P;
        if (g >= p.total_chunks) break;
        const Chunk h = chunk_info(p, g);
        const int slot = k & 1;
        mbar_wait(&sfull[slot], (k >> 1) & 1, abort, p.status);
        if (warp == 2) {
          if (lane == 0)
            wait_count(&p.cnt[h.u * kScoreCnt + 2 * p.group + 1], nann * h.nch, abort, p.status,
                       p.abort_all, p.wait_ns);
          __syncwarp();
          // sums over the unit's chunks (and earlier row groups), fixed order
          float sa = 0.f, se = 0.f;
          for (int q = lane; q < h.nch; q += 32) {
            const float* xi = p.xsum + static_cast<int64_t>(h.g0 + q) * (2 * kScoreMaxGroups);
            float x = 0.f;
            for (int gq = 0; gq <= p.group; ++gq) x += __ldcg(xi + 2 * gq);
            sa += x;
            if (CLOSED) se += __ldcg(xi + 2 * p.group + 1);
          }
          sa = warp_reduce_sum(sa);
          se = warp_reduce_sum(se);
          if (lane == 0) {
            osum[0] = sa > 0.f ? 1.f / sa : 0.f;
            osum[1] = se > 0.f ? 1.f / se : 0.f;
          }
        }
        named_bar_sync(4, 64);
        RKV_STAMP(k, 5);
        const float inv_sa = osum[0], inv_se = osum[1];
        const float* ab = abuf + slot * CHT;
        const float* ma = marr + slot * CHT;
        for (int i = ctid; i < h.len; i += 64) {
          const int j = h.start + i;
          const int64_t gi = h.base + j;
          if (j < h.c) {
            float x = ab[i];
            if (p.group > 0) x = p.a_out[gi] + x;
            p.a_out[gi] = x * inv_sa;
            if constexpr (CLOSED) {
              const float m = ma[i];
              p.r_out[gi] = ex2(m * kLog2e) * inv_se;
              if (p.m_out) p.m_out[gi] = m;
            }
          } else {
            p.a_out[gi] = 0.f;
            p.r_out[gi] = 0.f;   // the redundancy GEMM writes the candidates' r and m
            if (p.m_out) p.m_out[gi] = 0.f;
          }
        }
        named_bar_sync(4, 64);
        RKV_STAMP(k, 6);
        if (ctid == 0) mbar_arrive(&sfree[slot]);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------------------------------------- statistics warps (pass 1)
    // thread = 4 tokens x NR query rows of a tile (16x256b loads); no global waits
    constexpr int NR = RP / 4;               // query rows a thread holds
    const int ctid = threadIdx.x - 128;      // 0..127
    const int q4 = warp & 3;                 // tensor-memory lane quarter
    const int qd = lane >> 2, tq = lane & 3;
    float* red1 = reinterpret_cast<float*>(sm + L.red1);   // [4 quarters][RP][2]
    uint32_t tph = 0;   // phase bits of tready[32]
    const bool all_real = p.Rg >= RP;
    int g = b0;
    Chunk cur = g < p.total_chunks ? chunk_info(p, g) : no_chunk();
    for (int k = 0; cur.g >= 0; ++k) {
      const int buf = k & 1;
      RKV_STAMP(k, 0);
      float st_m[NR], st_s[NR];
#pragma unroll
      for (int q = 0; q < NR; ++q) { st_m[q] = kNegBig; st_s[q] = 0.f; }
#ifdef RKV_TRACE
      long long c_ready = 0, c_tw = 0;
      const long long c_loop0 = clock64();
#endif
      for (int t = 0; t < cur.nt; ++t) {
        const int bi = buf * 16 + t;
        RKV_TSTAMP(k, t, 0);
        RKV_CLK_BEGIN(cr0);
        mbar_wait(&tready[bi], (tph >> bi) & 1u, abort, p.status);
        RKV_CLK_ADD(c_ready, cr0);
        RKV_TSTAMP(k, t, 1);
        tph ^= 1u << bi;
        __syncwarp();
        tc_fence_after();
        const int t0 = cur.start + kTile * t;
        const bool inside = t0 + kTile <= cur.c;   // no causal limit or end in this tile
        uint32_t v[2][RP / 2];
        RKV_CLK_BEGIN(cw0);
#pragma unroll
        for (int h = 0; h < 2; ++h)
          tmem_ld_tile<RP>(tmem + (static_cast<uint32_t>(q4 * 32 + 16 * h) << 16) +
                               buf * kBufCols + t * RP, v[h]);
        tmem_wait_ld();
        RKV_CLK_ADD(c_tw, cw0);
        RKV_TSTAMP(k, t, 2);
        // y = log2-scaled logits (in place of the raw ones), -inf where masked
        // (padding row, beyond N, causal); the thread's tokens are
        // qd, qd + 8 (h = 0) and 16 + qd, 24 + qd (h = 1) of the quarter.  A
        // tile inside the candidates with every query row real needs no mask.
        if (inside && all_real) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int x = 0; x < RP / 2; ++x)
              v[h][x] = __float_as_uint(__uint_as_float(v[h][x]) * p.scale_log2);
        } else {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int ja = t0 + q4 * 32 + 16 * h + qd, jb = ja + 8;
#pragma unroll
            for (int i = 0; i < RP / 8; ++i)
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int r = 8 * i + 2 * tq + e;
                const bool real = ((rmask >> r) & 1u) != 0;
                const bool va = real && (inside || (ja < cur.n && ja <= cur.c + row_t[r]));
                const bool vb = real && (inside || (jb < cur.n && jb <= cur.c + row_t[r]));
                v[h][4 * i + e] = __float_as_uint(
                    va ? __uint_as_float(v[h][4 * i + e]) * p.scale_log2 : -INFINITY);
                v[h][4 * i + 2 + e] = __float_as_uint(
                    vb ? __uint_as_float(v[h][4 * i + 2 + e]) * p.scale_log2 : -INFINITY);
              }
          }
        }
        // online statistics, one update per row and tile (no branches): the
        // running max takes the tile's max over the thread's four tokens
#pragma unroll
        for (int i = 0; i < RP / 8; ++i)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int q = 2 * i + e;
            const float y0 = __uint_as_float(v[0][4 * i + e]);
            const float y1 = __uint_as_float(v[0][4 * i + 2 + e]);
            const float y2 = __uint_as_float(v[1][4 * i + e]);
            const float y3 = __uint_as_float(v[1][4 * i + 2 + e]);
            const float mn = fmaxf(st_m[q], fmaxf(fmaxf(y0, y1), fmaxf(y2, y3)));
            st_s[q] = fmaf(st_s[q], ex2(st_m[q] - mn),
                           (ex2(y0 - mn) + ex2(y1 - mn)) + (ex2(y2 - mn) + ex2(y3 - mn)));
            st_m[q] = mn;
          }
        RKV_TSTAMP(k, t, 3);
      }
#ifdef RKV_TRACE
      RKV_STORE(k, 7, c_ready);
      RKV_STORE(k, 8, c_tw);
      RKV_STORE(k, 15, clock64() - c_loop0);
#endif
      // the next chunk's bookkeeping loads overlap the merge below
      const int gn = g + P;
      const Chunk nxt = gn < p.total_chunks ? chunk_info(p, gn) : no_chunk();
      RKV_STAMP(k, 11);
      const int slot = quad_rows_merge<NR>(st_m, st_s, lane);
      {
        const int r = 8 * (slot >> 1) + 2 * tq + (slot & 1);
        if (NR == 8 || (lane & 4) == 0) {
          red1[(q4 * RP + r) * 2 + 0] = st_m[0];
          red1[(q4 * RP + r) * 2 + 1] = st_s[0];
        }
      }
      named_bar_sync(1, 128);
      float* xs_out = p.xstat + static_cast<int64_t>(cur.g) * XS;
      if (ctid < RP) {
        float m = kNegBig, sx = 0.f;
        for (int q = 0; q < 4; ++q)
          merge_stat(m, sx, red1[(q * RP + ctid) * 2], red1[(q * RP + ctid) * 2 + 1]);
        xs_out[2 * ctid] = m;
        xs_out[2 * ctid + 1] = sx;
      }
      named_bar_sync(1, 128);
      if (ctid == 0 && cur.g != p.drop_chunk) {
        __threadfence();
        atomicAdd(&p.cnt[cur.u * kScoreCnt + 2 * p.group], 1);
      }
      RKV_STAMP(k, 1);
      g = gn;
      cur = nxt;
    }
  } else if ((warp >= 8 && warp < 12) || warp >= 16) {
    // ---------------------------------------------- pass-2 warps
    // step k: merge the statistics of x_k-1 and turn its logits into abar.
    // NPAR sets of four warps (warps 8-11 [and 16-19]) take alternate tiles.
    constexpr int NPAR = (score_threads(CLOSED) - 512) / 128 + 1;
    constexpr int NP2 = 128 * NPAR;          // pass-2 threads
    const int tp = warp >= 16 ? 1 : 0;       // this set's tile parity
    const int ctid = tp * 128 + (threadIdx.x - 256 - (tp ? 256 : 0));   // 0 .. NP2-1
    const int q4 = warp & 3;
    float* abuf = reinterpret_cast<float*>(sm + L.abuf);   // [2 slots][CHT]
    float* mpart = reinterpret_cast<float*>(sm + L.mpart); // [NP2][2]
    float* mfin = reinterpret_cast<float*>(sm + L.mrow);   // [RP][2] merged (max, 1 / sum)
    float* psum = reinterpret_cast<float*>(sm + L.rsum);   // [4] + inverse sum at [8]
    Chunk c1 = no_chunk();
    for (int k = 0;; ++k) {
      const int g = b0 + k * P;
      const bool have = g < p.total_chunks;
      if (!have && c1.g < 0) break;
      // ---- W(x_k-1), pass 2, its sum
      if (c1.g >= 0) {
        const int buf = (k - 1) & 1;   // tensor-memory buffer and smem slot of x_k-1
        if (ctid == 0)
          wait_count(&p.cnt[c1.u * kScoreCnt + 2 * p.group], nann * c1.nch, abort, p.status,
                     p.abort_all, p.wait_ns);
        // the slot's previous chunk (x_k-3) has been written out
        if (red) mbar_wait(&sfree[buf], (((k - 1) >> 1) & 1) ^ 1, abort, p.status);
        RKV_STAMP(k, 2);
        named_bar_sync(2, NP2);
        {
          // every thread folds a fixed subset of the unit's chunks for one row
          // (eight loads in flight at a time), then the subsets are merged in
          // order: every CTA of the unit gets identical values
          constexpr int TPRX = NP2 / RP;   // threads per query row
          const int rr = ctid / TPRX, tt = ctid - rr * TPRX;
          const float* xs_in = p.xstat + static_cast<int64_t>(c1.g0) * XS + 2 * rr;
          float M = kNegBig, S = 0.f;
          for (int q0 = tt; q0 < c1.nch; q0 += 8 * TPRX) {
            float lm[8], ls[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              const int q = q0 + x * TPRX;
              lm[x] = q < c1.nch ? __ldcg(xs_in + q * XS) : kNegBig;
              ls[x] = q < c1.nch ? __ldcg(xs_in + q * XS + 1) : 0.f;
            }
#pragma unroll
            for (int x = 0; x < 8; ++x)
              if (q0 + x * TPRX < c1.nch) merge_stat(M, S, lm[x], ls[x]);
          }
          mpart[2 * ctid] = M;
          mpart[2 * ctid + 1] = S;
        }
        named_bar_sync(2, NP2);
        if (ctid < RP) {
          constexpr int TPRX = NP2 / RP;
          float M = kNegBig, S = 0.f;
#pragma unroll
          for (int tt = 0; tt < TPRX; ++tt)
            merge_stat(M, S, mpart[2 * (ctid * TPRX + tt)], mpart[2 * (ctid * TPRX + tt) + 1]);
          mfin[2 * ctid] = M;
          mfin[2 * ctid + 1] = S > 0.f ? 1.f / S : 0.f;
        }
        named_bar_sync(2, NP2);
        RKV_STAMP(k, 3);
        const float* mrow2 = mfin;   // (max, 1 / sum) per query row
        // p = 2^(y - M) / L = 2^(y - (M + log2 L)) for the NR rows this thread
        // holds; padding rows (and rows that see no key) get +inf there, so
        // they add exactly 0
        constexpr int NR = RP / 4;
        const int qd = lane >> 2, tq = lane & 3;
        float ML[NR];
#pragma unroll
        for (int i = 0; i < RP / 8; ++i)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int r = 8 * i + 2 * tq + e;
            const float il = mrow2[2 * r + 1];
            const bool real = ((rmask >> r) & 1u) != 0 && il > 0.f;
            ML[2 * i + e] = real ? mrow2[2 * r] - __log2f(il) : INFINITY;
          }
        float* ab = abuf + buf * CHT;
        float part = 0.f;
#ifdef RKV_TRACE
        long long c_tw2 = 0;
        const long long c_p2 = clock64();
#endif
        for (int t = tp; t < c1.nt; t += NPAR) {
          const int t0 = c1.start + kTile * t;
          const bool inside = t0 + kTile <= c1.c;
          float sum[4];   // tokens qd, qd + 8, 16 + qd, 24 + qd of the quarter
          uint32_t v[2][RP / 2];
          RKV_CLK_BEGIN(cw1);
#pragma unroll
          for (int h = 0; h < 2; ++h)
            tmem_ld_tile<RP>(tmem + (static_cast<uint32_t>(q4 * 32 + 16 * h) << 16) +
                                 buf * kBufCols + t * RP, v[h]);
          tmem_wait_ld();
          RKV_CLK_ADD(c_tw2, cw1);
          if (inside) {
            // padding rows carry an infinite shift, so they add exactly 0
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float pa = 0.f, pb = 0.f;
#pragma unroll
              for (int i = 0; i < RP / 8; ++i)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  pa += ex2(fmaf(__uint_as_float(v[h][4 * i + e]), p.scale_log2, -ML[2 * i + e]));
                  pb += ex2(fmaf(__uint_as_float(v[h][4 * i + 2 + e]), p.scale_log2,
                                 -ML[2 * i + e]));
                }
              sum[2 * h] = pa;
              sum[2 * h + 1] = pb;
            }
          } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int ja = t0 + q4 * 32 + 16 * h + qd, jb = ja + 8;
              float pa = 0.f, pb = 0.f;
#pragma unroll
              for (int i = 0; i < RP / 8; ++i)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const int r = 8 * i + 2 * tq + e;
                  const bool real = ((rmask >> r) & 1u) != 0;
                  if (real && ja < c1.n && ja <= c1.c + row_t[r])
                    pa += ex2(fmaf(__uint_as_float(v[h][4 * i + e]), p.scale_log2, -ML[2 * i + e]));
                  if (real && jb < c1.n && jb <= c1.c + row_t[r])
                    pb += ex2(fmaf(__uint_as_float(v[h][4 * i + 2 + e]), p.scale_log2,
                                   -ML[2 * i + e]));
                }
              sum[2 * h] = pa;
              sum[2 * h + 1] = pb;
            }
          }
          // the four lanes of a quad hold the same tokens' other rows
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            sum[x] += __shfl_xor_sync(0xffffffffu, sum[x], 1);
            sum[x] += __shfl_xor_sync(0xffffffffu, sum[x], 2);
          }
          // lane tq writes token (tq >> 1) * 16 + qd + (tq & 1) * 8 of the quarter
          const float mine = tq == 0 ? sum[0] : (tq == 1 ? sum[1] : (tq == 2 ? sum[2] : sum[3]));
          const int trow = q4 * 32 + (tq >> 1) * 16 + qd + (tq & 1) * 8;
          const int j = t0 + trow;
          if (j < c1.c) {
            ab[kTile * t + trow] = mine;
            part += mine;
          }
        }
#ifdef RKV_TRACE
        RKV_STORE(k, 9, c_tw2);
        RKV_STORE(k, 10, clock64() - c_p2);
#endif
        // this buffer's logits have been read: the MMA may reuse it
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tfree[buf]);
        RKV_STAMP(k, 4);

        part = warp_reduce_sum(part);
        if (lane == 0) psum[tp * 4 + q4] = part;
        named_bar_sync(2, NP2);
        if (ctid == 0) {
          float* xo = p.xsum + static_cast<int64_t>(c1.g) * (2 * kScoreMaxGroups) + 2 * p.group;
          float sa = (psum[0] + psum[1]) + (psum[2] + psum[3]);
          if (NPAR > 1) sa += (psum[4] + psum[5]) + (psum[6] + psum[7]);
          xo[0] = sa;
          if (red) {
            __threadfence();
            atomicAdd(&p.cnt[c1.u * kScoreCnt + 2 * p.group + 1], 1);
            mbar_arrive(&sfull[buf]);   // the output warps may write this chunk out
          }
        }
        if (!red) {
          // an earlier row group: add this group's probabilities to a (not yet
          // normalised); the last group normalises
          for (int i = ctid; i < c1.len; i += NP2) {
            const int j = c1.start + i;
            const int64_t gi = c1.base + j;
            if (j < c1.c) p.a_out[gi] = p.group > 0 ? p.a_out[gi] + ab[i] : ab[i];
          }
        }
      }
      named_bar_sync(2, NP2);   // psum is reused
      c1 = have ? chunk_info(p, g) : no_chunk();
    }
  } else if (warp >= 12 && red) {
    // ---------------------------------------------- norm warps
    // pass 1: rho = 1/||k|| (GEMM form: stored for the redundancy GEMM; closed
    // form: U = sum_j rho_j k_j, announced per chunk); closed form pass 2: m_j
    // of x_k-1 from the K tiles read again and the unit's U, then r of x_k-2
    const int ctid = threadIdx.x - 384;      // 0..127
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    float* red2 = reinterpret_cast<float*>(sm + L.red2);   // [4 quarters][128]
    float* rhot = reinterpret_cast<float*>(sm + L.rhot);   // [2][128]
    float* ufin = reinterpret_cast<float*>(sm + L.ufin);   // [128]
    float* rhoc = reinterpret_cast<float*>(sm + L.rhoc);   // [2 slots][CHT] rho of a chunk
    float* marr = reinterpret_cast<float*>(sm + L.marr);   // [2 slots][CHT]
    float* esum = reinterpret_cast<float*>(sm + L.esum);   // [4] + inverse sum at [8]
    int stage = 0;
    uint32_t ph = 0;
    int ntile = 0;
    Chunk c1 = no_chunk();
    // U += rho_row * k_row over the warp's 32 rows of a tile
    auto u_accumulate = [&](uint32_t sb, float rho, float (&U4)[4]) {
      float* rt = rhot + (ntile & 1) * 128;
      rt[row] = rho;
      named_bar_sync(3, 128);
      const int hd = lane >> 4;
      const uint32_t cidx = (lane & 15) >> 1;
      const uint32_t sub = (lane & 1) * 8;
      float U8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 8
      for (int rr = 0; rr < 32; ++rr) {
        const int rw = q4 * 32 + rr;
        const float rr_rho = rt[rw];
        const uint32_t ad = sb + hd * (kTileBytes / 2) + rw * 128 + ((cidx ^ (rw & 7)) << 4) + sub;
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
    };
    for (int k = 0;; ++k) {
      const int g = b0 + k * P;
      const bool have = g < p.total_chunks;
      if (!have && c1.g < 0) break;
      const Chunk cur = have ? chunk_info(p, g) : no_chunk();
      // ---- pass 1 of x_k
      if (have) {
        float U4[4] = {0.f, 0.f, 0.f, 0.f};
        float* rho_u = CLOSED ? nullptr : p.rho_out + p.rho_off[cur.u];
        for (int t = 0; t < cur.nt; ++t) {
          const int j = cur.start + kTile * t + row;
          mbar_wait(&full[stage], ph, abort, p.status);
          __syncwarp();
          const uint32_t sb = smem_u32(sm + L.stages + stage * kTileBytes);
          uint4 xs[16];
          load_row(sb, row, xs);
          const float n2 = row_norm2(xs);
          const float rho = (j < cur.n && n2 > 0.f) ? 1.f / sqrtf(n2) : 0.f;
          if constexpr (CLOSED) {
            rhoc[(k & 1) * CHT + kTile * t + row] = rho;
            u_accumulate(sb, rho, U4);
          } else {
            if (j < cur.n) rho_u[j] = rho;
          }
          ++ntile;
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[stage]);
          if (++stage == NS) { stage = 0; ph ^= 1; }
        }
        if constexpr (CLOSED) {
#pragma unroll
          for (int i = 0; i < 4; ++i) red2[q4 * 128 + lane * 4 + i] = U4[i];
          named_bar_sync(3, 128);
          p.xstat[static_cast<int64_t>(cur.g) * XS + 2 * RP + ctid] =
              ((red2[ctid] + red2[128 + ctid]) + red2[256 + ctid]) + red2[384 + ctid];
          named_bar_sync(3, 128);
          if (ctid == 0 && cur.g != p.drop_chunk) {
            __threadfence();
            atomicAdd(&p.cnt[cur.u * kScoreCnt + 2 * p.group], 1);
          }
        } else if (cur.g == cur.g0 + cur.nch - 1) {
          // the unit's last chunk zeroes the pads of its rho segment
          const int64_t pe = p.rho_off[cur.u + 1];
          for (int64_t gi = p.rho_off[cur.u] + cur.n + ctid; gi < pe; gi += 128)
            p.rho_out[gi] = 0.f;
        }
      }
      if constexpr (CLOSED) {
        // ---- W(x_k-1): the unit's U; m of x_k-1 from its tiles read again
        if (c1.g >= 0) {
          const int slot = (k - 1) & 1;
          if (ctid == 0)
            wait_count(&p.cnt[c1.u * kScoreCnt + 2 * p.group], nann * c1.nch, abort, p.status,
                       p.abort_all, p.wait_ns);
          mbar_wait(&sfree[slot], (((k - 1) >> 1) & 1) ^ 1, abort, p.status);
          named_bar_sync(3, 128);
          {
            // thread = one dimension of U, the unit's chunks in order
            const float* ui = p.xstat + static_cast<int64_t>(c1.g0) * XS + 2 * RP + ctid;
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int q0 = 0; q0 < c1.nch; q0 += 8) {
#pragma unroll
              for (int x = 0; x < 8; ++x)
                if (q0 + x < c1.nch) acc[x] += __ldcg(ui + (q0 + x) * XS);
            }
            ufin[ctid] = ((acc[0] + acc[1]) + (acc[2] + acc[3])) +
                         ((acc[4] + acc[5]) + (acc[6] + acc[7]));
          }
          named_bar_sync(3, 128);
          const float inv_nm1 = c1.n > 1 ? 1.f / static_cast<float>(c1.n - 1) : 0.f;
          float* ma = marr + slot * CHT;
          const float* rc = rhoc + slot * CHT;
          float part = 0.f;
          for (int t = 0; t < c1.nt; ++t) {
            const int j = c1.start + kTile * t + row;
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
            if (j < c1.c) {
              const float rho = rc[kTile * t + row];
              const float dot = (dq[0] + dq[1]) + (dq[2] + dq[3]);
              const float m = (rho * dot - (rho > 0.f ? 1.f : 0.f)) * inv_nm1;
              ma[kTile * t + row] = m;
              part += ex2(m * kLog2e);
            }
          }
          part = warp_reduce_sum(part);
          if (lane == 0) esum[q4] = part;
          named_bar_sync(3, 128);
          if (ctid == 0) {
            float* xo =
                p.xsum + static_cast<int64_t>(c1.g) * (2 * kScoreMaxGroups) + 2 * p.group + 1;
            *xo = (esum[0] + esum[1]) + (esum[2] + esum[3]);
            __threadfence();
            atomicAdd(&p.cnt[c1.u * kScoreCnt + 2 * p.group + 1], 1);
            mbar_arrive(&sfull[slot]);
          }
          named_bar_sync(3, 128);   // esum is reused
        }
        c1 = cur;
      } else if (!have) {
        break;
      }
    }
  }

  // ---------------------------------------------------------------- teardown
  tc_fence_before();
  __syncthreads();
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

cudaError_t score_configure(int rp, bool closed, int smem_bytes) {
  return cudaFuncSetAttribute(pick(rp, closed), cudaFuncAttributeMaxDynamicSharedMemorySize,
                              smem_bytes);
}

int score_max_ctas(int rp, bool closed, int smem_bytes) {
  int per = 0, dev = 0, nsm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, pick(rp, closed), score_threads(closed),
                                                    smem_bytes) != cudaSuccess ||
      cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  // one CTA per SM: each allocates all 512 tensor-memory columns
  return per >= 1 ? nsm : 0;
}

bool score_plan(int R, const int64_t* off, int U, int max_ctas, int tpc_fixed, ScoreDims* d) {
  d->rp = R <= 16 ? 16 : 32;
  d->ngroups = (R + 31) / 32;
  if (d->ngroups > kScoreMaxGroups) return false;
  const int tpc_max = score_chunk_tokens(d->rp) / kTile;
  int64_t tiles = 0, tmax = 0;
  for (int u = 0; u < U; ++u) {
    const int64_t t = (off[u + 1] - off[u] + kTile - 1) / kTile;
    tiles += t;
    if (t > tmax) tmax = t;
  }
  int tpc = tpc_fixed;
  if (tpc <= 0) {
    // spread small batches over every SM; chunks of at most tpc_max tiles
    const int64_t want = (tiles + max_ctas - 1) / max_ctas;
    tpc = static_cast<int>(want < 1 ? 1 : (want > tpc_max ? tpc_max : want));
  }
  if (tpc > tpc_max) return false;
  for (;;) {
    int64_t chunks = 0, cmax = 0;
    for (int u = 0; u < U; ++u) {
      const int64_t t = (off[u + 1] - off[u] + kTile - 1) / kTile;
      const int64_t c = (t + tpc - 1) / tpc;
      chunks += c;
      if (c > cmax) cmax = c;
    }
    const int64_t grid = chunks < max_ctas ? chunks : max_ctas;
    // progress needs every unit within 2 * grid chunks
    if (cmax <= 2 * grid) {
      d->tpc = tpc;
      d->chunks = chunks;
      d->grid = static_cast<int>(grid);
      return true;
    }
    if (tpc_fixed > 0 || tpc >= tpc_max) return false;
    ++tpc;
  }
}

cudaError_t launch_score(const CUtensorMap& kmap, const CUtensorMap& qmap, const ScoreParams& p,
                         int rp, bool closed, int grid, cudaStream_t st) {
  const ScoreLayout L = score_layout(rp, closed, p.nstages);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(score_threads(closed), 1, 1);
  cfg.dynamicSmemBytes = L.total + 1024;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: chunk exchanges
  at[0].val.cooperative = 1;
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

#ifdef RKV_TRACE
extern "C" int rkv_debug_score_trace(void* dst, size_t bytes) {
  return static_cast<int>(cudaMemcpyFromSymbol(dst, rkv::g_score_trace, bytes));
}
extern "C" int rkv_debug_tile_trace(void* dst, size_t bytes) {
  return static_cast<int>(cudaMemcpyFromSymbol(dst, rkv::g_tile_trace, bytes));
}
#endif
