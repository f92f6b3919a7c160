// Internal declarations shared by the kernels and the C ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rkv {

constexpr int kHeadDim = 128;        // d (the only supported head size)
constexpr int kTile = 128;           // tokens per K tile (TMA box rows, MMA M)
constexpr int kTileBytes = kTile * kHeadDim * 2;
constexpr int kMaxTokensPerUnit = 49152;  // select keeps a unit's keys in shared memory
constexpr int kMaxRows = 32;         // G * w limit (MMA N of the logits tile)
constexpr int kScoreThreads = 512;   // 16 warps
constexpr int kGemmThreads = 640;    // producer, MMA, 2 idle, 16 epilogue warps
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- score
struct ScoreParams {
  const int64_t* tok_off;  // [U+1]
  int num_units;
  int R;                   // G * w real query rows
  int w;
  int cs;                  // CTAs per cluster (one unit per cluster)
  int nstages;             // K tile ring depth
  float scale_log2;        // log2(e) / sqrt(d)
  float* a_out;            // [T]
  float* r_out;            // [T]
  float* m_out;            // [T] or null
  float* rho_out;          // 1/||k|| at rho_off[u] + j (pads zeroed), or null
  const int64_t* rho_off;  // [U+1] 256-aligned per-unit offsets into rho_out
  int* status;
};

struct ScoreLayout {
  uint32_t stages, q, abar, marr, rhoc, rhot, ufin, gath, gath2, mrow, invl, red1, red2, rsum,
      rowt, xbuf, bars, slot, flags, total;
};

constexpr int kMaxClusterSize = 16;
constexpr int kTmemColsTotal = 512;

// Logit tiles of one CTA live in TMEM for the whole unit: 512 columns hold
// 512 / rp tiles of 128 tokens.
__host__ __device__ inline int score_res_tiles(int rp) { return kTmemColsTotal / rp; }
__host__ __device__ inline int score_lmax(int rp) { return score_res_tiles(rp) * kTile; }
// Floats of one CTA's round-1 partials: (max, sum) per query row [, U].
__host__ __device__ inline int score_xb(int rp, bool closed) { return 2 * rp + (closed ? 128 : 0); }
constexpr int kScoreBarsFixed = 32 + 1 + 2 + 2 + 2;  // tile-ready, TMEM-free, Q, Q, exchange

__host__ __device__ inline ScoreLayout score_layout(int rp, bool closed, int ns) {
  ScoreLayout L;
  uint32_t o = 0;
  const int lmax = score_lmax(rp);
  L.stages = o; o += ns * kTileBytes;
  L.q = o; o += 2 * rp * 256;
  L.abar = o; o += lmax * 4;
  L.marr = o; if (closed) o += lmax * 4;
  L.rhoc = o; if (closed) o += lmax * 4;
  L.rhot = o; if (closed) o += 2 * 128 * 4;
  L.ufin = o; if (closed) o += 128 * 4;
  L.gath = o; o += kMaxClusterSize * score_xb(rp, closed) * 4;   // round-1 inbox
  L.gath2 = o; o += kMaxClusterSize * 4 * 4;                       // round-2 inbox
  L.mrow = o; o += rp * 4;
  L.invl = o; o += rp * 4;
  L.red1 = o; o += 4 * rp * 2 * 4;
  L.red2 = o; if (closed) o += 4 * 128 * 4;
  L.rsum = o; o += 32 * 4;
  L.rowt = o; o += 32 * 4;
  L.xbuf = o; o += (score_xb(rp, closed) + 4) * 4;
  o = (o + 15u) & ~15u;
  L.bars = o; o += (2 * ns + kScoreBarsFixed) * 8;
  L.slot = o; o += 16;
  L.flags = o; o += 16;
  L.total = o;
  return L;
}

// Deepest K-tile ring that fits next to the rest of the layout.
__host__ __device__ inline int score_stages(int rp, bool closed, int smem_cap) {
  for (int ns = 8; ns >= 2; --ns)
    if (static_cast<int>(score_layout(rp, closed, ns).total) + 1024 <= smem_cap) return ns;
  return 0;
}

// Cluster size of the score kernel for a batch of `units` units of at most
// nmax tokens.  It is the smallest power of two whose CTAs hold a unit's logits
// in TMEM (at most max_cs).  A unit is spread further, to at most 1024 tokens
// per CTA, only while the batch has fewer units than clusters of that size can
// be resident (clusters[log2 cs]): with more units, every extra CTA per unit
// only adds cluster exchanges.  Returns 0 when no size fits.
inline int score_cluster_size(int nmax, int rp, int max_cs, int64_t units, const int* clusters) {
  int cs = 1;
  while ((((nmax + cs - 1) / cs + kTile - 1) / kTile) * kTile > score_lmax(rp)) {
    if (cs >= max_cs) return 0;
    cs <<= 1;
  }
  auto log2i = [](int x) { int l = 0; while ((1 << l) < x) ++l; return l; };
  while (cs < max_cs && (nmax + cs - 1) / cs > 1024 && units < clusters[log2i(cs)]) cs <<= 1;
  return cs;
}

// ---------------------------------------------------------------- redundancy GEMM
struct GemmParams {
  const int64_t* tok_off;  // [U+1]
  const int* item_off;     // [U+1] prefix of row blocks per unit
  int num_units;
  int w;
  const float* rho;        // 1/||k|| at rho_off[u] + j, zero up to rho_off[u+1]
  const int64_t* rho_off;  // [U+1] multiples of kRhoAlign
  float* m_dst;            // [T] receives m (may equal r_dst)
  float* r_dst;            // [T] receives r
  int* unit_cnt;           // [U] zeroed by the plan kernel
  int* status;
  // symmetric form only: scratch of column and row partial sums (layout at
  // sym_scratch_floats) and its per-unit offsets
  float* cs;               // [cs_off[U]]
  const int64_t* cs_off;   // [U+1]
};

template <bool kPair>
struct GemmCfg {
  static constexpr int kCtaGroup = kPair ? 2 : 1;
  static constexpr int kRowsPerCta = 128;                    // A rows held by a CTA
  static constexpr int kRowsPerItem = kPair ? 256 : 128;
  static constexpr int kN = 256;                             // key columns per tile
  static constexpr int kBRows = kPair ? 128 : 256;           // key rows a CTA loads
  static constexpr int kStages = kPair ? 5 : 2;
  static constexpr int kABytes = kRowsPerCta * 256;          // 32 KiB
  static constexpr int kBBytes = kBRows * 256;
  static constexpr int kMmaM = kPair ? 256 : 128;
};

constexpr int kRhoAlign = 256;   // per-unit rho segments start at multiples of this
constexpr int kRhoSlots = 8;     // ring of 256-column rho tiles in the GEMM kernel
constexpr int kRowRing = 4;      // symmetric form: ring of per-tile row-partial buffers

struct GemmLayout {
  uint32_t a, b, rho, rowx, fin, colx, rowr, bars, slot, flags, total;
};
template <bool kPair>
__host__ __device__ inline GemmLayout gemm_layout() {
  using C = GemmCfg<kPair>;
  GemmLayout L;
  uint32_t o = 0;
  L.a = o; o += C::kABytes;
  L.b = o; o += C::kStages * C::kBBytes;
  L.rho = o; o += kRhoSlots * 256 * 4;
  L.rowx = o; o += 4 * 128 * 4;
  L.fin = o; o += 32 * 4;
  L.colx = o; o += 2 * 4 * 4 * 32 * 8;   // symmetric form: [2][cg][q][lane] float2
  L.rowr = o; o += kRowRing * 4 * 128 * 4;   // symmetric form: [kRowRing][cg][128 rows]
  L.bars = o; o += (2 + 2 * C::kStages + 4 + 2 * kRhoSlots + 2 * kRowRing) * 8;
  L.slot = o; o += 16;
  L.flags = o; o += 16;
  L.total = o;
  return L;
}

// ---------------------------------------------------------------- launches
// Each returns a cudaError_t of the launch (cudaSuccess when enqueued).
cudaError_t launch_score(const CUtensorMap& kmap, const CUtensorMap& qmap, const ScoreParams& p,
                         int rp, bool closed, int nclusters, cudaStream_t st);
cudaError_t score_configure(int rp, bool closed, int smem_bytes, int cs);
int score_max_clusters(int rp, bool closed, int smem_bytes, int cs);

cudaError_t launch_plan(const int64_t* tok_off, int U, int w, int rows_per_item, int* item_off,
                        int* unit_cnt, int64_t* rho_off, int64_t* cs_off, cudaStream_t st);
cudaError_t launch_gemm(const CUtensorMap& amap, const CUtensorMap& bmap, const GemmParams& p,
                        bool pair, bool rowmax, bool sym, int nctas, cudaStream_t st);
cudaError_t launch_sym_finish(const GemmParams& p, int nsm, cudaStream_t st);
cudaError_t gemm_configure(bool pair, bool rowmax, bool sym);
int gemm_max_ctas(bool pair, bool rowmax, bool sym);
// Scratch of the symmetric form for one unit of nb = ceil(n / 256) blocks:
// the two CTAs' column sums of every block (2 x 256 floats per block), then
// for each block a the row sums of the slots (a, b), b = a + 1 .. nb - 1
// (256 floats each).  128 nb (nb + 3) floats in all; every float is written
// by exactly one store of the GEMM.
__host__ __device__ inline int64_t sym_scratch_floats(int64_t n, int w) {
  if (n - w <= 0) return 0;
  const int64_t nb = (n + 255) / 256;
  return 128 * nb * (nb + 3);
}
// GEMM work items of one unit: its blocks of candidate rows, or in the
// symmetric form all its 256-key blocks (when it has candidates).
__host__ __device__ inline int64_t gemm_unit_items(int64_t n, int64_t c, int rows_per_item,
                                                   bool sym) {
  if (c <= 0) return 0;
  return sym ? (n + 255) / 256 : (c + rows_per_item - 1) / rows_per_item;
}

cudaError_t launch_select(const int64_t* tok_off, int U, int w, int cmax, const float* a,
                          const float* r, float lam, int budget, const int32_t* budgets,
                          int sinks, int W, int32_t* idx, int32_t* n_kept, cudaStream_t st);
cudaError_t select_configure();

cudaError_t launch_compact(const int64_t* tok_off, int U, int W, const int32_t* idx,
                           const int32_t* n_kept, const void* K, const void* V, void* Ko,
                           void* Vo, int* status, int nsm, cudaStream_t st);

int refree_padded_group(int G);   // heads per token in the refree logit scratch
cudaError_t launch_refree(const int64_t* tok_off, int U, int G, int w, const void* Q,
                          const void* K, int sinks, float T, int max_budget, float* zbuf,
                          float* p_last, int32_t* budgets, int32_t* keep_count, int nsm,
                          cudaStream_t st);
cudaError_t inplace_configure();
cudaError_t launch_evict_in_place(const int64_t* tok_off, int U, int nmax, int W,
                                  const int32_t* idx, const int32_t* n_kept, uint8_t* keep,
                                  int32_t* free_slots, int32_t* n_free, int* status, int nsm,
                                  cudaStream_t st);
cudaError_t launch_fill_slots(const int64_t* tok_off, int U, const int64_t* new_off,
                              const void* K_new, const void* V_new, void* K, void* V,
                              uint8_t* keep, int32_t* free_slots, int32_t* n_free, int* status,
                              int nsm, cudaStream_t st);

}  // namespace rkv
