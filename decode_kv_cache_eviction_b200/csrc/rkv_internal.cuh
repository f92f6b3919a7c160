// Internal declarations shared by the kernels and the C ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

namespace rkv {

// Host-side NVTX range around one public call (a named span in Nsight
// Systems; a no-op without a tool attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kHeadDim = 128;        // d (the only supported head size)
constexpr int kTile = 128;           // tokens per K tile (TMA box rows, MMA M)
constexpr int kTileBytes = kTile * kHeadDim * 2;
// Longest unit: the in-place eviction keeps a byte per token of a unit and the
// selection a bit per candidate on chip.
constexpr int kMaxTokensPerUnit = 131072;
constexpr int kMaxRows = 256;        // G * w limit (row groups of 32 per launch)
// Score kernel threads: 16 warps, or 20 in the GEMM form (a second set of four
// pass-2 warps; the closed form's norm warps need the registers instead).
__host__ __device__ constexpr int score_threads(bool closed) { return closed ? 512 : 640; }
constexpr int kGemmThreads = 640;    // producer, MMA, 2 idle, 16 epilogue warps
// The symmetric form: producer, MMA, row-sum store, 1 idle, 8 epilogue warps.
__host__ __device__ constexpr int gemm_threads(bool sym) { return sym ? 384 : kGemmThreads; }
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- score
constexpr int kScoreMaxGroups = 8;              // row groups of 32: G * w <= 256
constexpr int kScoreCnt = 2 * kScoreMaxGroups;  // exchange counters per unit

struct ScoreParams {
  const int64_t* tok_off;  // [U+1]
  const int* chunk_off;    // [U+1] prefix of chunks per unit
  const int* chunk_unit;   // [chunks] unit of each chunk
  int num_units;
  int total_chunks;
  int R;                   // G * w query rows of a unit
  int row0;                // first query row of this launch's group
  int Rg;                  // rows of this group (<= RP)
  int w;
  int tpc;                 // tiles of 128 tokens per chunk
  int nstages;             // K tile ring depth
  int group;               // row group of this launch
  int final_pass;          // last row group: normalises, computes the redundancy side
  int drop_chunk;          // fault injection: chunk that skips its first announcement (-1)
  float scale_log2;        // log2(e) / sqrt(d)
  uint64_t wait_ns;        // limit of a wait on another CTA
  float* a_out;            // [T]
  float* r_out;            // [T]
  float* m_out;            // [T] or null
  float* rho_out;          // 1/||k|| at rho_off[u] + j (pads zeroed), or null
  const int64_t* rho_off;  // [U+1] 256-aligned per-unit offsets into rho_out
  int* cnt;                // [U][kScoreCnt] announcement counters, zeroed by the plan kernel
  int* abort_all;          // set when a CTA of this call gives up; zeroed by the plan kernel
  float* xstat;            // [chunks][score_xs] per-chunk (max, sum) per row [, U]
  float* xsum;             // [chunks][kScoreMaxGroups][2] per-chunk sums of abar, exp(m)
  int* status;
};

constexpr int kTmemColsTotal = 512;

// Tokens per chunk: two logit buffers of 256 tensor-memory columns, RP per tile.
__host__ __device__ constexpr int score_chunk_tokens(int rp) { return (256 / rp) * kTile; }
// Floats of one chunk's exchange slot: (max, sum) per query row [, partial U].
__host__ __device__ constexpr int score_xs(int rp, bool closed) {
  return 2 * rp + (closed ? 128 : 0);
}

struct ScoreLayout {
  uint32_t stages, q, abuf, marr, rhoc, red1, red2, rhot, ufin, mpart, mrow, rsum, esum,
      osum, rowt, bars, slot, flags, issued, total;
};

__host__ __device__ inline ScoreLayout score_layout(int rp, bool closed, int ns) {
  ScoreLayout L;
  uint32_t o = 0;
  const int cht = score_chunk_tokens(rp);
  L.stages = o; o += ns * kTileBytes;
  L.q = o; o += 2 * rp * 256;
  L.abuf = o; o += 2 * cht * 4;
  L.marr = o; if (closed) o += 2 * cht * 4;   // (read by the output warps only when closed)
  L.rhoc = o; if (closed) o += 2 * cht * 4;
  L.red1 = o; o += 4 * rp * 2 * 4;
  L.red2 = o; if (closed) o += 4 * 128 * 4;
  L.rhot = o; if (closed) o += 2 * 128 * 4;
  L.ufin = o; if (closed) o += 128 * 4;
  L.mpart = o; o += 256 * 2 * 4;
  L.mrow = o; o += 2 * rp * 4;   // merged (max, 1 / sum) per query row
  L.rsum = o; o += 16 * 4;
  L.esum = o; o += 16 * 4;
  L.osum = o; o += 4 * 4;
  L.rowt = o; o += 32 * 4;
  o = (o + 15u) & ~15u;
  L.bars = o; o += (2 * ns + 32 + 6 + 1 + 4) * 8;
  L.slot = o; o += 16;
  L.flags = o; o += 16;
  L.issued = o; o += 32;
  L.total = o;
  return L;
}

// Deepest K-tile ring that fits next to the rest of the layout.
__host__ __device__ inline int score_stages(int rp, bool closed, int smem_cap) {
  for (int ns = 8; ns >= 2; --ns)
    if (static_cast<int>(score_layout(rp, closed, ns).total) + 1024 <= smem_cap) return ns;
  return 0;
}

// Launch shape of the score kernel for one batch.
struct ScoreDims {
  int rp;          // padded query rows per launch (16, 32)
  int ngroups;     // launches (row groups of 32)
  int tpc;         // tiles per chunk
  int64_t chunks;  // chunks of the batch
  int grid;        // CTAs (<= max_ctas)
};

// Chooses the chunk size (tpc_fixed > 0 forces it) and grid for a batch of U
// units with host row offsets `off`; false if G * w > 256 or a unit is too long
// for the progress rule (every unit within 2 * grid chunks).
bool score_plan(int R, const int64_t* off, int U, int max_ctas, int tpc_fixed, ScoreDims* d);
// Upper bound of the chunks of any batch within the capacities.
constexpr int64_t score_max_chunks(int64_t max_tokens, int max_units, int max_ctas, int rp) {
  const int64_t tpc_max = score_chunk_tokens(rp) / kTile;
  const int64_t a = (max_tokens / kTile + 2 * static_cast<int64_t>(max_units)) / tpc_max + 1;
  return (a > max_ctas ? a : max_ctas) + max_units;
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
                         int rp, bool closed, int grid, cudaStream_t st);
cudaError_t score_configure(int rp, bool closed, int smem_bytes);
int score_max_ctas(int rp, bool closed, int smem_bytes);

// Per-batch offsets and zeroed counters, one block (before the score kernel).
struct PlanParams {
  const int64_t* tok_off;  // [U+1]
  int U;
  int w;
  int tpc;                 // score: tiles per chunk
  int* chunk_off;          // [U+1] score chunks prefix
  int* chunk_unit;         // [chunks] unit of each chunk
  int* score_cnt;          // [U][kScoreCnt] zeroed
  int* score_abort;        // [1] zeroed
  int rows_per_item;       // GEMM: rows per work item (0: no GEMM)
  int* item_off;           // [U+1] GEMM items prefix (or null)
  int* unit_cnt;           // [U] zeroed (or null)
  int64_t* rho_off;        // [U+1] 256-aligned rho offsets (or null)
  int64_t* cs_off;         // [U+1] symmetric scratch offsets (or null)
};
cudaError_t launch_plan(const PlanParams& pp, cudaStream_t st);
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

cudaError_t launch_select(const int64_t* tok_off, int U, int64_t Ttot, int w, int cmax,
                          const float* a,
                          const float* r, float lam, int budget, const int32_t* budgets,
                          int sinks, int W, int32_t* idx, int32_t* n_kept, cudaStream_t st);
cudaError_t select_configure();
// Intermediate arrays of the last score call (rkv_debug_intermediates).
cudaError_t launch_gather_rho(const int64_t* tok_off, const int64_t* rho_off, int U,
                              const float* rho, float* out, cudaStream_t st);
cudaError_t launch_sum_unit_U(const int* chunk_off, int U, const float* xstat, int xs, int u0,
                              float* out, cudaStream_t st);

cudaError_t launch_compact(const int64_t* tok_off, int U, int W, const int32_t* idx,
                           const int32_t* n_kept, const void* K, const void* V, void* Ko,
                           void* Vo, int* status, int nsm, cudaStream_t st);

int refree_padded_group(int G);   // heads per token in the refree logit scratch
constexpr int kRfChunk = 2048;    // tokens per refree work chunk
int64_t refree_max_chunks(int64_t max_tokens, int max_units);
struct RefreeArgs {
  const int64_t* tok_off;
  int U;
  int64_t nchunks;      // sum over units of ceil(N_u / kRfChunk)
  int G, w;
  const void* Q;
  const void* K;
  int sinks;
  float T;
  int max_budget;
  int* chunk_off;       // scratch [U + 1]
  float* zbuf;          // scratch [T_tokens * padded G]
  float2* cstat;        // scratch [nchunks * padded G]
  float* cenergy;       // scratch [nchunks]
  float* p_last;
  int32_t* budgets;
  int32_t* keep_count;
  int nsm;
};
cudaError_t launch_refree(const RefreeArgs& a, cudaStream_t st);
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
