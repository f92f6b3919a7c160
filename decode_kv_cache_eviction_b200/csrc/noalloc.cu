// rkv_score_noalloc: GEMM-mode scoring for callers that cannot allocate device
// memory.  The scratch that rkv_score keeps in an engine's workspace (1/||k||
// per row, the score kernel's per-chunk exchange slots and counters, per-unit
// offsets and finished-block counters, a status word) lives here in one
// file-scope __device__ array of fixed size; the call allocates and frees
// nothing.
//
// The array's device address is looked up once per device with that device
// current (cudaGetSymbolAddress); the host-side symbol itself is only a
// stand-in and is never passed to a kernel.  Every call rewrites the parts it
// reads: the plan kernel rewrites the offsets and zeroes the counters, the
// score kernel rewrites the exchange slots and 1/||k|| of every row it covers.
// Calls that overlap on the GPU share the array and race.  The status word is
// the one part that persists: a device wait that timed out leaves its bit
// there until rkv_noalloc_check_status reads and clears it.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstddef>
#include <mutex>

#include "../../include/rkv.h"
#include "ptx.cuh"
#include "rkv_internal.cuh"

using namespace rkv;

namespace {

constexpr int kMaxUnits = RKV_NOALLOC_MAX_UNITS;
constexpr int64_t kMaxTokens = RKV_NOALLOC_MAX_TOKENS;
constexpr int kMaxRp = 32;                 // G * w <= 32: one score pass
// chunks of any batch within the limits: score_max_chunks with up to 256 CTAs
constexpr int kMaxChunks = 8192;
static_assert(score_max_chunks(kMaxTokens, kMaxUnits, 256, 16) <= kMaxChunks &&
                  score_max_chunks(kMaxTokens, kMaxUnits, 256, 32) <= kMaxChunks,
              "static chunk scratch covers every batch within the limits");
constexpr int kMaxDevices = 64;
constexpr int kSmemCap = 227 * 1024;

struct Scratch {
  float rho[kMaxTokens + static_cast<int64_t>(kRhoAlign) * kMaxUnits];
  float xstat[static_cast<int64_t>(kMaxChunks) * score_xs(kMaxRp, false)];
  float xsum[static_cast<int64_t>(kMaxChunks) * 2 * kScoreMaxGroups];
  int64_t rho_off[kMaxUnits + 1];
  int item_off[kMaxUnits + 1];
  int unit_cnt[kMaxUnits];
  int chunk_off[kMaxUnits + 1];
  int chunk_unit[kMaxChunks];
  int score_cnt[kMaxUnits * kScoreCnt];
  int score_abort[4];
  int status[4];
};

__device__ __align__(256) Scratch g_scratch;

struct DeviceState {
  bool ready = false;
  Scratch* scratch = nullptr;  // device address of g_scratch on this device
  int nstages[2] = {};         // [rp == 32]
  int smem[2] = {};
  int ctas[2] = {};
  int gemm_ctas = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Once per device, with the device current.
int setup(int dev, DeviceState** out) {
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& d = g_dev[dev];
  if (d.ready) {
    *out = &d;
    return RKV_OK;
  }
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
    cudaGetLastError();
    return RKV_ERR_CUDA;
  }
  if (major != 10 || minor != 0) return RKV_ERR_UNSUPPORTED;
  if (!g_encode) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn) {
      cudaGetLastError();
      return RKV_ERR_CUDA;
    }
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  // With lazy module loading the module that holds the array, and so the
  // array itself, may only be loaded here; that is an allocation the caller
  // could not have accounted for if its memory pool is already reserved.
  void* ptr = nullptr;
  const cudaError_t se = cudaGetSymbolAddress(&ptr, g_scratch);
  if (se != cudaSuccess || !ptr) {
    cudaGetLastError();
    return se == cudaErrorMemoryAllocation ? RKV_ERR_OOM : RKV_ERR_CUDA;
  }
  d.scratch = static_cast<Scratch*>(ptr);
  for (int k = 0; k < 2; ++k) {
    const int rp = k ? 32 : 16;
    d.nstages[k] = score_stages(rp, false, kSmemCap);
    d.smem[k] = score_layout(rp, false, d.nstages[k]).total + 1024;
    if (d.nstages[k] == 0 || score_configure(rp, false, d.smem[k]) != cudaSuccess) {
      cudaGetLastError();
      return RKV_ERR_CUDA;
    }
    d.ctas[k] = score_max_ctas(rp, false, d.smem[k]);
    if (d.ctas[k] <= 0) return RKV_ERR_UNSUPPORTED;
  }
  if (gemm_configure(true, false, false) != cudaSuccess) {
    cudaGetLastError();
    return RKV_ERR_CUDA;
  }
  d.gemm_ctas = gemm_max_ctas(true, false, false);
  if (d.gemm_ctas <= 0) return RKV_ERR_UNSUPPORTED;
  d.ready = true;
  *out = &d;
  return RKV_OK;
}

int encode(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kHeadDim) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RKV_OK : RKV_ERR_CUDA;
}

bool aligned_to(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int fail() {
  cudaGetLastError();
  return RKV_ERR_CUDA;
}

}  // namespace

extern "C" int rkv_score_noalloc(int group, int window, const rkv_batch* b, float* a, float* r,
                                 float* m, rkv_stream_t stream) {
  NvtxRange nvtx_("rkv_score_noalloc");
  if (group < 1 || window < 1 || !b || !a || !r) return RKV_ERR_INVALID_ARG;
  if (static_cast<int64_t>(group) * window > kMaxRp) return RKV_ERR_UNSUPPORTED;
  const int U = b->num_units;
  if (U < 0 || !b->tok_off || !b->tok_off_host || !b->K || !b->Q) return RKV_ERR_INVALID_ARG;
  if (U > kMaxUnits) return RKV_ERR_CAPACITY;
  const int64_t* off = b->tok_off_host;
  if (off[0] != 0) return RKV_ERR_INVALID_ARG;
  for (int u = 0; u < U; ++u) {
    const int64_t n = off[u + 1] - off[u];
    if (n < window) return RKV_ERR_INVALID_ARG;
    if (n > kMaxTokensPerUnit) return RKV_ERR_UNSUPPORTED;
  }
  const int64_t T = off[U];
  if (T > kMaxTokens) return RKV_ERR_CAPACITY;
  if (!aligned_to(b->K, 16) || !aligned_to(b->Q, 16) || !aligned_to(a, 4) ||
      !aligned_to(r, 4) || (m && !aligned_to(m, 4)) || !aligned_to(b->tok_off, 8))
    return RKV_ERR_INVALID_ARG;
  if (U == 0) return RKV_OK;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return fail();
  DeviceState* d = nullptr;
  int rc = setup(dev, &d);
  if (rc != RKV_OK) return rc;

  const int R = group * window;
  const int k = R > 16 ? 1 : 0;
  ScoreDims dims;
  if (!score_plan(R, off, U, d->ctas[k], 0, &dims)) return RKV_ERR_UNSUPPORTED;
  if (dims.chunks > kMaxChunks) return RKV_ERR_CAPACITY;

  CUtensorMap kmap, qmap, amap, bmap;
  if (encode(&kmap, b->K, static_cast<uint64_t>(T), kTile) != RKV_OK ||
      encode(&qmap, b->Q, static_cast<uint64_t>(U) * R, dims.rp) != RKV_OK ||
      encode(&amap, b->K, static_cast<uint64_t>(T), GemmCfg<true>::kRowsPerCta) != RKV_OK ||
      encode(&bmap, b->K, static_cast<uint64_t>(T), GemmCfg<true>::kBRows) != RKV_OK)
    return RKV_ERR_CUDA;

  Scratch* s = d->scratch;  // device address, never the host-side symbol
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  constexpr int kRows = GemmCfg<true>::kRowsPerItem;

  PlanParams pp = {};
  pp.tok_off = b->tok_off;
  pp.U = U;
  pp.w = window;
  pp.tpc = dims.tpc;
  pp.chunk_off = s->chunk_off;
  pp.chunk_unit = s->chunk_unit;
  pp.score_cnt = s->score_cnt;
  pp.score_abort = s->score_abort;
  pp.rows_per_item = kRows;
  pp.item_off = s->item_off;
  pp.unit_cnt = s->unit_cnt;
  pp.rho_off = s->rho_off;
  pp.cs_off = nullptr;
  if (launch_plan(pp, st) != cudaSuccess) return fail();

  ScoreParams p = {};
  p.tok_off = b->tok_off;
  p.chunk_off = s->chunk_off;
  p.chunk_unit = s->chunk_unit;
  p.num_units = U;
  p.total_chunks = static_cast<int>(dims.chunks);
  p.R = R;
  p.row0 = 0;
  p.Rg = R;
  p.w = window;
  p.tpc = dims.tpc;
  p.nstages = d->nstages[k];
  p.group = 0;
  p.final_pass = 1;
  p.drop_chunk = -1;
  p.scale_log2 = kLog2e / sqrtf(static_cast<float>(kHeadDim));
  p.wait_ns = 2000000000ull;
  p.a_out = a;
  p.r_out = r;
  p.m_out = m;
  p.rho_out = s->rho;
  p.rho_off = s->rho_off;
  p.cnt = s->score_cnt;
  p.abort_all = s->score_abort;
  p.xstat = s->xstat;
  p.xsum = s->xsum;
  p.status = s->status;
  if (launch_score(kmap, qmap, p, dims.rp, false, dims.grid, st) != cudaSuccess) return fail();

  int64_t items = 0;
  for (int u = 0; u < U; ++u) {
    const int64_t c = off[u + 1] - off[u] - window;
    if (c > 0) items += (c + kRows - 1) / kRows;
  }
  if (items == 0) return RKV_OK;
  GemmParams g;
  g.tok_off = b->tok_off;
  g.item_off = s->item_off;
  g.num_units = U;
  g.w = window;
  g.rho = s->rho;
  g.rho_off = s->rho_off;
  g.m_dst = m ? m : r;
  g.r_dst = r;
  g.unit_cnt = s->unit_cnt;
  g.status = s->status;
  g.cs = nullptr;
  g.cs_off = nullptr;
  int64_t nctas = d->gemm_ctas;
  if (nctas > 2 * items) nctas = 2 * items;
  if (launch_gemm(amap, bmap, g, true, false, false, static_cast<int>(nctas), st) != cudaSuccess)
    return fail();
  return RKV_OK;
}

extern "C" int rkv_noalloc_check_status(rkv_stream_t stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return fail();
  DeviceState* d = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_dev[dev].ready) d = &g_dev[dev];
  }
  if (!d) return RKV_OK;   // no call has run on this device
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return fail();
  int h = 0;
  if (cudaMemcpy(&h, d->scratch->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return fail();
  if (h != 0 && cudaMemset(d->scratch->status, 0, sizeof(int)) != cudaSuccess) return fail();
  if (h & kStatusTimeout) return RKV_ERR_TIMEOUT;
  if (h != 0) return RKV_ERR_CUDA;
  return RKV_OK;
}
