// rkv_score_noalloc: GEMM-mode scoring for callers that cannot allocate device
// memory.  The scratch that rkv_score keeps in an engine's workspace (1/||k||
// per row, per-unit row-block offsets and finished-block counters, a status
// word) lives here in one file-scope __device__ array of fixed size; the call
// allocates and frees nothing.
//
// The array's device address is looked up once per device with that device
// current (cudaGetSymbolAddress); the host-side symbol itself is only a
// stand-in and is never passed to a kernel.  Every call rewrites the parts it
// reads: the plan kernel rewrites the offsets and zeroes the counters, the
// score kernel rewrites 1/||k|| of every row it covers.  Calls that overlap on
// the GPU share the array and race.
#include <cudaTypedefs.h>

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
constexpr int kMaxDevices = 64;
constexpr int kSmemCap = 227 * 1024;

struct Scratch {
  float rho[kMaxTokens + static_cast<int64_t>(kRhoAlign) * kMaxUnits];
  int64_t rho_off[kMaxUnits + 1];
  int item_off[kMaxUnits + 1];
  int unit_cnt[kMaxUnits];
  int status[4];
};

__device__ __align__(256) Scratch g_scratch;

struct DeviceState {
  bool ready = false;
  Scratch* scratch = nullptr;  // device address of g_scratch on this device
  int clusters[2][5] = {};     // [rp == 32][log2 cluster size]
  int max_cs[2] = {};
  int nstages[2] = {};
  int smem[2] = {};
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
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_scratch) != cudaSuccess || !ptr) {
    cudaGetLastError();
    return RKV_ERR_CUDA;
  }
  d.scratch = static_cast<Scratch*>(ptr);
  for (int k = 0; k < 2; ++k) {
    const int rp = k ? 32 : 16;
    d.nstages[k] = score_stages(rp, false, kSmemCap);
    d.smem[k] = score_layout(rp, false, d.nstages[k]).total + 1024;
    if (d.nstages[k] == 0 || score_configure(rp, false, d.smem[k], 16) != cudaSuccess) {
      cudaGetLastError();
      return RKV_ERR_CUDA;
    }
    d.max_cs[k] = 0;
    for (int i = 0; i < 5; ++i) {
      d.clusters[k][i] = score_max_clusters(rp, false, d.smem[k], 1 << i);
      if (d.clusters[k][i] > 0) d.max_cs[k] = 1 << i;
      else break;
    }
    if (d.max_cs[k] == 0) return RKV_ERR_UNSUPPORTED;
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

}  // namespace

extern "C" int rkv_score_noalloc(int group, int window, const rkv_batch* b, float* a, float* r,
                                 float* m, rkv_stream_t stream) {
  if (group < 1 || window < 1 || !b || !a || !r) return RKV_ERR_INVALID_ARG;
  if (static_cast<int64_t>(group) * window > kMaxRows) return RKV_ERR_UNSUPPORTED;
  const int U = b->num_units;
  if (U < 0 || !b->tok_off || !b->tok_off_host || !b->K || !b->Q) return RKV_ERR_INVALID_ARG;
  if (U > kMaxUnits) return RKV_ERR_CAPACITY;
  const int64_t* off = b->tok_off_host;
  if (off[0] != 0) return RKV_ERR_INVALID_ARG;
  int nmax = 0;
  for (int u = 0; u < U; ++u) {
    const int64_t n = off[u + 1] - off[u];
    if (n < window) return RKV_ERR_INVALID_ARG;
    if (n > kMaxTokensPerUnit) return RKV_ERR_UNSUPPORTED;
    if (n > nmax) nmax = static_cast<int>(n);
  }
  const int64_t T = off[U];
  if (T > kMaxTokens) return RKV_ERR_CAPACITY;
  if (!aligned_to(b->K, 16) || !aligned_to(b->Q, 16) || !aligned_to(a, 4) ||
      !aligned_to(r, 4) || (m && !aligned_to(m, 4)) || !aligned_to(b->tok_off, 8))
    return RKV_ERR_INVALID_ARG;
  if (U == 0) return RKV_OK;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return RKV_ERR_CUDA;
  }
  DeviceState* d = nullptr;
  int rc = setup(dev, &d);
  if (rc != RKV_OK) return rc;

  const int R = group * window;
  const int rp = R <= 16 ? 16 : 32;
  const int k = rp == 32 ? 1 : 0;
  const int cs = score_cluster_size(nmax, rp, d->max_cs[k], U, d->clusters[k]);
  if (cs == 0) return RKV_ERR_UNSUPPORTED;
  int ci = 0;
  while ((1 << ci) < cs) ++ci;
  int ncl = d->clusters[k][ci];
  if (ncl > U) ncl = U;

  CUtensorMap kmap, qmap, amap, bmap;
  if (encode(&kmap, b->K, static_cast<uint64_t>(T), kTile) != RKV_OK ||
      encode(&qmap, b->Q, static_cast<uint64_t>(U) * R, rp) != RKV_OK ||
      encode(&amap, b->K, static_cast<uint64_t>(T), GemmCfg<true>::kRowsPerCta) != RKV_OK ||
      encode(&bmap, b->K, static_cast<uint64_t>(T), GemmCfg<true>::kBRows) != RKV_OK)
    return RKV_ERR_CUDA;

  Scratch* s = d->scratch;  // device address, never the host-side symbol
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  ScoreParams p;
  p.tok_off = b->tok_off;
  p.num_units = U;
  p.R = R;
  p.w = window;
  p.cs = cs;
  p.nstages = d->nstages[k];
  p.scale_log2 = kLog2e / sqrtf(static_cast<float>(kHeadDim));
  p.a_out = a;
  p.r_out = r;
  p.m_out = m;
  p.rho_out = s->rho;
  p.rho_off = s->rho_off;
  p.status = s->status;
  constexpr int kRows = GemmCfg<true>::kRowsPerItem;
  if (launch_plan(b->tok_off, U, window, kRows, s->item_off, s->unit_cnt, s->rho_off, nullptr, st) !=
      cudaSuccess) {
    cudaGetLastError();
    return RKV_ERR_CUDA;
  }
  if (launch_score(kmap, qmap, p, rp, false, ncl, st) != cudaSuccess) {
    cudaGetLastError();
    return RKV_ERR_CUDA;
  }
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
  if (launch_gemm(amap, bmap, g, true, false, false, static_cast<int>(nctas), st) != cudaSuccess) {
    cudaGetLastError();
    return RKV_ERR_CUDA;
  }
  return RKV_OK;
}
