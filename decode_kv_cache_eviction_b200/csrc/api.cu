// C ABI of the engine: argument validation, workspace, tensor maps, launches.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <new>

#include "../../include/rkv.h"
#include "engine.cuh"
#include "ptx.cuh"
#include "rkv_internal.cuh"

using namespace rkv;

namespace {

// Bytes rounded up to a 256-byte boundary (sub-buffers of one allocation).
size_t round_up(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

constexpr int kSmemCap = 227 * 1024;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int cuda_fail(cudaError_t e) {
  (void)e;
  cudaGetLastError();
  return RKV_ERR_CUDA;
}

int make_map(rkv_engine* e, CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows) {
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(kHeadDim) * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = e->encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? RKV_OK : RKV_ERR_CUDA;
}

// Host-side checks of a batch against the engine; fills T and the largest N.
int check_batch(const rkv_engine* e, const rkv_batch* b, int64_t* T, int* nmax, int* cmax) {
  if (!b) return RKV_ERR_INVALID_ARG;
  if (b->num_units < 0) return RKV_ERR_INVALID_ARG;
  if (b->num_units > e->cfg.max_units) return RKV_ERR_CAPACITY;
  if (!b->tok_off_host || !b->tok_off) return RKV_ERR_INVALID_ARG;
  const int64_t* off = b->tok_off_host;
  if (off[0] != 0) return RKV_ERR_INVALID_ARG;
  int nm = 0;
  for (int u = 0; u < b->num_units; ++u) {
    const int64_t n = off[u + 1] - off[u];
    if (n < e->cfg.window) return RKV_ERR_INVALID_ARG;
    if (n > e->max_n) return RKV_ERR_UNSUPPORTED;
    if (n > nm) nm = static_cast<int>(n);
  }
  const int64_t t = off[b->num_units];
  if (t > e->cfg.max_tokens) return RKV_ERR_CAPACITY;
  if (!aligned(b->tok_off, 8)) return RKV_ERR_INVALID_ARG;
  *T = t;
  *nmax = nm;
  *cmax = nm - e->cfg.window;
  return RKV_OK;
}

// Record the start event of a launch of `kernel` (when timing is on).
void t_begin(rkv_engine* e, int kernel, cudaStream_t st) {
  if (!e->timing || e->nev >= rkv_engine::kMaxEv) return;
  e->ev_kernel[e->nev] = kernel;
  cudaEventRecord(e->ev[e->nev][0], st);
}
void t_end(rkv_engine* e, cudaStream_t st) {
  if (!e->timing || e->nev >= rkv_engine::kMaxEv) return;
  cudaEventRecord(e->ev[e->nev][1], st);
  ++e->nev;
}

// Fault injected for the next engine creation (rkv_inject_fault(NULL, ...)).
int g_create_fault = 0;

// cudaMalloc that fails once when an allocation fault is armed.
cudaError_t dev_alloc(int* fault, void** p, size_t bytes) {
  if (*fault == RKV_FAULT_ALLOC) {
    *fault = 0;
    *p = nullptr;
    return cudaErrorMemoryAllocation;
  }
  return cudaMalloc(p, bytes);
}

// Floats of symmetric-form scratch that any batch within the capacities can
// need.  A unit of n tokens needs 128 nb (nb + 3) with nb = ceil(n / 256) <=
// x + 1, x = n / 256, so at most 128 (x^2 + 5 x + 4).  Over a batch, sum x^2 <=
// (L / 256) sum x with L the longest unit, sum x <= max_tokens / 256 and there
// are at most max_units units; no batch needs more than max_units units of L
// tokens either.
int64_t sym_scratch_bound(int64_t max_tokens, int max_units, int64_t max_len) {
  const double X = static_cast<double>(max_tokens) / 256.0;
  const double b1 = 128.0 * (static_cast<double>(max_len) / 256.0 * X + 5.0 * X +
                             4.0 * static_cast<double>(max_units));
  const double b2 = static_cast<double>(max_units) * sym_scratch_floats(max_len, 0);
  return static_cast<int64_t>(std::min(b1, b2)) + 1;
}

}  // namespace

cudaError_t rkv_engine_alloc(rkv_engine* e, void** p, size_t bytes) {
  return dev_alloc(&e->fault, p, bytes);
}

extern "C" {

int rkv_version(void) { return 10000; }

const char* rkv_status_string(int s) {
  switch (s) {
    case RKV_OK: return "ok";
    case RKV_ERR_INVALID_ARG: return "invalid argument";
    case RKV_ERR_UNSUPPORTED: return "unsupported configuration or device";
    case RKV_ERR_CUDA: return "CUDA runtime error";
    case RKV_ERR_TIMEOUT: return "device wait timed out";
    case RKV_ERR_OOM: return "device allocation failed";
    case RKV_ERR_CAPACITY: return "batch exceeds engine capacity";
    case RKV_ERR_DEVICE: return "kept index outside its unit";
    default: return "unknown status";
  }
}

int rkv_create(const rkv_config* cfg, rkv_engine** out) {
  NvtxRange nvtx_("rkv_create");
  if (!cfg || !out) return RKV_ERR_INVALID_ARG;
  *out = nullptr;
  if (cfg->group < 1 || cfg->window < 1 || cfg->max_units < 1 || cfg->max_tokens < 1 ||
      cfg->max_unit_tokens < 0)
    return RKV_ERR_INVALID_ARG;
  if (cfg->redundancy != RKV_REDUNDANCY_GEMM && cfg->redundancy != RKV_REDUNDANCY_CLOSED_FORM &&
      cfg->redundancy != RKV_REDUNDANCY_MAX)
    return RKV_ERR_INVALID_ARG;
  if ((cfg->flags & ~(RKV_FLAG_GEMM_SINGLE_CTA | RKV_FLAG_GEMM_SYMMETRIC)) != 0)
    return RKV_ERR_INVALID_ARG;
  if ((cfg->flags & RKV_FLAG_GEMM_SYMMETRIC) &&
      ((cfg->flags & RKV_FLAG_GEMM_SINGLE_CTA) || cfg->redundancy != RKV_REDUNDANCY_GEMM))
    return RKV_ERR_UNSUPPORTED;
  if (cfg->head_dim != kHeadDim) return RKV_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(cfg->group) * cfg->window > kMaxRows) return RKV_ERR_UNSUPPORTED;
  if (cfg->max_tokens >= (static_cast<int64_t>(1) << 31)) return RKV_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(cfg->max_units) * cfg->group * cfg->window >=
      (static_cast<int64_t>(1) << 31))
    return RKV_ERR_UNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cuda_fail(cudaErrorNoDevice);
  int major = 0, minor = 0, nsm = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return cuda_fail(cudaErrorUnknown);
  if (major != 10 || minor != 0) return RKV_ERR_UNSUPPORTED;

  rkv_engine* e = new (std::nothrow) rkv_engine();
  if (!e) return RKV_ERR_OOM;
  e->cfg = *cfg;
  e->device = dev;
  e->nsm = nsm;
  e->pair = (cfg->flags & RKV_FLAG_GEMM_SINGLE_CTA) == 0;
  e->rowmax = cfg->redundancy == RKV_REDUNDANCY_MAX;
  e->sym = (cfg->flags & RKV_FLAG_GEMM_SYMMETRIC) != 0;

  cudaDriverEntryPointQueryResult q;
  void* fn = nullptr;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn) {
    delete e;
    return cuda_fail(cudaErrorUnknown);
  }
  e->encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);

  // Score kernel: deepest K-tile ring that fits, one persistent CTA per SM.
  const bool closed = cfg->redundancy == RKV_REDUNDANCY_CLOSED_FORM;
  const int R = cfg->group * cfg->window;
  e->rp = R <= 16 ? 16 : 32;
  e->nstages = score_stages(e->rp, closed, kSmemCap);
  e->score_smem = score_layout(e->rp, closed, e->nstages).total + 1024;
  if (e->nstages == 0 || score_configure(e->rp, closed, e->score_smem) != cudaSuccess) {
    delete e;
    return cuda_fail(cudaErrorUnknown);
  }
  e->score_ctas = score_max_ctas(e->rp, closed, e->score_smem);
  if (e->score_ctas <= 0) {
    delete e;
    return RKV_ERR_UNSUPPORTED;
  }
  // a unit spans at most 2 * score_ctas chunks; select keeps its keys on chip
  const int64_t score_n = 2 * static_cast<int64_t>(e->score_ctas) * score_chunk_tokens(e->rp);
  e->max_n = static_cast<int>(std::min<int64_t>(score_n, kMaxTokensPerUnit));
  if (cfg->max_unit_tokens < 0 || cfg->max_unit_tokens > e->max_n) {
    delete e;
    return cfg->max_unit_tokens < 0 ? RKV_ERR_INVALID_ARG : RKV_ERR_UNSUPPORTED;
  }
  if (cfg->max_unit_tokens > 0) e->max_n = static_cast<int>(cfg->max_unit_tokens);
  e->max_chunks = score_max_chunks(cfg->max_tokens, cfg->max_units, e->score_ctas, e->rp);

  if (select_configure() != cudaSuccess || inplace_configure() != cudaSuccess) {
    delete e;
    return cuda_fail(cudaErrorUnknown);
  }
  if (!closed) {
    if (gemm_configure(e->pair, e->rowmax, e->sym) != cudaSuccess) {
      delete e;
      return cuda_fail(cudaErrorUnknown);
    }
    e->gemm_ctas = gemm_max_ctas(e->pair, e->rowmax, e->sym);
    if (e->gemm_ctas <= 0) {
      delete e;
      return RKV_ERR_UNSUPPORTED;
    }
  }

  int* fault = &g_create_fault;
  auto alloc = [&](void** p, size_t bytes) { return dev_alloc(fault, p, bytes) == cudaSuccess; };
  bool ok = alloc(reinterpret_cast<void**>(&e->status), 16);
  ok = ok && alloc(reinterpret_cast<void**>(&e->chunk_off), sizeof(int) * (cfg->max_units + 1));
  ok = ok && alloc(reinterpret_cast<void**>(&e->chunk_unit),
                   sizeof(int) * static_cast<size_t>(e->max_chunks));
  ok = ok && alloc(reinterpret_cast<void**>(&e->score_cnt),
                   sizeof(int) * (static_cast<size_t>(cfg->max_units) * kScoreCnt + 1));
  ok = ok && alloc(reinterpret_cast<void**>(&e->xstat),
                   sizeof(float) * static_cast<size_t>(e->max_chunks) * score_xs(e->rp, closed));
  ok = ok && alloc(reinterpret_cast<void**>(&e->xsum),
                   sizeof(float) * static_cast<size_t>(e->max_chunks) * 2 * kScoreMaxGroups);
  if (!closed) {
    const int64_t nrho = cfg->max_tokens + static_cast<int64_t>(kRhoAlign) * cfg->max_units;
    ok = ok && alloc(reinterpret_cast<void**>(&e->item_off), sizeof(int) * (cfg->max_units + 1));
    ok = ok && alloc(reinterpret_cast<void**>(&e->unit_cnt), sizeof(int) * cfg->max_units);
    ok = ok && alloc(reinterpret_cast<void**>(&e->rho), sizeof(float) * nrho);
    ok = ok && alloc(reinterpret_cast<void**>(&e->rho_off),
                     sizeof(int64_t) * (cfg->max_units + 1));
  }
  if (e->sym) {
    // the partial-sum scratch of the largest batch the capacities allow, so that
    // rkv_score never allocates
    e->cs_cap = sym_scratch_bound(cfg->max_tokens, cfg->max_units, e->max_n);
    ok = ok && alloc(reinterpret_cast<void**>(&e->cs_off), sizeof(int64_t) * (cfg->max_units + 1));
    ok = ok && alloc(reinterpret_cast<void**>(&e->cs),
                     sizeof(float) * static_cast<size_t>(std::max<int64_t>(e->cs_cap, 1)));
  }
  ok = ok && cudaMemset(e->status, 0, 16) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    cudaFree(e->status);
    cudaFree(e->chunk_off);
    cudaFree(e->chunk_unit);
    cudaFree(e->score_cnt);
    cudaFree(e->xstat);
    cudaFree(e->xsum);
    cudaFree(e->item_off);
    cudaFree(e->unit_cnt);
    cudaFree(e->rho);
    cudaFree(e->rho_off);
    cudaFree(e->cs_off);
    cudaFree(e->cs);
    delete e;
    return RKV_ERR_OOM;
  }
  *out = e;
  return RKV_OK;
}

int rkv_set_timing(rkv_engine* e, int enable) {
  if (!e) return RKV_ERR_INVALID_ARG;
  if (enable && !e->ev_made) {
    for (int i = 0; i < rkv_engine::kMaxEv; ++i)
      for (int k = 0; k < 2; ++k)
        if (cudaEventCreate(&e->ev[i][k]) != cudaSuccess) return cuda_fail(cudaErrorUnknown);
    e->ev_made = true;
  }
  e->timing = enable != 0;
  e->nev = 0;
  return RKV_OK;
}

int rkv_read_timing(rkv_engine* e, int kernel, double* total_ms, int64_t* launches) {
  if (!e || !total_ms || !launches || kernel < 0 || kernel >= RKV_NUM_KERNELS)
    return RKV_ERR_INVALID_ARG;
  double tot = 0.0;
  int64_t n = 0;
  for (int i = 0; i < e->nev; ++i) {
    if (e->ev_kernel[i] != kernel) continue;
    if (cudaEventSynchronize(e->ev[i][1]) != cudaSuccess) return cuda_fail(cudaErrorUnknown);
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, e->ev[i][0], e->ev[i][1]) != cudaSuccess)
      return cuda_fail(cudaErrorUnknown);
    tot += ms;
    ++n;
  }
  *total_ms = tot;
  *launches = n;
  return RKV_OK;
}

int rkv_destroy(rkv_engine* e) {
  NvtxRange nvtx_("rkv_destroy");
  if (!e) return RKV_OK;
  cudaDeviceSynchronize();
  if (e->ev_made)
    for (int i = 0; i < rkv_engine::kMaxEv; ++i)
      for (int k = 0; k < 2; ++k) cudaEventDestroy(e->ev[i][k]);
  rkv_host_pipeline_free(e);
  cudaFree(e->rf_z);
  cudaFree(e->status);
  cudaFree(e->chunk_off);
  cudaFree(e->chunk_unit);
  cudaFree(e->score_cnt);
  cudaFree(e->xstat);
  cudaFree(e->xsum);
  cudaFree(e->item_off);
  cudaFree(e->unit_cnt);
  cudaFree(e->rho);
  cudaFree(e->rho_off);
  cudaFree(e->cs_off);
  cudaFree(e->cs);
  delete e;
  return RKV_OK;
}

int64_t rkv_launch_count(const rkv_engine* e) { return e ? e->launches : 0; }

int rkv_inject_fault(rkv_engine* e, int fault) {
  if (fault != RKV_FAULT_NONE && fault != RKV_FAULT_ALLOC && fault != RKV_FAULT_DROP_ANNOUNCE)
    return RKV_ERR_INVALID_ARG;
  if (!e) {
    if (fault == RKV_FAULT_DROP_ANNOUNCE) return RKV_ERR_INVALID_ARG;
    g_create_fault = fault;
    return RKV_OK;
  }
  e->fault = fault;
  return RKV_OK;
}

int rkv_score(rkv_engine* e, const rkv_batch* b, float* a, float* r, float* m,
              rkv_stream_t stream) {
  NvtxRange nvtx_("rkv_score");
  if (!e) return RKV_ERR_INVALID_ARG;
  int64_t T = 0;
  int nmax = 0, cmax = 0;
  int rc = check_batch(e, b, &T, &nmax, &cmax);
  if (rc != RKV_OK) return rc;
  if (!a || !r || !b->K || !b->Q) return RKV_ERR_INVALID_ARG;
  if (!aligned(b->K, 16) || !aligned(b->Q, 16) || !aligned(a, 4) || !aligned(r, 4) ||
      (m && !aligned(m, 4)))
    return RKV_ERR_INVALID_ARG;
  const int U = b->num_units;
  if (U == 0) return RKV_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const bool closed = e->cfg.redundancy == RKV_REDUNDANCY_CLOSED_FORM;
  const int R = e->cfg.group * e->cfg.window;
  ScoreDims d;
  if (!score_plan(R, b->tok_off_host, U, e->score_ctas, e->score_tpc_fixed, &d))
    return RKV_ERR_UNSUPPORTED;
  if (d.chunks > e->max_chunks) return RKV_ERR_CAPACITY;
  if (e->sym) {   // the scratch sized at creation covers every batch within the capacities
    int64_t cs_need = 0;
    for (int u = 0; u < U; ++u)
      cs_need += sym_scratch_floats(b->tok_off_host[u + 1] - b->tok_off_host[u], e->cfg.window);
    if (cs_need > e->cs_cap) return RKV_ERR_CAPACITY;
  }

  CUtensorMap kmap, qmap;
  if (make_map(e, &kmap, b->K, static_cast<uint64_t>(T), kTile) != RKV_OK) return RKV_ERR_CUDA;
  if (make_map(e, &qmap, b->Q, static_cast<uint64_t>(U) * R, d.rp) != RKV_OK)
    return RKV_ERR_CUDA;

  const int rows_per_item = e->pair ? GemmCfg<true>::kRowsPerItem : GemmCfg<false>::kRowsPerItem;
  PlanParams pp = {};
  pp.tok_off = b->tok_off;
  pp.U = U;
  pp.w = e->cfg.window;
  pp.tpc = d.tpc;
  pp.chunk_off = e->chunk_off;
  pp.chunk_unit = e->chunk_unit;
  pp.score_cnt = e->score_cnt;
  pp.score_abort = e->score_cnt + static_cast<int64_t>(e->cfg.max_units) * kScoreCnt;
  if (!closed) {   // GEMM row blocks and the padded rho layout the score kernel writes
    pp.rows_per_item = rows_per_item;
    pp.item_off = e->item_off;
    pp.unit_cnt = e->unit_cnt;
    pp.rho_off = e->rho_off;
    pp.cs_off = e->sym ? e->cs_off : nullptr;
  }
  t_begin(e, RKV_KERNEL_PLAN, st);
  cudaError_t err = launch_plan(pp, st);
  t_end(e, st);
  if (err != cudaSuccess) return cuda_fail(err);
  ++e->launches;

  ScoreParams p = {};
  p.tok_off = b->tok_off;
  p.chunk_off = e->chunk_off;
  p.chunk_unit = e->chunk_unit;
  p.num_units = U;
  p.total_chunks = static_cast<int>(d.chunks);
  p.R = R;
  p.w = e->cfg.window;
  p.tpc = d.tpc;
  p.nstages = e->nstages;
  p.scale_log2 = kLog2e / sqrtf(static_cast<float>(kHeadDim));
  p.wait_ns = e->wait_ns;
  p.drop_chunk = -1;
  if (e->fault == RKV_FAULT_DROP_ANNOUNCE) {   // test hook: one announcement goes missing
    e->fault = 0;
    p.drop_chunk = 0;
    p.wait_ns = 50000000ull;
  }
  p.a_out = a;
  p.r_out = r;
  p.m_out = m;
  p.rho_out = closed ? nullptr : e->rho;
  p.rho_off = closed ? nullptr : e->rho_off;
  p.cnt = e->score_cnt;
  p.abort_all = pp.score_abort;
  p.xstat = e->xstat;
  p.xsum = e->xsum;
  p.status = e->status;
  for (int gq = 0; gq < d.ngroups; ++gq) {
    p.group = gq;
    p.row0 = 32 * gq;
    p.Rg = std::min(d.rp, R - p.row0);
    p.final_pass = gq == d.ngroups - 1;
    t_begin(e, RKV_KERNEL_SCORE, st);
    err = launch_score(kmap, qmap, p, d.rp, closed, d.grid, st);
    t_end(e, st);
    if (err != cudaSuccess) return cuda_fail(err);
    ++e->launches;
  }
  if (closed) return RKV_OK;

  // redundancy GEMM
  CUtensorMap amap, bmap;
  if (make_map(e, &amap, b->K, static_cast<uint64_t>(T), GemmCfg<true>::kRowsPerCta) != RKV_OK)
    return RKV_ERR_CUDA;
  if (make_map(e, &bmap, b->K, static_cast<uint64_t>(T),
               e->pair ? GemmCfg<true>::kBRows : GemmCfg<false>::kBRows) != RKV_OK)
    return RKV_ERR_CUDA;
  GemmParams g;
  g.tok_off = b->tok_off;
  g.item_off = e->item_off;
  g.num_units = U;
  g.w = e->cfg.window;
  g.rho = e->rho;
  g.rho_off = e->rho_off;
  g.m_dst = m ? m : r;
  g.r_dst = r;
  g.unit_cnt = e->unit_cnt;
  g.status = e->status;
  g.cs = e->sym ? e->cs : nullptr;
  g.cs_off = e->sym ? e->cs_off : nullptr;
  int64_t items = 0;
  for (int u = 0; u < U; ++u) {
    const int64_t n = b->tok_off_host[u + 1] - b->tok_off_host[u];
    items += gemm_unit_items(n, n - e->cfg.window, rows_per_item, e->sym);
  }
  if (items == 0) return RKV_OK;
  int64_t nctas = e->gemm_ctas;
  const int64_t need = items * (e->pair ? 2 : 1);
  if (nctas > need) nctas = need;
  t_begin(e, RKV_KERNEL_GEMM, st);
  err = launch_gemm(amap, bmap, g, e->pair, e->rowmax, e->sym, static_cast<int>(nctas), st);
  t_end(e, st);
  if (err == cudaSuccess && e->sym) {
    ++e->launches;
    t_begin(e, RKV_KERNEL_FINISH, st);
    err = launch_sym_finish(g, e->nsm, st);
    t_end(e, st);
  }
  if (err != cudaSuccess) return cuda_fail(err);
  ++e->launches;
  return RKV_OK;
}

int rkv_select(rkv_engine* e, const rkv_batch* b, const float* a, const float* r, float lambda,
               int budget, int32_t* idx, int32_t* n_kept, rkv_stream_t stream) {
  NvtxRange nvtx_("rkv_select");
  if (!e) return RKV_ERR_INVALID_ARG;
  int64_t T = 0;
  int nmax = 0, cmax = 0;
  int rc = check_batch(e, b, &T, &nmax, &cmax);
  if (rc != RKV_OK) return rc;
  if (!(lambda >= 0.f && lambda <= 1.f) || budget < 0) return RKV_ERR_INVALID_ARG;
  if (!a || !r || !idx || !n_kept) return RKV_ERR_INVALID_ARG;
  if (!aligned(a, 4) || !aligned(r, 4) || !aligned(idx, 4) || !aligned(n_kept, 4))
    return RKV_ERR_INVALID_ARG;
  const int U = b->num_units;
  if (U == 0) return RKV_OK;
  if (static_cast<int64_t>(budget) + e->cfg.window >= (static_cast<int64_t>(1) << 30) ||
      static_cast<int64_t>(U) * (budget + e->cfg.window) >= (static_cast<int64_t>(1) << 31))
    return RKV_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  t_begin(e, RKV_KERNEL_SELECT, st);
  cudaError_t err = launch_select(b->tok_off, U, T, e->cfg.window, cmax, a, r, lambda, budget,
                                  nullptr, 0, budget + e->cfg.window, idx, n_kept, st);
  t_end(e, st);
  if (err != cudaSuccess) return cuda_fail(err);
  ++e->launches;
  return RKV_OK;
}

int rkv_select_ex(rkv_engine* e, const rkv_batch* b, const float* a, const float* r,
                  float lambda, int budget, const int32_t* budgets, int sinks, int32_t* idx,
                  int32_t* n_kept, rkv_stream_t stream) {
  NvtxRange nvtx_("rkv_select_ex");
  if (!e) return RKV_ERR_INVALID_ARG;
  int64_t T = 0;
  int nmax = 0, cmax = 0;
  int rc = check_batch(e, b, &T, &nmax, &cmax);
  if (rc != RKV_OK) return rc;
  if (!(lambda >= 0.f && lambda <= 1.f) || budget < 0 || sinks < 0) return RKV_ERR_INVALID_ARG;
  if (!a || !r || !idx || !n_kept) return RKV_ERR_INVALID_ARG;
  if (!aligned(a, 4) || !aligned(r, 4) || !aligned(idx, 4) || !aligned(n_kept, 4) ||
      (budgets && !aligned(budgets, 4)))
    return RKV_ERR_INVALID_ARG;
  const int U = b->num_units;
  if (U == 0) return RKV_OK;
  const int64_t W = static_cast<int64_t>(budget) + sinks + e->cfg.window;
  if (W >= (static_cast<int64_t>(1) << 30) || U * W >= (static_cast<int64_t>(1) << 31))
    return RKV_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  t_begin(e, RKV_KERNEL_SELECT, st);
  cudaError_t err = launch_select(b->tok_off, U, T, e->cfg.window, cmax, a, r, lambda, budget,
                                  budgets, sinks, static_cast<int>(W), idx, n_kept, st);
  t_end(e, st);
  if (err != cudaSuccess) return cuda_fail(err);
  ++e->launches;
  return RKV_OK;
}

int rkv_compact(rkv_engine* e, const rkv_batch* b, const int32_t* idx, const int32_t* n_kept,
                int budget, void* K_out, void* V_out, rkv_stream_t stream) {
  NvtxRange nvtx_("rkv_compact");
  if (!e) return RKV_ERR_INVALID_ARG;
  int64_t T = 0;
  int nmax = 0, cmax = 0;
  int rc = check_batch(e, b, &T, &nmax, &cmax);
  if (rc != RKV_OK) return rc;
  if (budget < 0 || !idx || !n_kept || !K_out || !V_out || !b->K || !b->V)
    return RKV_ERR_INVALID_ARG;
  if (!aligned(b->K, 16) || !aligned(b->V, 16) || !aligned(K_out, 16) || !aligned(V_out, 16) ||
      !aligned(idx, 4) || !aligned(n_kept, 4))
    return RKV_ERR_INVALID_ARG;
  const int U = b->num_units;
  if (U == 0) return RKV_OK;
  const int64_t W = static_cast<int64_t>(budget) + e->cfg.window;
  if (U * W >= (static_cast<int64_t>(1) << 31)) return RKV_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  t_begin(e, RKV_KERNEL_COMPACT, st);
  cudaError_t err = launch_compact(b->tok_off, U, static_cast<int>(W), idx, n_kept, b->K, b->V,
                                   K_out, V_out, e->status, e->nsm, st);
  t_end(e, st);
  if (err != cudaSuccess) return cuda_fail(err);
  ++e->launches;
  return RKV_OK;
}

int rkv_evict_in_place(rkv_engine* e, const rkv_batch* b, const int32_t* idx,
                       const int32_t* n_kept, int budget, uint8_t* keep, int32_t* free_slots,
                       int32_t* n_free, rkv_stream_t stream) {
  NvtxRange nvtx_("rkv_evict_in_place");
  if (!e) return RKV_ERR_INVALID_ARG;
  int64_t T = 0;
  int nmax = 0, cmax = 0;
  int rc = check_batch(e, b, &T, &nmax, &cmax);
  if (rc != RKV_OK) return rc;
  if (budget < 0 || !idx || !n_kept || !keep || !free_slots || !n_free) return RKV_ERR_INVALID_ARG;
  if (!aligned(idx, 4) || !aligned(n_kept, 4) || !aligned(free_slots, 4) || !aligned(n_free, 4))
    return RKV_ERR_INVALID_ARG;
  const int U = b->num_units;
  if (U == 0) return RKV_OK;
  const int64_t W = static_cast<int64_t>(budget) + e->cfg.window;
  if (U * W >= (static_cast<int64_t>(1) << 31)) return RKV_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  t_begin(e, RKV_KERNEL_EVICT, st);
  cudaError_t err = launch_evict_in_place(b->tok_off, U, nmax, static_cast<int>(W), idx, n_kept,
                                          keep, free_slots, n_free, e->status, e->nsm, st);
  t_end(e, st);
  if (err != cudaSuccess) return cuda_fail(err);
  ++e->launches;
  return RKV_OK;
}

int rkv_fill_slots(rkv_engine* e, const rkv_batch* b, void* K, void* V, const int64_t* new_off,
                   const int64_t* new_off_host, const void* K_new, const void* V_new,
                   uint8_t* keep, int32_t* free_slots, int32_t* n_free, rkv_stream_t stream) {
  NvtxRange nvtx_("rkv_fill_slots");
  if (!e) return RKV_ERR_INVALID_ARG;
  int64_t T = 0;
  int nmax = 0, cmax = 0;
  int rc = check_batch(e, b, &T, &nmax, &cmax);
  if (rc != RKV_OK) return rc;
  if (!K || !V || !new_off || !new_off_host || !keep || !free_slots || !n_free)
    return RKV_ERR_INVALID_ARG;
  const int U = b->num_units;
  if (new_off_host[0] != 0) return RKV_ERR_INVALID_ARG;
  for (int u = 0; u < U; ++u)
    if (new_off_host[u + 1] < new_off_host[u]) return RKV_ERR_INVALID_ARG;
  const int64_t Tn = new_off_host[U];
  if (Tn > 0 && (!K_new || !V_new)) return RKV_ERR_INVALID_ARG;
  if (!aligned(K, 16) || !aligned(V, 16) || (Tn > 0 && (!aligned(K_new, 16) ||
      !aligned(V_new, 16))) || !aligned(new_off, 8) || !aligned(free_slots, 4) ||
      !aligned(n_free, 4))
    return RKV_ERR_INVALID_ARG;
  if (U == 0 || Tn == 0) return RKV_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  t_begin(e, RKV_KERNEL_FILL, st);
  cudaError_t err = launch_fill_slots(b->tok_off, U, new_off, K_new, V_new, K, V, keep,
                                      free_slots, n_free, e->status, e->nsm, st);
  t_end(e, st);
  if (err != cudaSuccess) return cuda_fail(err);
  ++e->launches;
  return RKV_OK;
}

int rkv_refree_budget(rkv_engine* e, const rkv_batch* b, float T, int sinks, int max_budget,
                      float* p_last, int32_t* budgets, int32_t* keep_count,
                      rkv_stream_t stream) {
  NvtxRange nvtx_("rkv_refree_budget");
  if (!e) return RKV_ERR_INVALID_ARG;
  int64_t Tn = 0;
  int nmax = 0, cmax = 0;
  int rc = check_batch(e, b, &Tn, &nmax, &cmax);
  if (rc != RKV_OK) return rc;
  if (!(T >= 0.f && T < 1.f) || sinks < 0 || max_budget < 0 || !p_last || !budgets || !b->K ||
      !b->Q)
    return RKV_ERR_INVALID_ARG;
  if (!aligned(p_last, 4) || !aligned(budgets, 4) || (keep_count && !aligned(keep_count, 4)) ||
      !aligned(b->K, 16) || !aligned(b->Q, 16))
    return RKV_ERR_INVALID_ARG;
  if (e->cfg.group > 8) return RKV_ERR_UNSUPPORTED;
  const int U = b->num_units;
  if (U == 0) return RKV_OK;
  // scratch, on first use: logits [max_tokens x GP], per-unit chunk offsets,
  // per-chunk head statistics and energies
  const int GP = refree_padded_group(e->cfg.group);
  const int64_t max_ch = refree_max_chunks(e->cfg.max_tokens, e->cfg.max_units);
  const size_t z_bytes = round_up(sizeof(float) * static_cast<size_t>(e->cfg.max_tokens) * GP);
  const size_t off_bytes = round_up(sizeof(int) * (static_cast<size_t>(e->cfg.max_units) + 1));
  const size_t cs_bytes = round_up(sizeof(float2) * static_cast<size_t>(max_ch) * GP);
  const size_t ce_bytes = round_up(sizeof(float) * static_cast<size_t>(max_ch));
  if (!e->rf_z) {
    if (dev_alloc(&e->fault, reinterpret_cast<void**>(&e->rf_z),
                  z_bytes + off_bytes + cs_bytes + ce_bytes) != cudaSuccess) {
      cudaGetLastError();
      e->rf_z = nullptr;
      return RKV_ERR_OOM;
    }
  }
  int64_t nchunks = 0;
  for (int u = 0; u < U; ++u)
    nchunks += (b->tok_off_host[u + 1] - b->tok_off_host[u] + kRfChunk - 1) / kRfChunk;
  uint8_t* scr = reinterpret_cast<uint8_t*>(e->rf_z);
  RefreeArgs ra;
  ra.tok_off = b->tok_off;
  ra.U = U;
  ra.nchunks = nchunks;
  ra.G = e->cfg.group;
  ra.w = e->cfg.window;
  ra.Q = b->Q;
  ra.K = b->K;
  ra.sinks = sinks;
  ra.T = T;
  ra.max_budget = max_budget;
  ra.zbuf = reinterpret_cast<float*>(scr);
  ra.chunk_off = reinterpret_cast<int*>(scr + z_bytes);
  ra.cstat = reinterpret_cast<float2*>(scr + z_bytes + off_bytes);
  ra.cenergy = reinterpret_cast<float*>(scr + z_bytes + off_bytes + cs_bytes);
  ra.p_last = p_last;
  ra.budgets = budgets;
  ra.keep_count = keep_count;
  ra.nsm = e->nsm;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  t_begin(e, RKV_KERNEL_REFREE, st);
  cudaError_t err = launch_refree(ra, st);
  t_end(e, st);
  if (err != cudaSuccess) return cuda_fail(err);
  e->launches += nchunks > 0 ? 4 : 1;
  return RKV_OK;
}

int rkv_compress(rkv_engine* e, const rkv_batch* b, float lambda, int budget, float* a, float* r,
                 int32_t* idx, int32_t* n_kept, void* K_out, void* V_out, rkv_stream_t stream) {
  NvtxRange nvtx_("rkv_compress");
  if (!e) return RKV_ERR_INVALID_ARG;
  // validate everything before enqueuing anything
  int64_t T = 0;
  int nmax = 0, cmax = 0;
  int rc = check_batch(e, b, &T, &nmax, &cmax);
  if (rc != RKV_OK) return rc;
  if (!(lambda >= 0.f && lambda <= 1.f) || budget < 0 || !a || !r || !idx || !n_kept ||
      !K_out || !V_out || !b->K || !b->V || !b->Q)
    return RKV_ERR_INVALID_ARG;
  if (!aligned(b->V, 16) || !aligned(K_out, 16) || !aligned(V_out, 16))
    return RKV_ERR_INVALID_ARG;
  rc = rkv_score(e, b, a, r, nullptr, stream);
  if (rc != RKV_OK) return rc;
  rc = rkv_select(e, b, a, r, lambda, budget, idx, n_kept, stream);
  if (rc != RKV_OK) return rc;
  return rkv_compact(e, b, idx, n_kept, budget, K_out, V_out, stream);
}

int rkv_debug_intermediates(rkv_engine* e, const rkv_batch* b, float* rho, float* U_out,
                            rkv_stream_t stream) {
  NvtxRange nvtx_("rkv_debug_intermediates");
  if (!e) return RKV_ERR_INVALID_ARG;
  int64_t T = 0;
  int nmax = 0, cmax = 0;
  int rc = check_batch(e, b, &T, &nmax, &cmax);
  if (rc != RKV_OK) return rc;
  if ((rho && !aligned(rho, 4)) || (U_out && !aligned(U_out, 4))) return RKV_ERR_INVALID_ARG;
  const bool closed = e->cfg.redundancy == RKV_REDUNDANCY_CLOSED_FORM;
  if ((rho && closed) || (U_out && !closed)) return RKV_ERR_UNSUPPORTED;
  const int U = b->num_units;
  if (U == 0) return RKV_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t err = cudaSuccess;
  if (rho) err = launch_gather_rho(b->tok_off, e->rho_off, U, e->rho, rho, st);
  if (err == cudaSuccess && U_out)
    err = launch_sum_unit_U(e->chunk_off, U, e->xstat, score_xs(e->rp, true), 2 * e->rp, U_out,
                            st);
  if (err != cudaSuccess) return cuda_fail(err);
  e->launches += (rho ? 1 : 0) + (U_out ? 1 : 0);
  return RKV_OK;
}

int rkv_check_status(rkv_engine* e, rkv_stream_t stream) {
  NvtxRange nvtx_("rkv_check_status");
  if (!e) return RKV_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return cuda_fail(cudaErrorUnknown);
  int h = 0;
  if (cudaMemcpy(&h, e->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return cuda_fail(cudaErrorUnknown);
  if (h != 0 && cudaMemset(e->status, 0, sizeof(int)) != cudaSuccess)
    return cuda_fail(cudaErrorUnknown);
  if (h & kStatusTimeout) return RKV_ERR_TIMEOUT;
  if (h & kStatusBadIndex) return RKV_ERR_DEVICE;
  if (h != 0) return RKV_ERR_CUDA;
  return RKV_OK;
}

}  // extern "C"
