// rkv_compress_host: the whole path from host buffers to host buffers, with
// copy-in, compute and copy-out of consecutive chunks overlapped.
//
// Chunk i uses staging slot i % 2.  Three internal streams carry the work:
//   copy-in  : [wait compute(i-2) done] K, V, Q, offsets -> slot      [in(i)]
//   compute  : [wait in(i), copy-out(i-2) done] score, select, compact [comp(i)]
//   copy-out : [wait comp(i)] idx, n_kept, K_out, V_out -> host        [out(i)]
// Compute is serial on its stream, so the engine's workspace and the shared
// score scratch are never used by two chunks at once.
//
// V is needed only for the kept rows (B + w of each unit's N).  When the
// caller's V is page-locked and mapped into the device address space (every
// cudaHostAlloc / cudaMallocHost allocation on a 64-bit system with unified
// addressing), the compaction kernel gathers the kept rows straight from host
// memory and V is never copied in whole; otherwise each chunk's V is copied
// like K.  Every kernel works per unit and every chunk scores with the
// chunk size of the whole batch, so a chunk's results do not depend on how
// the units were split: the outputs equal those of one rkv_compress over the
// whole batch.
#include <algorithm>
#include <cstring>
#include <vector>

#include "engine.cuh"
#include "rkv_internal.cuh"

namespace {

constexpr int64_t kDefaultChunk = int64_t{1} << 20;
constexpr int64_t kRowBytes = 128 * 2;   // one bf16 row of d = 128

void free_slots(rkv_engine* e) {
  for (auto& s : e->hslot) {
    cudaFree(s.K);
    cudaFree(s.V);
    cudaFree(s.Q);
    cudaFree(s.off);
    cudaFree(s.idx);
    cudaFree(s.nk);
    cudaFree(s.Ko);
    cudaFree(s.Vo);
    s = rkv_host_slot();
  }
  cudaFree(e->h_a);
  cudaFree(e->h_r);
  e->h_a = e->h_r = nullptr;
  e->hcap_tokens = 0;
  e->hcap_units = 0;
}

int make_streams(rkv_engine* e) {
  if (e->h_made) return RKV_OK;
  bool ok = true;
  for (auto& s : e->hs) ok = ok && cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) == cudaSuccess;
  cudaEvent_t* evs[] = {&e->h_start, &e->h_done, &e->h_in[0], &e->h_in[1],
                        &e->h_comp[0], &e->h_comp[1], &e->h_out[0], &e->h_out[1]};
  for (auto* ev : evs)
    ok = ok && cudaEventCreateWithFlags(ev, cudaEventDisableTiming) == cudaSuccess;
  e->h_made = true;   // partial creations are released by rkv_host_pipeline_free
  if (!ok) {
    cudaGetLastError();
    return RKV_ERR_CUDA;
  }
  return RKV_OK;
}

// Grow the device staging to hold chunks of `tokens` rows and `units` units.
int reserve_slots(rkv_engine* e, int64_t tokens, int units) {
  if (tokens <= e->hcap_tokens && units <= e->hcap_units) return RKV_OK;
  tokens = std::max(tokens, e->hcap_tokens);
  units = std::max(units, e->hcap_units);
  if (e->h_made && cudaEventSynchronize(e->h_done) != cudaSuccess) {
    cudaGetLastError();
    return RKV_ERR_CUDA;
  }
  free_slots(e);
  const int64_t R = static_cast<int64_t>(e->cfg.group) * e->cfg.window;
  bool ok = true;
  // an armed allocation fault (rkv_inject_fault) fails the first of these
  ok = rkv_engine_alloc(e, &e->hslot[0].K, tokens * kRowBytes) == cudaSuccess;
  for (auto& s : e->hslot) {
    if (!s.K) ok = ok && cudaMalloc(&s.K, tokens * kRowBytes) == cudaSuccess;
    ok = ok && cudaMalloc(&s.V, tokens * kRowBytes) == cudaSuccess;
    ok = ok && cudaMalloc(&s.Q, units * R * kRowBytes) == cudaSuccess;
    ok = ok && cudaMalloc(&s.off, (units + 1) * sizeof(int64_t)) == cudaSuccess;
    ok = ok && cudaMalloc(&s.idx, tokens * sizeof(int32_t)) == cudaSuccess;
    ok = ok && cudaMalloc(&s.nk, units * sizeof(int32_t)) == cudaSuccess;
    ok = ok && cudaMalloc(&s.Ko, tokens * kRowBytes) == cudaSuccess;
    ok = ok && cudaMalloc(&s.Vo, tokens * kRowBytes) == cudaSuccess;
  }
  ok = ok && cudaMalloc(&e->h_a, tokens * sizeof(float)) == cudaSuccess;
  ok = ok && cudaMalloc(&e->h_r, tokens * sizeof(float)) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    free_slots(e);
    return RKV_ERR_OOM;
  }
  e->hcap_tokens = tokens;
  e->hcap_units = units;
  return RKV_OK;
}

int reserve_pinned(rkv_engine* e, int64_t n) {
  if (n <= e->h_off_cap) return RKV_OK;
  cudaFreeHost(e->h_off_pinned);
  e->h_off_pinned = nullptr;
  e->h_off_cap = 0;
  if (cudaHostAlloc(reinterpret_cast<void**>(&e->h_off_pinned), n * sizeof(int64_t),
                    cudaHostAllocDefault) != cudaSuccess) {
    cudaGetLastError();
    return RKV_ERR_OOM;
  }
  e->h_off_cap = n;
  return RKV_OK;
}

struct Chunk {
  int u0, nu;         // first unit, unit count
  int64_t r0, rows;   // first row, row count
  int64_t off_at;     // position of its relative offsets in the pinned array
};

}  // namespace

void rkv_host_pipeline_free(rkv_engine* e) {
  free_slots(e);
  cudaFreeHost(e->h_off_pinned);
  e->h_off_pinned = nullptr;
  e->h_off_cap = 0;
  if (!e->h_made) return;
  for (auto& s : e->hs)
    if (s) cudaStreamDestroy(s);
  cudaEvent_t evs[] = {e->h_start, e->h_done, e->h_in[0], e->h_in[1],
                       e->h_comp[0], e->h_comp[1], e->h_out[0], e->h_out[1]};
  for (auto ev : evs)
    if (ev) cudaEventDestroy(ev);
  e->h_made = false;
}

extern "C" int rkv_compress_host(rkv_engine* e, const rkv_host_batch* hb, float lambda,
                                 int budget, int32_t* idx, int32_t* n_kept, void* K_out,
                                 void* V_out, int64_t chunk_tokens, rkv_stream_t stream) {
  rkv::NvtxRange nvtx_("rkv_compress_host");
  if (!e || !hb) return RKV_ERR_INVALID_ARG;
  const int U = hb->num_units;
  const int w = e->cfg.window;
  if (U < 0 || !hb->tok_off || chunk_tokens < 0) return RKV_ERR_INVALID_ARG;
  if (!(lambda >= 0.f && lambda <= 1.f) || budget < 0) return RKV_ERR_INVALID_ARG;
  if (U == 0) return RKV_OK;
  if (!hb->K || !hb->V || !hb->Q || !idx || !n_kept || !K_out || !V_out)
    return RKV_ERR_INVALID_ARG;
  // the whole batch is checked before anything is enqueued
  const int64_t* off = hb->tok_off;
  if (off[0] != 0) return RKV_ERR_INVALID_ARG;
  int64_t nmax = 0;
  for (int u = 0; u < U; ++u) {
    const int64_t n = off[u + 1] - off[u];
    if (n < w) return RKV_ERR_INVALID_ARG;
    if (n > e->max_n) return RKV_ERR_UNSUPPORTED;
    nmax = std::max(nmax, n);
  }
  const int64_t W = static_cast<int64_t>(budget) + w;   // output rows per unit
  if (W >= (int64_t{1} << 30)) return RKV_ERR_UNSUPPORTED;
  int64_t cap = chunk_tokens > 0 ? chunk_tokens : kDefaultChunk;
  cap = std::max(cap, std::max(nmax, W));
  if (cap > e->cfg.max_tokens) {
    if (std::max(nmax, W) > e->cfg.max_tokens) return RKV_ERR_CAPACITY;
    cap = e->cfg.max_tokens;
  }
  // chunks: consecutive units while rows, output rows and unit count fit
  std::vector<Chunk> chunks;
  int max_units = 0;
  for (int u = 0; u < U;) {
    Chunk c{u, 0, off[u], 0, 0};
    while (u < U && c.nu < e->cfg.max_units) {
      const int64_t n = off[u + 1] - off[u];
      if (c.nu > 0 && (c.rows + n > cap || (c.nu + 1) * W > cap)) break;
      c.rows += n;
      ++c.nu;
      ++u;
    }
    max_units = std::max(max_units, c.nu);
    chunks.push_back(c);
  }
  const int64_t npin = U + static_cast<int64_t>(chunks.size());
  if (npin >= (int64_t{1} << 31)) return RKV_ERR_UNSUPPORTED;

  // every chunk scores with the chunk size of the whole batch, so each unit's
  // partial sums are grouped as rkv_compress on the batch groups them
  rkv::ScoreDims whole;
  if (!rkv::score_plan(e->cfg.group * w, off, U, e->score_ctas, 0, &whole))
    return RKV_ERR_UNSUPPORTED;

  int rc = make_streams(e);
  if (rc != RKV_OK) return rc;
  // the previous call may still be reading the pinned offsets or the slots
  if (cudaEventSynchronize(e->h_done) != cudaSuccess) {
    cudaGetLastError();
    return RKV_ERR_CUDA;
  }
  int64_t rows_cap = 0;
  for (const Chunk& c : chunks) rows_cap = std::max(rows_cap, std::max(c.rows, c.nu * W));
  rc = reserve_slots(e, rows_cap, max_units);
  if (rc != RKV_OK) return rc;
  rc = reserve_pinned(e, npin);
  if (rc != RKV_OK) return rc;
  int64_t at = 0;
  for (Chunk& c : chunks) {
    c.off_at = at;
    for (int k = 0; k <= c.nu; ++k) e->h_off_pinned[at + k] = off[c.u0 + k] - c.r0;
    at += c.nu + 1;
  }

  const int64_t R = static_cast<int64_t>(e->cfg.group) * w;
  // device view of a page-locked, mapped V (nullptr: copy V chunk by chunk)
  const char* dV = nullptr;
  {
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, hb->V) == cudaSuccess) {
      if (pa.type == cudaMemoryTypeHost && pa.devicePointer != nullptr)
        dV = static_cast<const char*>(pa.devicePointer);
    } else {
      cudaGetLastError();   // pageable memory unknown to CUDA: copy it
    }
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t s_in = e->hs[0], s_comp = e->hs[1], s_out = e->hs[2];
  auto fail = [&](cudaError_t err) {
    (void)err;
    cudaGetLastError();
    // leave the internal streams ordered behind everything enqueued so far
    cudaEventRecord(e->h_done, s_out);
    return RKV_ERR_CUDA;
  };
  if (cudaEventRecord(e->h_start, st) != cudaSuccess) return fail(cudaErrorUnknown);
  for (cudaStream_t s : e->hs)
    if (cudaStreamWaitEvent(s, e->h_start, 0) != cudaSuccess) return fail(cudaErrorUnknown);

  const char* hK = static_cast<const char*>(hb->K);
  const char* hV = static_cast<const char*>(hb->V);
  const char* hQ = static_cast<const char*>(hb->Q);
  struct FixedChunk {
    rkv_engine* e;
    FixedChunk(rkv_engine* en, int tpc) : e(en) { e->score_tpc_fixed = tpc; }
    ~FixedChunk() { e->score_tpc_fixed = 0; }
  } fixed_tpc(e, whole.tpc);
  for (size_t i = 0; i < chunks.size(); ++i) {
    const Chunk& c = chunks[i];
    const int s = static_cast<int>(i & 1);
    rkv_host_slot& sl = e->hslot[s];
    // copy-in
    if (i >= 2 && cudaStreamWaitEvent(s_in, e->h_comp[s], 0) != cudaSuccess)
      return fail(cudaErrorUnknown);
    cudaError_t err = cudaMemcpyAsync(sl.K, hK + c.r0 * kRowBytes, c.rows * kRowBytes,
                                      cudaMemcpyHostToDevice, s_in);
    if (err == cudaSuccess && !dV)
      err = cudaMemcpyAsync(sl.V, hV + c.r0 * kRowBytes, c.rows * kRowBytes,
                            cudaMemcpyHostToDevice, s_in);
    if (err == cudaSuccess)
      err = cudaMemcpyAsync(sl.Q, hQ + c.u0 * R * kRowBytes, c.nu * R * kRowBytes,
                            cudaMemcpyHostToDevice, s_in);
    if (err == cudaSuccess)
      err = cudaMemcpyAsync(sl.off, e->h_off_pinned + c.off_at, (c.nu + 1) * sizeof(int64_t),
                            cudaMemcpyHostToDevice, s_in);
    if (err == cudaSuccess) err = cudaEventRecord(e->h_in[s], s_in);
    if (err != cudaSuccess) return fail(err);
    // compute
    if (cudaStreamWaitEvent(s_comp, e->h_in[s], 0) != cudaSuccess ||
        (i >= 2 && cudaStreamWaitEvent(s_comp, e->h_out[s], 0) != cudaSuccess))
      return fail(cudaErrorUnknown);
    rkv_batch b;
    b.num_units = c.nu;
    b.tok_off = sl.off;
    b.tok_off_host = e->h_off_pinned + c.off_at;
    b.K = sl.K;
    b.V = dV ? static_cast<const void*>(dV + c.r0 * kRowBytes) : sl.V;
    b.Q = sl.Q;
    rc = rkv_compress(e, &b, lambda, budget, e->h_a, e->h_r, sl.idx, sl.nk, sl.Ko, sl.Vo,
                      reinterpret_cast<rkv_stream_t>(s_comp));
    if (rc != RKV_OK) {
      cudaEventRecord(e->h_done, s_out);
      return rc;
    }
    if (cudaEventRecord(e->h_comp[s], s_comp) != cudaSuccess) return fail(cudaErrorUnknown);
    // copy-out
    if (cudaStreamWaitEvent(s_out, e->h_comp[s], 0) != cudaSuccess) return fail(cudaErrorUnknown);
    err = cudaMemcpyAsync(idx + c.u0 * W, sl.idx, c.nu * W * sizeof(int32_t),
                          cudaMemcpyDeviceToHost, s_out);
    if (err == cudaSuccess)
      err = cudaMemcpyAsync(n_kept + c.u0, sl.nk, c.nu * sizeof(int32_t), cudaMemcpyDeviceToHost,
                            s_out);
    if (err == cudaSuccess)
      err = cudaMemcpyAsync(static_cast<char*>(K_out) + c.u0 * W * kRowBytes, sl.Ko,
                            c.nu * W * kRowBytes, cudaMemcpyDeviceToHost, s_out);
    if (err == cudaSuccess)
      err = cudaMemcpyAsync(static_cast<char*>(V_out) + c.u0 * W * kRowBytes, sl.Vo,
                            c.nu * W * kRowBytes, cudaMemcpyDeviceToHost, s_out);
    if (err == cudaSuccess) err = cudaEventRecord(e->h_out[s], s_out);
    if (err != cudaSuccess) return fail(err);
  }
  // the caller's stream continues after the last copy-out (which follows the
  // last compute and, through the slot events, every copy-in)
  if (cudaEventRecord(e->h_done, s_out) != cudaSuccess ||
      cudaStreamWaitEvent(st, e->h_done, 0) != cudaSuccess)
    return fail(cudaErrorUnknown);
  return RKV_OK;
}
