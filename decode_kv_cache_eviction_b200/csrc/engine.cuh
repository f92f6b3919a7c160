// Engine object behind the opaque rkv_engine handle (shared by the C ABI
// translation units; not part of the public header).
#pragma once
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "../../include/rkv.h"

// Device staging of one chunk of the host-buffer pipeline (rkv_compress_host).
struct rkv_host_slot {
  void* K = nullptr;         // bf16 [cap_tokens, d]
  void* V = nullptr;
  void* Q = nullptr;         // bf16 [cap_units, G*w, d]
  int64_t* off = nullptr;    // [cap_units + 1] chunk-relative row offsets
  int32_t* idx = nullptr;    // [cap_tokens]: idx of the chunk, units * (budget + w) entries
  int32_t* nk = nullptr;     // [cap_units]
  void* Ko = nullptr;        // bf16 [cap_tokens, d]: compacted K of the chunk
  void* Vo = nullptr;
};

struct rkv_engine {
  rkv_config cfg;
  int device = 0;
  int nsm = 0;
  int rp = 32;                 // padded query rows per score launch (16, 32, 64)
  int nstages = 0;             // score K-tile ring depth
  int score_smem = 0;
  int score_ctas = 0;          // persistent score grid (one CTA per SM)
  int score_tpc_fixed = 0;     // > 0: score chunk size set by rkv_compress_host
  int max_n = 0;               // largest supported N_u
  int64_t max_chunks = 0;      // score chunks the exchange workspace holds
  bool pair = true;
  bool rowmax = false;   // row-max redundancy epilogue
  bool sym = false;      // symmetric GEMM (tiles on and above the diagonal)
  int gemm_ctas = 0;
  float* rho = nullptr;        // [max_tokens + kRhoAlign * max_units] padded 1/||k||
  int64_t* rho_off = nullptr;  // [max_units + 1]
  int* item_off = nullptr;     // [max_units + 1]
  int* unit_cnt = nullptr;     // [max_units]
  int* status = nullptr;       // [1]
  int* chunk_off = nullptr;    // [max_units + 1] score chunks prefix
  int* chunk_unit = nullptr;   // [max_chunks] unit of each score chunk
  int* score_cnt = nullptr;    // [max_units * kScoreCnt] score exchange counters
  float* xstat = nullptr;      // [max_chunks * score_xs] score chunk statistics
  float* xsum = nullptr;       // [max_chunks * 2 * kScoreMaxGroups] score chunk sums
  int64_t* cs_off = nullptr;   // [max_units + 1] symmetric form: scratch offsets
  float* cs = nullptr;         // symmetric form: partial sums, sized at creation
  int64_t cs_cap = 0;          // floats allocated in cs
  uint64_t wait_ns = 2000000000ull;   // limit of a score wait on another CTA
  int fault = 0;               // RKV_FAULT_* armed by rkv_inject_fault
  int64_t launches = 0;
  PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  // per-kernel timing (rkv_set_timing)
  static constexpr int kMaxEv = 4096;
  bool timing = false;
  cudaEvent_t ev[kMaxEv][2] = {};
  int ev_kernel[kMaxEv] = {};
  int nev = 0;
  bool ev_made = false;
  // host-buffer pipeline: two staging slots, shared score scratch, pinned
  // chunk offsets, copy-in / compute / copy-out streams and their events;
  // created on first use by rkv_compress_host
  rkv_host_slot hslot[2];
  float* h_a = nullptr;        // [hcap_tokens]
  float* h_r = nullptr;
  int64_t hcap_tokens = 0;
  int hcap_units = 0;
  int64_t* h_off_pinned = nullptr;   // host, page-locked
  int64_t h_off_cap = 0;
  cudaStream_t hs[3] = {};           // copy-in, compute, copy-out
  cudaEvent_t h_start = nullptr, h_done = nullptr;
  cudaEvent_t h_in[2] = {}, h_comp[2] = {}, h_out[2] = {};
  bool h_made = false;
  // rkv_refree_budget's logit scratch (max_tokens x padded G floats), on first use
  float* rf_z = nullptr;
};

// Frees everything rkv_compress_host allocated (called by rkv_destroy).
void rkv_host_pipeline_free(rkv_engine* e);

// cudaMalloc for the engine's lazily grown buffers; fails (once) when an
// allocation fault has been armed with rkv_inject_fault.
cudaError_t rkv_engine_alloc(rkv_engine* e, void** p, size_t bytes);
