/*
 * rkv.h -- C ABI of the decode-time KV-cache compression engine (R-KV hot path)
 * for NVIDIA B200 (sm_100a).
 *
 * Method: the R-KV article (QbitAI repost, section "R-KV三步走：冗余识别+重要性评估+
 * 动态淘汰").  While decoding, each (sequence, layer, KV head) cache is scored by
 *   - importance (重要性打分): attention that the last w decode queries pay to each
 *     cached token, softmax per query, averaged over the window and the GQA group;
 *   - redundancy (冗余打分): cosine similarity between each key and all other cached
 *     keys, averaged over the row (diagonal excluded), then a softmax over tokens;
 * and the joint eviction step (联合淘汰: high importance, low redundancy, lambda ~ 0.1)
 * keeps the last w tokens plus the top-B of the rest and compacts K/V into a B+w
 * slot buffer (gather compaction, named as the R-KV-style baseline in the ThinKV
 * summary, "Continuous Thinking" section).
 *
 * Limits: head_dim = 128, G*w <= 256 (up to 32 query rows per pass over K; more
 * rows take several passes), N_u <= 131072.
 *
 * Terms used below.  A *unit* is one (sequence, layer, KV head).  Unit u has
 * N_u cached tokens, stored as rows tok_off[u] .. tok_off[u+1]-1 of K and V.
 * d = head_dim (= 128), G = query heads per KV head, w = window.  Query (g, t)
 * of unit u is Q[u][g][t][:] and sits at position N_u - w + t; it attends to
 * keys 0 .. N_u - w + t.  The candidates are C_u = {0 .. N_u - w - 1}.
 *
 * Conventions (every call):
 *   - All data pointers are DEVICE pointers, owned by the caller, unless the
 *     parameter says "host".  Inputs are read only.  K, V, Q, K_out, V_out
 *     must be 16-byte aligned; float/int32 arrays 4-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t) and never synchronise
 *     the host, except rkv_check_status.  They never throw.
 *   - Return value: RKV_OK (0) or a negative RKV_ERR_* code.  Arguments are
 *     validated on the host before anything is enqueued; on an error nothing is
 *     enqueued.  Faults found on the device (a wait that timed out, a kept index
 *     outside its unit) are recorded in the engine's device status word and
 *     reported by rkv_check_status.
 *   - One engine may be used from one host thread at a time.  Calls that share
 *     an engine must be ordered on one stream (the engine's workspace is reused).
 */
#ifndef RKV_H_
#define RKV_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* rkv_stream_t; /* identical to cudaStream_t */
typedef struct rkv_engine rkv_engine;     /* opaque; owns its workspace and staging */

enum {
  RKV_OK = 0,
  RKV_ERR_INVALID_ARG = -1, /* null/unaligned pointer, bad size, N_u < w, ... */
  RKV_ERR_UNSUPPORTED = -2, /* head_dim != 128, G*w > 256, N_u too long, not sm_100 */
  RKV_ERR_CUDA = -3,        /* a CUDA runtime call or launch failed */
  RKV_ERR_TIMEOUT = -4,     /* a device-side wait ran out of time (see rkv_check_status) */
  RKV_ERR_OOM = -5,         /* workspace allocation failed */
  RKV_ERR_CAPACITY = -6,    /* batch larger than the engine's max_units / max_tokens */
  RKV_ERR_DEVICE = -7       /* a kept index outside its unit (see rkv_check_status) */
};

/* How rkv_score computes the redundancy m_i. */
enum {
  /* Tensor-core K K^T tile products with the norm scaling, diagonal mask,
   * row mean and token softmax fused into the epilogue (N x N never stored). */
  RKV_REDUNDANCY_GEMM = 0,
  /* The same m_i by linearity of the row sum:
   * sum_{j != i} khat_i . khat_j = khat_i . (sum_j khat_j) - khat_i . khat_i. */
  RKV_REDUNDANCY_CLOSED_FORM = 1,
  /* Nearest-duplicate reading of the cosine-similarity redundancy (R-KV,
   * "冗余打分"): m_i = max_{j != i, j < N} khat_i . khat_j, from the same
   * tensor-core tiles with a max fold in the epilogue.  A token with an exact
   * copy anywhere in the unit gets m_i = 1. */
  RKV_REDUNDANCY_MAX = 2
};

typedef struct {
  int head_dim;       /* d; must be 128 */
  int group;          /* G >= 1: query heads per KV head */
  int window;         /* w >= 1: window queries and always-kept tail tokens */
  int max_units;      /* capacity: units per batch (>= 1) */
  int64_t max_tokens; /* capacity: total cached rows per batch (>= 1) */
  int redundancy;     /* RKV_REDUNDANCY_GEMM, _CLOSED_FORM or _MAX */
  int flags;          /* 0, or RKV_FLAG_* bits */
  int64_t max_unit_tokens; /* capacity: longest unit N_u (0: the engine's limit);
                              sizes the symmetric GEMM's scratch */
} rkv_config;

/* rkv_config.flags */
enum {
  /* Redundancy GEMM on single CTAs (M = 128 tcgen05 MMAs) instead of CTA
   * pairs (M = 256, cta_group::2).  Same results; slower. */
  RKV_FLAG_GEMM_SINGLE_CTA = 1,
  /* Row-mean GEMM on the tiles on and above the diagonal only: S is symmetric,
   * so tile (a, b > a) gives block a its row sums and block b its column sums
   * (rho-weighted, reduced on CUDA cores).  Every partial sum is written once
   * to a scratch, and a finish kernel adds the parts in a fixed order.  About
   * half the MMA work; same results up to fp32 rounding order, and
   * deterministic.  CTA pairs and RKV_REDUNDANCY_GEMM only
   * (RKV_ERR_UNSUPPORTED otherwise).  The scratch (128 nb (nb + 3) fp32 for a
   * unit of nb = ceil(N_u / 256) blocks, about N_u^2 / 128 bytes) is allocated
   * by rkv_create for the largest batch the capacities allow (max_tokens in
   * units of max_unit_tokens) and freed by rkv_destroy; rkv_score allocates
   * nothing. */
  RKV_FLAG_GEMM_SYMMETRIC = 2
};

typedef struct {
  int num_units;               /* U, 0 <= U <= max_units */
  const int64_t* tok_off;      /* device [U+1]: row offsets, tok_off[0] = 0, nondecreasing */
  const int64_t* tok_off_host; /* HOST copy of the same [U+1] values (validation, sizing) */
  const void* K;               /* device bf16 [T, d] row-major keys, T = tok_off[U] */
  const void* V;               /* device bf16 [T, d] row-major values */
  const void* Q;               /* device bf16 [U, G, w, d]: window queries (post-RoPE) */
} rkv_batch;

/* Create an engine and allocate its device workspace on the current device.
 * Fails with RKV_ERR_UNSUPPORTED on a device that is not sm_100, or when
 * max_unit_tokens exceeds the engine's limit; RKV_ERR_OOM when the workspace
 * cannot be allocated (nothing is kept then). */
int rkv_create(const rkv_config* cfg, rkv_engine** out);

/* Free the workspace (waits for the device to finish using it). NULL is a no-op. */
int rkv_destroy(rkv_engine* eng);

/* Importance and redundancy scores (R-KV 重要性打分 and 冗余打分).
 *   a [T] fp32: a_i = abar_i / sum_{j in C} abar_j for i in C, where
 *               abar_i = mean over (g, t) of softmax_j(q_{g,t} . k_j / sqrt(d))[i];
 *   r [T] fp32: r_i = exp(m_i) / sum_{j in C} exp(m_j) for i in C, where
 *               m_i = sum_{j != i, j < N} khat_i . khat_j / (N - 1)
 *               (RKV_REDUNDANCY_MAX: m_i = max_{j != i, j < N} khat_i . khat_j),
 *               khat = k / ||k|| (0 for a zero key);
 *   m [T] fp32, optional (NULL to skip): the m_i.
 * Row tok_off[u] + i holds token i of unit u; window rows (i >= N_u - w) are 0.
 * Allocates nothing and never synchronises the host.  The kernels exchange
 * per-chunk statistics through the engine's workspace and wait on each other
 * with a bounded wait; a wait that runs out sets RKV_ERR_TIMEOUT in the status
 * word (rkv_check_status).  RKV_ERR_UNSUPPORTED for a unit longer than the
 * engine's limit; RKV_ERR_CAPACITY for a batch beyond its capacities. */
int rkv_score(rkv_engine* eng, const rkv_batch* batch, float* a, float* r, float* m,
              rkv_stream_t stream);

/* Joint eviction (R-KV 联合淘汰): s_i = lambda * a_i - (1 - lambda) * r_i for i in C
 * (fp32); keep the min(budget, N_u - w) candidates ranked first by (s descending,
 * index ascending), in ascending index order, followed by the window
 * N_u - w .. N_u - 1.  -0 and +0 tie; a NaN score ranks below every number.
 * When N_u - w <= budget every token 0 .. N_u - 1 is kept.
 *   idx [U, budget + w] int32: kept token indices (unit-local); unused slots -1;
 *   n_kept [U] int32: number of valid slots of each unit.
 * lambda must lie in [0, 1]; budget >= 0. */
int rkv_select(rkv_engine* eng, const rkv_batch* batch, const float* a, const float* r,
               float lambda, int budget, int32_t* idx, int32_t* n_kept, rkv_stream_t stream);

/* rkv_select with attention sinks and per-unit budgets (sinks: the ReFreeKV
 * review's anchor tokens; per-head budgets: LU-KV; an adaptive budget from
 * rkv_refree_budget).  For unit u with c = N_u - w candidates, m = min(sinks, c)
 * and B_u = budgets ? clamp(budgets[u], 0, budget) : budget:
 *   - if c - m <= B_u, every token 0 .. N_u - 1 is kept;
 *   - else tokens 0 .. m-1 (always), then the B_u best of candidates m .. c-1
 *     by (s descending, index ascending) in ascending order, then the window.
 *   idx [U, W] int32 with W = budget + sinks + w; entries past n_kept[u] are -1.
 *   budgets: device [U] int32 or NULL.
 * For rkv_compact / rkv_evict_in_place on this idx, pass budget + sinks as
 * their budget (same row stride).  sinks = 0 and budgets = NULL is rkv_select. */
int rkv_select_ex(rkv_engine* eng, const rkv_batch* batch, const float* a, const float* r,
                  float lambda, int budget, const int32_t* budgets, int sinks, int32_t* idx,
                  int32_t* n_kept, rkv_stream_t stream);

/* Adaptive per-unit budget (the ReFreeKV review: initial ranking + Uni-Metric
 * stop, with k = 1 and threshold T, e.g. 0.01).
 *   p_last [T] fp32 (output): p_j = mean over the G heads of the newest query's
 *     attention softmax_j(q_{g, w-1} . k_j / sqrt(d)), over all N_u keys;
 *   keep_count [U] int32 (output, may be NULL): the smallest k such that the
 *     first k tokens of the ranking (tokens 0 .. m-1, m = min(sinks, N_u), then
 *     N_u - 1, N_u - 2, ... down to m) hold sum p^2 >= (1 - T)^2 sum_all p^2,
 *     i.e. their Frobenius norm is at least (1 - T) of the row's;
 *   budgets [U] int32 (output): clamp(k - min(sinks, N_u - w) - w, 0,
 *     max_budget), the rkv_select_ex budget that keeps k tokens in all.
 * Computed in fp32; requires G <= 8 (RKV_ERR_UNSUPPORTED otherwise).  The
 * first call allocates a scratch, kept until rkv_destroy (RKV_ERR_OOM if that
 * fails): max_tokens x GP logit floats (GP = G rounded up to a power of two),
 * max_units + 1 chunk offsets, and per 2048-token chunk GP (max, sum) pairs and
 * one energy, for max_tokens / 2048 + max_units chunks. */
int rkv_refree_budget(rkv_engine* eng, const rkv_batch* batch, float T, int sinks,
                      int max_budget, float* p_last, int32_t* budgets, int32_t* keep_count,
                      rkv_stream_t stream);

/* Gather compaction: K_out[u][j] = K[tok_off[u] + idx[u][j]] (and V likewise) for
 * j < n_kept[u]; rows n_kept[u] .. budget + w - 1 are zero.  Bit-exact copies.
 *   K_out, V_out: device bf16 [U, budget + w, d] (must not overlap K, V).
 * An index outside 0 .. N_u - 1 zero-fills its row and sets RKV_ERR_DEVICE. */
int rkv_compact(rkv_engine* eng, const rkv_batch* batch, const int32_t* idx,
                const int32_t* n_kept, int budget, void* K_out, void* V_out,
                rkv_stream_t stream);

/* In-place slot reuse, the alternative to rkv_compact (the ThinKV summary's
 * Continuous Thinking: evicted slots are reused instead of compacted away).
 * Rows stay where they are; for unit u, with idx / n_kept as rkv_select wrote
 * them (row stride budget + w):
 *   keep [T] uint8: keep[tok_off[u] + i] = 1 if token i is kept, else 0;
 *   free_slots [T] int32: rows tok_off[u] .. tok_off[u] + n_free[u] - 1 hold the
 *     evicted token indices of unit u (unit-local) in ascending order; the rest
 *     of the unit's rows hold -1;
 *   n_free [U] int32: N_u minus the number of distinct kept indices.
 * Moves 1 + 4 bytes per cached token instead of rkv_compact's 4 d bytes per
 * kept token.  A kept index outside 0 .. N_u - 1 (or an n_kept outside
 * 0 .. budget + w) is ignored and sets RKV_ERR_DEVICE (see rkv_check_status). */
int rkv_evict_in_place(rkv_engine* eng, const rkv_batch* batch, const int32_t* idx,
                       const int32_t* n_kept, int budget, uint8_t* keep, int32_t* free_slots,
                       int32_t* n_free, rkv_stream_t stream);

/* New tokens overwrite evicted slots (Continuous Thinking).  New token t of
 * unit u, row new_off[u] + t of K_new / V_new (bf16 [new_off[U], d]), is written
 * to row tok_off[u] + free_slots[tok_off[u] + t] of K and V (the batch's
 * caches, passed again as writable pointers), lowest free slot first, and
 * marked live in keep.  The used slots leave the free list (the remaining ones
 * move to the front) and n_free[u] drops by the count.  new_off is device
 * [U+1] with a host copy new_off_host (new_off[0] = 0, nondecreasing).  A unit
 * with more new tokens than free slots takes n_free[u] of them and sets
 * RKV_ERR_DEVICE; a slot outside the unit is skipped and sets it too. */
int rkv_fill_slots(rkv_engine* eng, const rkv_batch* batch, void* K, void* V,
                   const int64_t* new_off, const int64_t* new_off_host, const void* K_new,
                   const void* V_new, uint8_t* keep, int32_t* free_slots, int32_t* n_free,
                   rkv_stream_t stream);

/* rkv_score, rkv_select and rkv_compact in one call.  a and r are caller-owned
 * scratch [T] fp32 (they hold the scores afterwards). */
int rkv_compress(rkv_engine* eng, const rkv_batch* batch, float lambda, int budget,
                 float* a, float* r, int32_t* idx, int32_t* n_kept, void* K_out,
                 void* V_out, rkv_stream_t stream);

/* A batch in HOST memory (rkv_compress_host).  Same layouts as rkv_batch. */
typedef struct {
  int num_units;               /* U >= 0 */
  const int64_t* tok_off;      /* host [U+1]: row offsets, tok_off[0] = 0, nondecreasing */
  const void* K;               /* host bf16 [T, d] keys */
  const void* V;               /* host bf16 [T, d] values */
  const void* Q;               /* host bf16 [U, G, w, d] window queries */
} rkv_host_batch;

/* rkv_compress from host buffers to host buffers (the path a caller with the
 * cache in host memory takes; the paper has no counterpart).  Units are cut
 * into chunks of at most `chunk_tokens` rows (0 selects 1,048,576; raised to the
 * longest unit and to budget + w if smaller) and at most max_units units, and
 * the chunks are pipelined through two device staging slots on three internal
 * streams: copy-in of chunk i+1, scoring / selection / compaction of chunk i and
 * copy-out of chunk i-1 overlap.  Results equal those of rkv_compress on the
 * same units, bit for bit.
 *   idx [U, budget + w] int32, n_kept [U] int32, K_out / V_out bf16
 *   [U, budget + w, d]: HOST outputs, laid out as for rkv_select / rkv_compact.
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister) for the
 * copies to overlap; pageable memory works but serialises them.  When V is
 * page-locked and mapped into the device address space (cudaHostAlloc on a
 * 64-bit system, or cudaHostRegister with cudaHostRegisterMapped), only the
 * kept V rows cross the bus: the compaction kernel reads them from host memory.  Everything is
 * ordered after earlier work on `stream`, and later work on `stream` runs after
 * the last copy-out; the host buffers must stay untouched until then (e.g.
 * until rkv_check_status(eng, stream) returns).  The staging (about
 * 4 * chunk_tokens * 512 bytes of device memory and U + chunks page-locked
 * int64) is allocated on the first call, grown when a call needs more, and
 * freed by rkv_destroy.  A call first waits on the host for the engine's
 * previous rkv_compress_host call to finish.  Not capturable in a CUDA graph.
 * Errors: those of rkv_compress (all validation happens before anything is
 * enqueued), RKV_ERR_CAPACITY when one chunk cannot fit the engine's
 * max_tokens, RKV_ERR_OOM when the staging cannot be allocated. */
int rkv_compress_host(rkv_engine* eng, const rkv_host_batch* batch, float lambda, int budget,
                      int32_t* idx, int32_t* n_kept, void* K_out, void* V_out,
                      int64_t chunk_tokens, rkv_stream_t stream);

/* Synchronise `stream`, then read and clear the engine's device status word:
 * RKV_OK, RKV_ERR_TIMEOUT (a device wait gave up; outputs are invalid) or
 * RKV_ERR_DEVICE (an out-of-range kept index reached rkv_compact). */
int rkv_check_status(rkv_engine* eng, rkv_stream_t stream);

/* Fault injection, for testing the error paths without faulting a GPU.
 *   RKV_FAULT_ALLOC: the engine's next device allocation fails (RKV_ERR_OOM);
 *     with eng = NULL, the next rkv_create's workspace allocation fails;
 *   RKV_FAULT_DROP_ANNOUNCE: in the next score launch one chunk does not
 *     announce its statistics, and the waits of that launch give up after
 *     50 ms, so rkv_check_status then reports RKV_ERR_TIMEOUT;
 *   RKV_FAULT_NONE: disarm.
 * A fault fires once.  Returns RKV_ERR_INVALID_ARG for an unknown fault. */
enum { RKV_FAULT_NONE = 0, RKV_FAULT_ALLOC = 1, RKV_FAULT_DROP_ANNOUNCE = 2 };
int rkv_inject_fault(rkv_engine* eng, int fault);

/* Intermediate arrays of the last rkv_score call on this engine, for checks
 * against their definitions.  batch must be the batch that call scored,
 * unchanged, and no other rkv_score call may run in between.
 *   rho: device [T] fp32 or NULL: rho_j = 1/||k_j|| (0 for a zero key) of every
 *        token, as the redundancy GEMM consumes it (GEMM modes only);
 *   U:   device [U, 128] fp32 or NULL: U = sum_j k_j/||k_j|| over each unit's
 *        N_u keys (closed-form redundancy only).
 * Asking for rho in the closed form or U in a GEMM mode returns
 * RKV_ERR_UNSUPPORTED.  Enqueued on stream; no allocation. */
int rkv_debug_intermediates(rkv_engine* eng, const rkv_batch* batch, float* rho, float* U,
                            rkv_stream_t stream);

/* Number of kernel launches enqueued by this engine since creation. */
int64_t rkv_launch_count(const rkv_engine* eng);

/* Kernels, for per-kernel timing. */
enum {
  RKV_KERNEL_SCORE = 0,   /* importance (+ closed-form redundancy) */
  RKV_KERNEL_PLAN = 1,    /* per-unit row-block offsets for the GEMM */
  RKV_KERNEL_GEMM = 2,    /* redundancy GEMM + fused epilogue + token softmax */
  RKV_KERNEL_SELECT = 3,  /* joint score + top-B */
  RKV_KERNEL_COMPACT = 4, /* K/V gather */
  RKV_KERNEL_EVICT = 5,   /* in-place eviction: keep mask and free slots */
  RKV_KERNEL_FILL = 6,    /* new tokens into free slots */
  RKV_KERNEL_REFREE = 7,  /* adaptive budget (newest query's attention row) */
  RKV_KERNEL_FINISH = 8,  /* symmetric GEMM form: partial sums -> m, token softmax -> r */
  RKV_NUM_KERNELS = 9
};

/* Per-kernel timing.  While enabled, the engine records a pair of CUDA events
 * on the launch stream around each of its kernel launches (up to 4096 pairs
 * between reads).  rkv_read_timing synchronises on those events and returns,
 * for `kernel`, the summed device time in milliseconds and the number of
 * launches recorded since timing was last set; reading drops nothing.
 * rkv_set_timing (either value) drops the recorded events, and
 * rkv_set_timing(eng, 0) also stops recording. */
int rkv_set_timing(rkv_engine* eng, int enable);
int rkv_read_timing(rkv_engine* eng, int kernel, double* total_ms, int64_t* launches);

/* Scoring without any device allocation (no engine object).
 *
 * The paper has no counterpart to this call; it exists for callers that cannot
 * allocate device memory themselves or through the library: serving stacks that
 * reserve nearly all HBM up front for their own KV block pool and hand out no
 * further memory, or host frameworks that load this library as a plug-in and
 * forbid it from calling cudaMalloc behind their allocator's back.
 *
 * Computes exactly what rkv_score computes for an engine created with
 * RKV_REDUNDANCY_GEMM (CTA-pair GEMM), with head_dim = 128 and the given group and
 * window.  Its scratch (1/||k|| per row, the score kernel's per-chunk exchange
 * slots and counters, per-unit offsets and counters, a status word) lives in one
 * file-scope __device__ array of about 11 MB that every GPU holding the
 * library's module keeps until the process exits; nothing is allocated or freed
 * per call.  Limits: G*w <= 32, N_u <= 131072, at most RKV_NOALLOC_MAX_UNITS
 * units and RKV_NOALLOC_MAX_TOKENS rows per call (larger batches return
 * RKV_ERR_CAPACITY, longer units or larger G*w RKV_ERR_UNSUPPORTED, before
 * anything is enqueued).
 *
 * The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) and sets kernel attributes with that device current.
 * Under CUDA's lazy module loading (the default) that lookup may be the moment
 * the module, and with it the array, is loaded into the device's memory: make
 * the first call on each device before reserving a memory pool that leaves no
 * room for it (it returns RKV_ERR_OOM when the array cannot be loaded), and
 * before any stream capture.  All calls share the one array and each call
 * rewrites what it reads, so successive calls on one stream are safe, but calls
 * that overlap on the GPU (other streams, other host threads without ordering)
 * race on it.  A device-side wait that times out leaves a bit in the array's
 * status word; rkv_noalloc_check_status reports and clears it. */
enum { RKV_NOALLOC_MAX_UNITS = 4096, RKV_NOALLOC_MAX_TOKENS = 1048576 };
int rkv_score_noalloc(int group, int window, const rkv_batch* batch, float* a, float* r,
                      float* m, rkv_stream_t stream);

/* Status of the rkv_score_noalloc calls on the current device: synchronises
 * `stream`, then reads and clears the status word of the device's static
 * scratch.  RKV_OK, RKV_ERR_TIMEOUT (a device wait gave up; the outputs of the
 * calls since the last check are invalid) or RKV_ERR_CUDA.  Allocates nothing;
 * RKV_OK when no call has run on the device yet. */
int rkv_noalloc_check_status(rkv_stream_t stream);

/* Static description of a status code. */
const char* rkv_status_string(int status);

/* ABI version (major * 10000 + minor * 100 + patch). */
int rkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RKV_H_ */
