// Internal definitions shared by the host layer and the kernels of the
// low-rank KV-cache decode library.  Not part of the C ABI.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <atomic>
#include <vector>

#include "lr_kv.h"

#define LR_LOG2E 1.4426950408889634f
#define LR_LN2 0.6931471805599453f

// Latent storage kinds.
enum LatentKind { LK_F32 = 0, LK_BF16 = 1, LK_INT4 = 2 };

// Int4 storage: blocks of 128 tokens, group-major inside a block.  A latent row is
// b * lat_cap + slot (lat_cap = capacity rounded up to 128), so row >> 7 is the block
// and row & 127 the token inside it.
constexpr int kI4Block = 128;
__host__ __device__ __forceinline__ long long i4_code_index(long long row, int G, int g, int w) {
  return ((((row >> 7) * G + g) << 9) + ((row & 127) << 2)) + w;
}
__host__ __device__ __forceinline__ long long i4_param_index(long long row, int G, int g) {
  return (((row >> 7) * G + g) << 7) + (row & 127);
}
// Values (V) are stored rank-major inside a block, so that the decode's value-mix operand
// (rank rows, token columns) is read one rank row per thread: rank i of a block holds 16
// words, each with eight tokens' codes; the 16-byte column c of the row holds tokens
// 32 (c ^ ((i / 2) % 4)) .. +31 (the XOR spreads the rows of consecutive ranks over the
// shared-memory banks), and token t sits in nibble ((t & 1) << 2) | ((t >> 1) & 3) of its
// word, so that the two nibbles (m, m + 4) of a word are two consecutive tokens.  The
// params of one (block, group) are 128 fp16 scales (tokens 0..127) then 128 fp16 zeros.
__host__ __device__ __forceinline__ long long i4v_code_index(long long row, int G, int i) {
  const int t = (int)(row & 127);
  return ((((row >> 7) * G) << 5) + i) * 16 + ((((t >> 5) ^ ((i >> 1) & 3))) << 2) + ((t & 31) >> 3);
}
__host__ __device__ __forceinline__ int i4v_nibble(long long row) {
  const int t = (int)(row & 127);
  return ((t & 1) << 2) | ((t >> 1) & 3);
}
// index of the fp16 scale of token `row` in group g (the zero is 128 halves further on)
__host__ __device__ __forceinline__ long long i4v_scale_index(long long row, int G, int g) {
  return (((row >> 7) * G + g) << 8) + (row & 127);
}

// Where token t of sequence b is stored: row b * cap + t of the latent arrays, or, in a
// paged cache, row page * 128 + t % 128 of the page pool, with page = table[b][t / 128].
// Pages are as long as the tensor-core tile and the int4 block, so a tile or a block never
// straddles two pages.
constexpr int kPageTokens = 128;
struct RowMap {
  const int32_t* table;   // paged: [B][pps] page of each 128-token span (device), else null
  long long cap;          // contiguous: rows per sequence
  int pps;                // paged: pages per sequence
  int n_pages;            // paged: pages in the pool (table entries are clamped to it)
  __device__ __forceinline__ long long row(int b, int t) const {
    return table ? ((long long)page(b, t) << 7) + (t & 127) : (long long)b * cap + t;
  }
  // the page of token t of sequence b; an entry outside [0, n_pages) (a device-side table
  // the library did not check) is clamped, so every access stays inside the pool
  __device__ __forceinline__ int page(int b, int t) const {
    return min(max(__ldg(table + (long long)b * pps + (t >> 7)), 0), n_pages - 1);
  }
};

// RoPE factors (cos, sin) of position t and frequency pair i (of d/2), fp32 from fp64
// angles, stored in 128-token tiles, pair-major inside a tile: the 128 tokens of one pair are
// contiguous, so threads that own consecutive tokens read one coalesced run per pair.
__host__ __device__ __forceinline__ long long rope_cs_index(long long t, int i, int half) {
  return (((t >> 7) * half + i) << 7) + (t & 127);
}

struct lr_cache {
  lr_cache_desc desc;
  int D;                 // n_kv_heads * head_dim
  int G_k, G_v;          // int4 groups per token (0 when unquantised)
  int win_slots;         // window + 1 (ring), or 0
  long long lat_cap;     // latent rows per sequence: capacity (int4: rounded up to 128)
  int32_t* ptable = nullptr;  // paged caches: the device block table [B][pps], else null
  int pps = 0;           // paged: pages per sequence (capacity / 128)
  int n_pages = 0;       // paged: pages in the pool
  std::vector<int32_t> host_table;   // paged: staging copy of the last table set
  int32_t len, hist_len, win_len;
  int groups = 1;         // latent groups (desc ranks are the block-diagonal total g r)
  float* r_full = nullptr; // block-diagonal sync rotations (latent groups), [r_k^2 + r_v^2]
  int undo = 0;           // windowed caches: 0 = no undo, 1 = the last append only filled
                          // the window, 2 = it folded the oldest window token into history
  int32_t stable_len = 0; // history rows [0, stable_len) were written before the kernel that
                          // precedes the decode (the decode may read them before its
                          // grid-dependency wait); set by each decode entry point
  float scale_log2;      // softmax_scale * log2(e)
  int latent_kind;       // LatentKind
  size_t esize;          // bytes per dtype element

  // storage
  void* z_k = nullptr; void* z_v = nullptr;
  uint32_t* codes_k = nullptr; uint32_t* codes_v = nullptr;
  uint32_t* params_k = nullptr; uint32_t* params_v = nullptr;
  void* win_k = nullptr; void* win_v = nullptr;
  void* A_k = nullptr; void* B_k = nullptr; void* A_v = nullptr; void* B_v = nullptr;
  float2* rope_cs = nullptr;   // (cos, sin) per (position, pair), rope_cs_index; fp32 from fp64 angles

  // scratch
  float* qt = nullptr;         // [B][Hq][r_k] fp32 scaled query latents (or [B][Hq][d] for RoPE)
  void* qt16 = nullptr;        // [B][Hpad][r_k] 16-bit query latents for the tensor-core path
  float* part_o = nullptr;     // [B][S_max][Hq][r_v]
  float* part_ml = nullptr;    // [B][S_max][Hq][2]
  float* win_o = nullptr;      // [B][Hq][d]
  float* win_ml = nullptr;     // [B][Hq][2]
  int* dev_err = nullptr;      // device error word
  unsigned long long wait_ns = 0;   // bounded-wait limit of the tensor-core kernels (0: default)
  const int32_t* row_len = nullptr; // per-row history lengths of the decode in flight (device), or null
  int S_max = 1;

  bool has_A = false;         // projections given at creation (needed by lr_kv_append)
  int path_force = 0, splits_force = 0;
  int num_sms = 148;
  int device = 0;
  cudaStream_t last_stream = nullptr;
  void* tc_state = nullptr;    // tensor-core path state (tensor maps), owned
  void* sync_state = nullptr;  // tensor-core basis sync state (tensor maps, split R), owned
  void* isvd_state = nullptr;  // block-incremental SVD working memory, owned
  cudaEvent_t ev_start = nullptr, ev_stop = nullptr;   // caller-owned kernel timing events
  unsigned long long* trace = nullptr;                 // caller-owned decode timeline buffer
  unsigned long long* spans = nullptr;                 // its kernel spans (SPAN_KINDS pairs), or null
};

// ---- argument blocks --------------------------------------------------------

struct LatentRef {
  const void* z;          // unquantised [B][cap][r]
  const uint32_t* codes;  // int4, blocked (i4_code_index; values: i4v_code_index)
  const uint32_t* params; // int4, blocked (i4_param_index; values: i4v_scale_index)
  int r, G;
  int rank_major;         // int4 values: the rank-major block layout
  RowMap map;             // token -> latent row
};

struct DecodeSimtArgs {
  LatentRef k, v;
  const float* qs;        // [B][Hq][r_k] (latent path) or [B][Hq][d] (RoPE path), pre-scaled
  const void* B_k;        // RoPE path: [r_k][D]
  const float2* rope_cs;  // RoPE path: rope_cs_index layout
  float* part_o;          // [B][S][Hq][r_v]
  float* part_ml;         // [B][S][Hq][2]
  int Hq, Hkv, d, D;
  int hist_len, split_tokens, n_splits;
  int rope;
  int dtype;
  const int32_t* row_len;  // per-row history lengths (device), or null: every row has hist_len
  unsigned long long* span;  // timeline span of this kernel, or null
};

// History tokens row b attends to: its own length, clamped to [1, hist_len], or hist_len.
__device__ __forceinline__ int row_hist(const int32_t* row_len, int b, int hist_len) {
  return row_len ? min(max(row_len[b], 1), hist_len) : hist_len;
}

// ---- launchers (return cudaGetLastError) ------------------------------------
// pdl = false: launched after the preceding work completes (for bases the caller owns,
// which the kernel just before may have written)
cudaError_t launch_qproj(const lr_cache* c, const void* q, cudaStream_t s, bool pdl = true);
cudaError_t launch_decode_simt(const lr_cache* c, int n_splits, int split_tokens, cudaStream_t s);
// The window of a fused step, launched right after the step's append and query projection
// and computed from the step's inputs (k, v: the new token's rows; q: the query) and the ring
// rows of earlier steps, with the counters after the append.
struct WindowStep {
  const void* k; const void* v; const void* q;
  int hist_len, win_len;
};
// st: null for the window after the latent decode
cudaError_t launch_window(const lr_cache* c, cudaStream_t s, const WindowStep* st = nullptr);
// Where the merge reads its partials and what it writes: by default the cache's own split
// partials ([B][S][Hq]) merged and projected to `out`; with a MergeSource, partials at other
// addresses / strides, and (rs_o set) a rank-space result instead of the projection.
struct MergeSource {
  const float* part_o; const float* part_ml;
  long long b_stride, s_stride;   // head-row blocks: (b, s) at (b * b_stride + s * s_stride) * Hq
  float* rs_o; float* rs_ml;      // rank-space output [B][Hq][r_v], [B][Hq][2], or null
};
cudaError_t launch_merge(const lr_cache* c, int n_splits, void* out, float* lse, cudaStream_t s,
                         const MergeSource* src = nullptr);
// block-incremental SVD update of one side's basis (k_incsvd.cu)
cudaError_t launch_basis_update(lr_cache* c, int side, const void* blk, int n, float* gram, float* R_out,
                                void* B_out, void* A_out, cudaStream_t s);
void isvd_release(lr_cache* c);
// bstride: elements between the batch rows of k and v (0: D, rows of one token per sequence)
// row_pos: per-row destination slots (device), or null: the cache's next slot for every row
cudaError_t launch_append(lr_cache* c, const void* k, const void* v, cudaStream_t s, long long bstride = 0,
                          const int32_t* row_pos = nullptr);
// bulk prefill on tensor cores (k_prefill_tc.cu): n tokens per sequence, k / v [B][n][D]
bool prefill_tc_supported(const lr_cache_desc* d, int D);
cudaError_t launch_prefill_tc(lr_cache* c, const void* k, const void* v, int n, cudaStream_t s);
// append (with the cache's current counters) and query projection in one grid
cudaError_t launch_step_pre(lr_cache* c, const void* k, const void* v, const void* q, bool tc, cudaStream_t s);
cudaError_t launch_append_latent(lr_cache* c, const float* zk, const float* zv, int n,
                                 cudaStream_t s);
cudaError_t launch_sync_simt(lr_cache* c, const float* R, int which, cudaStream_t s);
size_t decode_simt_smem(const lr_cache* c);

// tensor-core path (k_decode_tc.cu)
bool tc_supported(const lr_cache_desc* d);
int tc_ctas_per_sm(const lr_cache_desc* d, int hist_len, int num_sms);   // decode blocks per SM
// (re)builds the path's tensor maps and derived operands; kernels it launches go on s
cudaError_t tc_prepare(lr_cache* c, cudaStream_t s);
// decode CTAs per (sequence, split): 1, or the KV-head pairs of the keys-before-RoPE grid
int tc_split_ctas(const lr_cache_desc* d);
void tc_release(lr_cache* c);
cudaError_t launch_qproj_tc(const lr_cache* c, const void* q, cudaStream_t s);
cudaError_t launch_decode_tc(const lr_cache* c, int n_splits, int split_tokens, cudaStream_t s);
// int4 latents on tensor cores (k_decode_tc_i4.cu)
bool tc_i4_supported(const lr_cache_desc* d);
cudaError_t tc_i4_prepare(lr_cache* c, cudaStream_t s);
int tc_i4_split_ctas(const lr_cache_desc* d);
void tc_i4_release(lr_cache* c);
cudaError_t launch_decode_tc_i4(const lr_cache* c, int n_splits, int split_tokens, cudaStream_t s);

// basis sync on tensor cores (k_sync_tc.cu)
bool sync_tc_supported(const lr_cache_desc* d);
cudaError_t launch_sync_tc(lr_cache* c, const float* R_k, const float* R_v, cudaStream_t s);
void sync_tc_release(lr_cache* c);

void lr_count_launch(int n = 1);

// Host-side fault injection (lr_debug_inject_fault): true when this device allocation or
// kernel launch is the one armed to fail; the caller then fails without allocating or
// launching.
// The row map of a cache's latents (paged or contiguous).
inline RowMap row_map(const lr_cache* c) {
  RowMap m;
  m.table = c->ptable;
  m.cap = c->lat_cap;
  m.pps = c->pps;
  m.n_pages = c->n_pages;
  return m;
}

bool lr_fault_alloc();
bool lr_fault_launch();

// Every device allocation of the library goes through here.
inline cudaError_t lr_dev_malloc(void** p, size_t bytes) {
  *p = nullptr;
  if (lr_fault_alloc()) return cudaErrorMemoryAllocation;
  return cudaMalloc(p, bytes);
}
template <typename T>
inline cudaError_t lr_dev_malloc(T** p, size_t bytes) {
  return lr_dev_malloc(reinterpret_cast<void**>(p), bytes);
}

// Programmatic dependent launch.  Every kernel of the library does its prologue on data
// no in-flight kernel writes, then pdl_wait() (the preceding grid has completed and its
// memory is visible), then pdl_trigger() (the next grid may start its own prologue).
// Because each kernel triggers only after its wait, everything before the preceding
// kernel has completed whenever a prologue runs.  Both are no-ops without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Kernel spans of the timeline trace (lr_cache_set_trace): for span kind k, word 2k holds
// the earliest CTA start and word 2k + 1 the latest CTA end of the kernels of that kind, in
// %globaltimer nanoseconds (the caller initialises the words to ~0 and 0).  A null pointer
// disables the stamps.  span_end synchronises the block, so every thread must reach it.
enum SpanKind { SPAN_PRE = 0, SPAN_DECODE = 1, SPAN_WINDOW = 2, SPAN_MERGE = 3, SPAN_KINDS = 4 };
__device__ __forceinline__ unsigned long long span_now() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void span_begin(unsigned long long* sp) {
  if (sp && threadIdx.x == 0) atomicMin(sp, span_now());
}
__device__ __forceinline__ void span_end(unsigned long long* sp) {
  if (!sp) return;
  __syncthreads();
  if (threadIdx.x == 0) atomicMax(sp + 1, span_now());
}
__host__ __device__ __forceinline__ unsigned long long* span_of(unsigned long long* spans, int kind) {
  return spans ? spans + 2 * kind : nullptr;
}

// Launch with the programmatic-stream-serialization attribute; returns the launch error.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (lr_fault_launch()) return cudaErrorLaunchFailure;
  lr_count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// As launch_pdl, with clusters of `cluster_x` CTAs along x (grid.x a multiple of it).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, int cluster_x, size_t smem,
                                      cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)cluster_x;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (lr_fault_launch()) return cudaErrorLaunchFailure;
  lr_count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Launch without the attribute: the kernel starts only after the preceding work on the
// stream has completed, so its prologue may read anything that work wrote.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_serial(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                 Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = nullptr;
  cfg.numAttrs = 0;
  if (lr_fault_launch()) return cudaErrorLaunchFailure;
  lr_count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Raise a kernel's dynamic shared-memory limit to the 227 KB opt-in maximum (less its
// static shared memory) once per device; later launches skip the call, so launches stay
// legal inside stream capture.
template <typename Kernel>
inline cudaError_t smem_optin(Kernel k, std::atomic<uint32_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint32_t bit = 1u << (dev & 31);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, k);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448 - (int)fa.sharedSizeBytes);
  // one carveout for every kernel of the library, so consecutive kernels do not
  // reconfigure the L1 / shared-memory split of the SMs between them
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  else (void)cudaGetLastError();   // do not leave a stale error for a later launch check
  return e;
}
