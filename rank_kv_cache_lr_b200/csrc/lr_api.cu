// Host layer of the C ABI declared in include/lr_kv.h: validation, cache
// lifetime, length bookkeeping, decode planning and kernel launches.
#include "lr_internal.cuh"

#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

namespace {

std::atomic<long long> g_launches{0};
// Armed faults: the number of operations of each kind still to succeed before one fails
// (-1: none armed).
std::atomic<long long> g_fault_left[2] = {{-1}, {-1}};

bool fault_fires(int kind) {
  long long left = g_fault_left[kind].load();
  while (left >= 0) {
    if (g_fault_left[kind].compare_exchange_weak(left, left - 1)) return left == 0;
  }
  return false;
}

int groups_of(const lr_cache_desc* d) { return d->latent_groups > 1 ? d->latent_groups : 1; }

// The description the kernels see: g latent groups of rank r stored as one block-diagonal
// latent of rank g r.
lr_cache_desc effective_desc(const lr_cache_desc* d) {
  lr_cache_desc e = *d;
  e.rank_k *= groups_of(d);
  e.rank_v *= groups_of(d);
  return e;
}

lr_status validate_user_desc(const lr_cache_desc* d);

lr_status validate_desc(const lr_cache_desc* d) {
  if (!d) return LR_ERR_INVALID_ARG;
  if (d->latent_groups < 0) return LR_ERR_INVALID_ARG;
  if (d->latent_groups > 1 && (d->n_kv_heads % d->latent_groups)) return LR_ERR_INVALID_ARG;
  if (d->rank_k < 16 || d->rank_k % 16 || d->rank_v < 16 || d->rank_v % 16) return LR_ERR_INVALID_ARG;
  const lr_cache_desc e = effective_desc(d);
  return validate_user_desc(&e);
}

lr_status validate_user_desc(const lr_cache_desc* d) {
  if (!d) return LR_ERR_INVALID_ARG;
  if (d->batch < 1 || d->n_q_heads < 1 || d->n_kv_heads < 1) return LR_ERR_INVALID_ARG;
  if (d->n_q_heads % d->n_kv_heads) return LR_ERR_INVALID_ARG;
  if (d->head_dim < 8 || d->head_dim % 8 || d->head_dim > 256) return LR_ERR_INVALID_ARG;
  if (d->rank_k < 16 || d->rank_k % 16 || d->rank_k > 512) return LR_ERR_INVALID_ARG;
  if (d->rank_v < 16 || d->rank_v % 16 || d->rank_v > 512) return LR_ERR_INVALID_ARG;
  if (d->capacity < 1 || d->window < 0 || d->window > d->capacity) return LR_ERR_INVALID_ARG;
  if (d->quant_bits != 0 && d->quant_bits != 4) return LR_ERR_INVALID_ARG;
  if (d->quant_bits == 4 && d->quant_group != 32) return LR_ERR_UNSUPPORTED;
  if (d->dtype != LR_F32 && d->dtype != LR_BF16) return LR_ERR_INVALID_ARG;
  if (d->rope_in_kernel != 0 && d->rope_in_kernel != 1) return LR_ERR_INVALID_ARG;
  if (d->rope_in_kernel && !(d->rope_theta > 0.0)) return LR_ERR_INVALID_ARG;
  if (d->rope_in_kernel && d->window > 0) return LR_ERR_UNSUPPORTED;
  if (!(d->softmax_scale >= 0.0f) || std::isinf(d->softmax_scale)) return LR_ERR_INVALID_ARG;
  for (int i = 0; i < 2; ++i)
    if (d->reserved[i] != 0) return LR_ERR_INVALID_ARG;
  if (d->page_tokens != 0 && d->page_tokens != kPageTokens) return LR_ERR_INVALID_ARG;
  if (d->page_tokens == 0 && d->n_pages != 0) return LR_ERR_INVALID_ARG;
  if (d->n_pages < 0 || d->n_pages > (1 << 22)) return LR_ERR_INVALID_ARG;
  if (d->page_tokens && (d->capacity % kPageTokens || d->window > 0)) return LR_ERR_UNSUPPORTED;
  if (d->page_tokens && d->n_pages == 0 && (long long)d->batch * (d->capacity / kPageTokens) > (1 << 22))
    return LR_ERR_INVALID_ARG;
  if ((long long)d->n_kv_heads * d->head_dim > 4096) return LR_ERR_UNSUPPORTED;
  if (d->n_q_heads > 128 || d->n_q_heads / d->n_kv_heads > 64) return LR_ERR_UNSUPPORTED;
  return LR_OK;
}

int pick_path(const lr_cache_desc* d, int forced) {
  if (forced == LR_PATH_SIMT) return LR_PATH_SIMT;
  if (forced == LR_PATH_TC) return tc_supported(d) ? LR_PATH_TC : -1;
  return tc_supported(d) ? LR_PATH_TC : LR_PATH_SIMT;
}

// Split the history into tiles and spread them over about two CTAs per SM.
lr_status plan(const lr_cache_desc* d, int hist_len, int num_sms, int path, int n_splits,
               lr_plan* out) {
  const int p = pick_path(d, path);
  if (p < 0) return LR_ERR_UNSUPPORTED;
  const int tile = (p == LR_PATH_TC) ? 128 : 16;
  const int tiles = std::max(1, (hist_len + tile - 1) / tile);
  int splits = n_splits;
  if (splits <= 0) {
    // SIMT: about two CTAs per SM; tensor-core path: one wave of its resident blocks
    const int sms = std::max(num_sms, 1);
    const int target =
        (p == LR_PATH_TC) ? std::max(1, tc_ctas_per_sm(d, hist_len, sms) * sms / (d->batch * tc_split_ctas(d)))
                          : std::max(1, (2 * sms + d->batch - 1) / d->batch);
    splits = std::min(tiles, target);
  }
  splits = std::max(1, std::min(splits, tiles));
  const int tiles_per = (tiles + splits - 1) / splits;
  splits = (tiles + tiles_per - 1) / tiles_per;
  out->path = p;
  out->n_splits = splits;
  out->tile_tokens = tile;
  out->split_tokens = tiles_per * tile;
  out->ctas = splits * d->batch * (p == LR_PATH_TC ? tc_split_ctas(d) : 1);
  return LR_OK;
}

// Partial buffers hold up to max(64, the automatic split count) splits per sequence,
// and never more than one split per 16-token tile.
int max_splits_for(const lr_cache_desc* d, int num_sms) {
  const int tiles = std::max(1, (d->capacity + 15) / 16);
  const int target = std::max(1, (2 * std::max(num_sms, 1) + d->batch - 1) / d->batch);
  return std::min(tiles, std::max(64, target));
}

template <typename T>
cudaError_t dalloc(T** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return cudaSuccess;
  cudaError_t e = lr_dev_malloc((void**)p, bytes);
  if (e != cudaSuccess) return e;
  return cudaMemset(*p, 0, bytes);
}

void free_all(lr_cache* c) {
  if (!c) return;
  tc_release(c);
  sync_tc_release(c);
  isvd_release(c);
  void* ptrs[] = {c->z_k, c->z_v, c->codes_k, c->codes_v, c->params_k, c->params_v, c->win_k, c->win_v,
                  c->A_k, c->B_k, c->A_v, c->B_v, c->rope_cs, c->qt, c->qt16, c->part_o, c->part_ml,
                  c->win_o, c->win_ml, c->dev_err, c->r_full, c->ptable};
  for (void* p : ptrs)
    if (p) cudaFree(p);
}

// Record a caller's timing event; inside stream capture it becomes an external event
// node, so that every replay of the graph records it.
cudaError_t record_event(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(s, &cs);
  if (e != cudaSuccess) return e;
  if (cs == cudaStreamCaptureStatusActive) return cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
  return cudaEventRecord(ev, s);
}

// dst [g rows][g cols] (zero outside the blocks) <- the g diagonal blocks src [g][rows][cols],
// elements of `es` bytes.
cudaError_t expand_blockdiag(void* dst, const void* src, int g, size_t rows, size_t cols, size_t es,
                             cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  for (int i = 0; i < g && e == cudaSuccess; ++i)
    e = cudaMemcpy2DAsync(static_cast<char*>(dst) + (i * rows * g * cols + i * cols) * es, g * cols * es,
                          static_cast<const char*>(src) + i * rows * cols * es, cols * es, cols * es, rows,
                          cudaMemcpyDeviceToDevice, s);
  return e;
}

// Copy a caller's basis into the cache: A [D][r] / B [r][D] as they are, or, with latent
// groups, the per-group blocks A [g][D/g][r/g] / B [g][r/g][D/g] onto the diagonal of the
// block-diagonal basis (its other entries stay zero from the allocation).
cudaError_t install_basis(lr_cache* c, void* dst, const void* src, bool is_A, bool is_k, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  const size_t r = is_k ? d.rank_k : d.rank_v, D = c->D, es = c->esize;
  const int g = c->groups;
  if (g == 1) return cudaMemcpyAsync(dst, src, r * D * es, cudaMemcpyDeviceToDevice, s);
  return is_A ? expand_blockdiag(dst, src, g, D / g, r / g, es, s) : expand_blockdiag(dst, src, g, r / g, D / g, es, s);
}

lr_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return LR_OK;
  if (e == cudaErrorMemoryAllocation) return LR_ERR_OOM;
  return LR_ERR_CUDA;
}

}  // namespace

void lr_count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }
bool lr_fault_alloc() { return fault_fires(0); }
bool lr_fault_launch() { return fault_fires(1); }

extern "C" {

const char* lr_status_string(lr_status s) {
  switch (s) {
    case LR_OK: return "LR_OK";
    case LR_ERR_INVALID_ARG: return "LR_ERR_INVALID_ARG";
    case LR_ERR_UNSUPPORTED: return "LR_ERR_UNSUPPORTED";
    case LR_ERR_CAPACITY: return "LR_ERR_CAPACITY";
    case LR_ERR_CUDA: return "LR_ERR_CUDA";
    case LR_ERR_OOM: return "LR_ERR_OOM";
    case LR_ERR_TIMEOUT: return "LR_ERR_TIMEOUT";
  }
  return "LR_ERR_UNKNOWN";
}

int64_t lr_launch_count(void) { return g_launches.load(); }

lr_status lr_plan_decode(const lr_cache_desc* desc, int32_t len, int32_t num_sms, int32_t path,
                         int32_t n_splits, lr_plan* out) {
  lr_status st = validate_desc(desc);
  if (st != LR_OK) return st;
  if (!out || len < 0 || len > desc->capacity || num_sms < 1) return LR_ERR_INVALID_ARG;
  if (path < 0 || path > 2 || n_splits < 0) return LR_ERR_INVALID_ARG;
  const int hist = desc->window > 0 ? std::max(0, len - desc->window) : len;
  const lr_cache_desc e = effective_desc(desc);
  return plan(&e, hist, num_sms, path, n_splits, out);
}

lr_status lr_cache_create(const lr_cache_desc* desc, const void* A_k, const void* B_k, const void* A_v,
                          const void* B_v, void* stream, lr_cache** out) {
  if (!out) return LR_ERR_INVALID_ARG;
  *out = nullptr;
  lr_status st = validate_desc(desc);
  if (st != LR_OK) return st;
  if (!B_k || !B_v) return LR_ERR_INVALID_ARG;
  if ((A_k == nullptr) != (A_v == nullptr)) return LR_ERR_INVALID_ARG;

  lr_cache* c = new (std::nothrow) lr_cache();
  if (!c) return LR_ERR_OOM;
  c->desc = effective_desc(desc);
  c->groups = groups_of(desc);
  const lr_cache_desc& d = c->desc;
  c->D = d.n_kv_heads * d.head_dim;
  c->esize = d.dtype == LR_BF16 ? 2 : 4;
  c->latent_kind = d.quant_bits == 4 ? LK_INT4 : (d.dtype == LR_BF16 ? LK_BF16 : LK_F32);
  c->G_k = d.quant_bits == 4 ? (d.rank_k + 31) / 32 : 0;
  c->G_v = d.quant_bits == 4 ? (d.rank_v + 31) / 32 : 0;
  c->win_slots = d.window > 0 ? d.window + 1 : 0;
  c->lat_cap = c->latent_kind == LK_INT4 ? ((long long)d.capacity + kI4Block - 1) / kI4Block * kI4Block
                                         : (long long)d.capacity;
  if (d.page_tokens) {
    c->pps = d.capacity / kPageTokens;
    c->n_pages = d.n_pages ? d.n_pages : d.batch * c->pps;
  }
  c->len = c->hist_len = c->win_len = 0;
  const float sm_scale = d.softmax_scale > 0.f ? d.softmax_scale : 1.0f / std::sqrt((float)d.head_dim);
  c->scale_log2 = sm_scale * LR_LOG2E;
  c->last_stream = (cudaStream_t)stream;

  cudaError_t e = cudaGetDevice(&c->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device);
  c->S_max = max_splits_for(&d, c->num_sms);
  const size_t B = d.batch, cap = d.capacity, es = c->esize, D = c->D;
  if (e == cudaSuccess) {
    if (c->latent_kind == LK_INT4) {
      const size_t rows = c->n_pages ? (size_t)c->n_pages * kPageTokens : B * (size_t)c->lat_cap;
      e = dalloc(&c->codes_k, rows * c->G_k * 4 * sizeof(uint32_t));
      if (e == cudaSuccess) e = dalloc(&c->codes_v, rows * c->G_v * 4 * sizeof(uint32_t));
      if (e == cudaSuccess) e = dalloc(&c->params_k, rows * c->G_k * sizeof(uint32_t));
      if (e == cudaSuccess) e = dalloc(&c->params_v, rows * c->G_v * sizeof(uint32_t));
    } else {
      const size_t rows = c->n_pages ? (size_t)c->n_pages * kPageTokens : B * cap;
      e = dalloc(&c->z_k, rows * d.rank_k * es);
      if (e == cudaSuccess) e = dalloc(&c->z_v, rows * d.rank_v * es);
    }
  }
  if (e == cudaSuccess && c->n_pages) {
    // the initial table: span j of sequence b in page (b * pps + j) % n_pages
    std::vector<int32_t> tab((size_t)d.batch * c->pps);
    for (size_t i = 0; i < tab.size(); ++i) tab[i] = (int32_t)(i % (size_t)c->n_pages);
    e = dalloc(&c->ptable, tab.size() * sizeof(int32_t));
    if (e == cudaSuccess) e = cudaMemcpy(c->ptable, tab.data(), tab.size() * sizeof(int32_t), cudaMemcpyHostToDevice);
  }
  if (e == cudaSuccess && c->win_slots) {
    e = dalloc(&c->win_k, B * c->win_slots * D * es);
    if (e == cudaSuccess) e = dalloc(&c->win_v, B * c->win_slots * D * es);
  }
  if (e == cudaSuccess) e = dalloc(&c->B_k, (size_t)d.rank_k * D * es);
  if (e == cudaSuccess) e = dalloc(&c->B_v, (size_t)d.rank_v * D * es);
  if (e == cudaSuccess) e = dalloc(&c->A_k, D * d.rank_k * es);
  if (e == cudaSuccess) e = dalloc(&c->A_v, D * d.rank_v * es);
  if (e == cudaSuccess) e = dalloc(&c->qt, B * d.n_q_heads * ((size_t)d.rank_k + d.head_dim) * sizeof(float));
  if (e == cudaSuccess) e = dalloc(&c->part_o, B * c->S_max * d.n_q_heads * (size_t)d.rank_v * sizeof(float));
  if (e == cudaSuccess) e = dalloc(&c->part_ml, B * c->S_max * d.n_q_heads * 2 * sizeof(float));
  if (e == cudaSuccess && c->win_slots) {
    e = dalloc(&c->win_o, B * d.n_q_heads * (size_t)d.head_dim * sizeof(float));
    if (e == cudaSuccess) e = dalloc(&c->win_ml, B * d.n_q_heads * 2 * sizeof(float));
  }
  if (e == cudaSuccess) e = dalloc(&c->dev_err, sizeof(int));
  if (e == cudaSuccess && d.rope_in_kernel) {
    const int half = d.head_dim / 2;
    const size_t cap128 = (cap + 127) / 128 * 128;
    std::vector<float2> cs(cap128 * half);
    std::vector<double> omega(half);
    for (int i = 0; i < half; ++i) omega[i] = std::pow(d.rope_theta, -2.0 * i / d.head_dim);
    for (size_t t = 0; t < cap128; ++t)
      for (int i = 0; i < half; ++i) {
        const double ang = (double)t * omega[i];
        cs[rope_cs_index((long long)t, i, half)] = make_float2((float)std::cos(ang), (float)std::sin(ang));
      }
    e = dalloc(&c->rope_cs, cs.size() * sizeof(float2));
    if (e == cudaSuccess) e = cudaMemcpy(c->rope_cs, cs.data(), cs.size() * sizeof(float2), cudaMemcpyHostToDevice);
  }
  cudaStream_t s = (cudaStream_t)stream;
  if (e == cudaSuccess) e = install_basis(c, c->B_k, B_k, false, true, s);
  if (e == cudaSuccess) e = install_basis(c, c->B_v, B_v, false, false, s);
  if (e == cudaSuccess && A_k) e = install_basis(c, c->A_k, A_k, true, true, s);
  if (e == cudaSuccess && A_v) e = install_basis(c, c->A_v, A_v, true, false, s);
  c->has_A = A_k != nullptr;
  if (e == cudaSuccess && tc_supported(&d)) e = tc_prepare(c, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    free_all(c);
    delete c;
    return cuda_status(e);
  }
  *out = c;
  return LR_OK;
}

lr_status lr_cache_destroy(lr_cache* c) {
  if (!c) return LR_OK;
  cudaError_t e = cudaDeviceSynchronize();
  free_all(c);
  delete c;
  return e == cudaSuccess ? LR_OK : LR_ERR_CUDA;
}

lr_status lr_kv_append(lr_cache* c, const void* k, const void* v, void* stream) {
  if (!c || !k || !v || !c->has_A) return LR_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15) return LR_ERR_INVALID_ARG;
  if (c->len >= c->desc.capacity) return LR_ERR_CAPACITY;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  cudaError_t e = launch_append(c, k, v, s);
  if (e != cudaSuccess) return LR_ERR_CUDA;
  if (c->win_slots) {
    c->undo = c->win_len == c->desc.window ? 2 : 1;
    if (c->undo == 2) ++c->hist_len;
    else ++c->win_len;
  } else {
    ++c->hist_len;
  }
  ++c->len;
  return LR_OK;
}

lr_status lr_kv_append_rows(lr_cache* c, const void* k, const void* v, const int32_t* pos, int32_t max_len,
                            void* stream) {
  if (!c || !k || !v || !pos || !c->has_A) return LR_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15) return LR_ERR_INVALID_ARG;
  if (c->win_slots) return LR_ERR_UNSUPPORTED;
  if (max_len < 0) return LR_ERR_INVALID_ARG;
  if (max_len > c->desc.capacity) return LR_ERR_CAPACITY;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  c->undo = 0;
  cudaError_t e = launch_append(c, k, v, s, 0, pos);
  if (e != cudaSuccess) return LR_ERR_CUDA;
  if (max_len > c->hist_len) c->hist_len = c->len = max_len;
  return LR_OK;
}

lr_status lr_kv_prefill(lr_cache* c, const void* k, const void* v, int32_t n, void* stream) {
  if (!c || !k || !v || n < 0 || !c->has_A) return LR_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15) return LR_ERR_INVALID_ARG;
  if (c->win_slots) return LR_ERR_UNSUPPORTED;
  if ((long long)c->len + n > c->desc.capacity) return LR_ERR_CAPACITY;
  c->undo = 0;
  if (n == 0) return LR_OK;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  cudaError_t e = cudaSuccess;
  if (prefill_tc_supported(&c->desc, c->D)) {
    e = launch_prefill_tc(c, k, v, n, s);
    if (e != cudaSuccess) return LR_ERR_CUDA;
    c->hist_len += n;
    c->len += n;
    return LR_OK;
  }
  // other dtypes and shapes: one append launch per token (CUDA cores)
  const size_t row = (size_t)c->D * c->esize;
  for (int t = 0; t < n; ++t) {
    e = launch_append(c, static_cast<const char*>(k) + t * row, static_cast<const char*>(v) + t * row, s,
                      (long long)n * c->D);
    if (e != cudaSuccess) return LR_ERR_CUDA;
    ++c->hist_len;
    ++c->len;
  }
  return LR_OK;
}

lr_status lr_kv_append_latent(lr_cache* c, const float* zk, const float* zv, int32_t n, void* stream) {
  if (!c || !zk || !zv || n < 0) return LR_ERR_INVALID_ARG;
  if (c->win_len > 0) return LR_ERR_INVALID_ARG;
  if ((long long)c->len + n > c->desc.capacity) return LR_ERR_CAPACITY;
  c->undo = 0;
  if (n == 0) return LR_OK;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  cudaError_t e = launch_append_latent(c, zk, zv, n, s);
  if (e != cudaSuccess) return LR_ERR_CUDA;
  c->hist_len += n;
  c->len += n;
  return LR_OK;
}

lr_status lr_cache_plan(const lr_cache* c, lr_plan* out) {
  if (!c || !out) return LR_ERR_INVALID_ARG;
  return plan(&c->desc, c->hist_len, c->num_sms, c->path_force, c->splits_force, out);
}

}  // extern "C"

namespace {

// The decode after its query projection: split-sequence attention (timed by the
// caller's events when set), exact window, split merge and output projection.
cudaError_t decode_rest(lr_cache* c, const lr_plan& p, void* out, float* lse, cudaStream_t s,
                        bool window_done = false) {
  cudaError_t e = cudaSuccess;
  if (c->hist_len > 0) {
    if (c->ev_start) e = record_event(c->ev_start, s);
    if (e == cudaSuccess)
      e = p.path == LR_PATH_TC ? launch_decode_tc(c, p.n_splits, p.split_tokens, s)
                               : launch_decode_simt(c, p.n_splits, p.split_tokens, s);
    if (e == cudaSuccess && c->ev_stop) e = record_event(c->ev_stop, s);
  }
  const int S = c->hist_len > 0 ? p.n_splits : 0;
  if (e == cudaSuccess && c->win_slots && !window_done) e = launch_window(c, s);
  if (e == cudaSuccess) e = launch_merge(c, S, out, lse, s);
  return e;
}

lr_status decode_plan(const lr_cache* c, int hist_len, lr_plan* p) {
  lr_status st = plan(&c->desc, hist_len, c->num_sms, c->path_force, c->splits_force, p);
  if (st != LR_OK) return st;
  if (p->n_splits > c->S_max) return LR_ERR_UNSUPPORTED;
  if (p->path != LR_PATH_TC && hist_len > 0 && decode_simt_smem(c) > 227 * 1024) return LR_ERR_UNSUPPORTED;
  return LR_OK;
}

}  // namespace

extern "C" {

lr_status lr_attn_decode(lr_cache* c, const void* q, void* out, float* lse, void* stream) {
  if (!c || !q || !out) return LR_ERR_INVALID_ARG;
  if (c->len == 0) return LR_ERR_INVALID_ARG;
  lr_plan p;
  lr_status st = decode_plan(c, c->hist_len, &p);
  if (st != LR_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  c->stable_len = c->hist_len;
  cudaError_t e = p.path == LR_PATH_TC ? launch_qproj_tc(c, q, s) : launch_qproj(c, q, s);
  if (e == cudaSuccess) e = decode_rest(c, p, out, lse, s);
  return e == cudaSuccess ? LR_OK : LR_ERR_CUDA;
}

lr_status lr_attn_decode_partial(lr_cache* c, const void* q, float* part_o, float* part_ml, void* stream) {
  if (!c || !q || !part_o || !part_ml) return LR_ERR_INVALID_ARG;
  if (c->win_slots || c->desc.rope_in_kernel) return LR_ERR_UNSUPPORTED;
  if (c->len == 0) return LR_ERR_INVALID_ARG;
  lr_plan p;
  lr_status st = decode_plan(c, c->hist_len, &p);
  if (st != LR_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  c->stable_len = c->hist_len;
  cudaError_t e = p.path == LR_PATH_TC ? launch_qproj_tc(c, q, s) : launch_qproj(c, q, s);
  if (e == cudaSuccess && c->ev_start) e = record_event(c->ev_start, s);
  if (e == cudaSuccess)
    e = p.path == LR_PATH_TC ? launch_decode_tc(c, p.n_splits, p.split_tokens, s)
                             : launch_decode_simt(c, p.n_splits, p.split_tokens, s);
  if (e == cudaSuccess && c->ev_stop) e = record_event(c->ev_stop, s);
  if (e == cudaSuccess) {
    MergeSource src{c->part_o, c->part_ml, p.n_splits, 1, part_o, part_ml};
    e = launch_merge(c, p.n_splits, nullptr, nullptr, s, &src);
  }
  return e == cudaSuccess ? LR_OK : LR_ERR_CUDA;
}

lr_status lr_merge_partials(lr_cache* c, int32_t n, const float* part_o, const float* part_ml, void* out,
                            float* lse, void* stream) {
  if (!c || !part_o || !part_ml || !out || n < 1) return LR_ERR_INVALID_ARG;
  if (c->win_slots || c->desc.rope_in_kernel) return LR_ERR_UNSUPPORTED;
  if (n > c->S_max) return LR_ERR_CAPACITY;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  MergeSource src{part_o, part_ml, 1, c->desc.batch, nullptr, nullptr};
  cudaError_t e = launch_merge(c, n, out, lse, s, &src);
  return e == cudaSuccess ? LR_OK : LR_ERR_CUDA;
}

lr_status lr_attn_decode_varlen(lr_cache* c, const void* q, void* out, float* lse, const int32_t* row_len,
                                void* stream) {
  if (!c || !q || !out || !row_len) return LR_ERR_INVALID_ARG;
  if (c->win_slots) return LR_ERR_UNSUPPORTED;
  if (c->len == 0) return LR_ERR_INVALID_ARG;
  lr_plan p;
  lr_status st = decode_plan(c, c->hist_len, &p);
  if (st != LR_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  c->stable_len = c->hist_len;
  c->row_len = row_len;
  cudaError_t e = p.path == LR_PATH_TC ? launch_qproj_tc(c, q, s) : launch_qproj(c, q, s);
  if (e == cudaSuccess) e = decode_rest(c, p, out, lse, s);
  c->row_len = nullptr;
  return e == cudaSuccess ? LR_OK : LR_ERR_CUDA;
}

lr_status lr_decode_step(lr_cache* c, const void* k, const void* v, const void* q, void* out, float* lse,
                         void* stream) {
  if (!c || !k || !v || !q || !out || !c->has_A) return LR_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v)) & 15) return LR_ERR_INVALID_ARG;
  if (c->len >= c->desc.capacity) return LR_ERR_CAPACITY;
  int32_t hist1 = c->hist_len, win1 = c->win_len;
  if (c->win_slots) {
    if (c->win_len == c->desc.window) ++hist1;
    else ++win1;
  } else {
    ++hist1;
  }
  lr_plan p;
  lr_status st = decode_plan(c, hist1, &p);
  if (st != LR_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  cudaError_t e = launch_step_pre(c, k, v, q, p.path == LR_PATH_TC, s);   // uses the pre-append counters
  if (e == cudaSuccess && c->win_slots) {
    // the exact window next, alongside the append and projection: its tokens are earlier
    // steps' ring rows and this step's k, v
    const WindowStep ws{k, v, q, hist1, win1};
    e = launch_window(c, s, &ws);
  }
  if (e != cudaSuccess) return LR_ERR_CUDA;
  c->stable_len = c->hist_len;   // the row the append writes (new token or fold) is not stable
  if (c->win_slots) c->undo = hist1 > c->hist_len ? 2 : 1;
  c->hist_len = hist1;
  c->win_len = win1;
  ++c->len;
  e = decode_rest(c, p, out, lse, s, c->win_slots != 0);
  return e == cudaSuccess ? LR_OK : LR_ERR_CUDA;
}

lr_status lr_basis_sync(lr_cache* c, const float* R_k, const float* R_v, const void* B_k_new,
                        const void* B_v_new, const void* A_k_new, const void* A_v_new, void* stream) {
  if (!c) return LR_ERR_INVALID_ARG;
  if (c->latent_kind == LK_INT4 && (R_k || R_v)) return LR_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  const lr_cache_desc& d = c->desc;
  cudaError_t e = cudaSuccess;
  if (c->groups > 1 && (R_k || R_v)) {
    // per-group rotations onto the diagonal of one block-diagonal rotation per side
    const size_t rk = d.rank_k, rv = d.rank_v;
    if (!c->r_full) {
      e = lr_dev_malloc(&c->r_full, (rk * rk + rv * rv) * sizeof(float));
      if (e == cudaSuccess) e = cudaMemsetAsync(c->r_full, 0, (rk * rk + rv * rv) * sizeof(float), s);
      if (e != cudaSuccess) {
        if (c->r_full) cudaFree(c->r_full);
        c->r_full = nullptr;
        return cuda_status(e);
      }
    }
    const int g = c->groups;
    if (R_k) e = expand_blockdiag(c->r_full, R_k, g, rk / g, rk / g, sizeof(float), s);
    if (e == cudaSuccess && R_v) e = expand_blockdiag(c->r_full + rk * rk, R_v, g, rv / g, rv / g, sizeof(float), s);
    if (e != cudaSuccess) return LR_ERR_CUDA;
    R_k = R_k ? c->r_full : nullptr;
    R_v = R_v ? c->r_full + rk * rk : nullptr;
  }
  if ((R_k || R_v) && sync_tc_supported(&d) && c->path_force != LR_PATH_SIMT) {
    e = launch_sync_tc(c, R_k, R_v, s);
  } else {
    if (R_k) e = launch_sync_simt(c, R_k, 0, s);
    if (e == cudaSuccess && R_v) e = launch_sync_simt(c, R_v, 1, s);
  }
  if (e == cudaSuccess && B_k_new) e = install_basis(c, c->B_k, B_k_new, false, true, s);
  if (e == cudaSuccess && B_v_new) e = install_basis(c, c->B_v, B_v_new, false, false, s);
  if (A_k_new || A_v_new) c->has_A = true;
  if (e == cudaSuccess && A_k_new) e = install_basis(c, c->A_k, A_k_new, true, true, s);
  if (e == cudaSuccess && A_v_new) e = install_basis(c, c->A_v, A_v_new, true, false, s);
  if (e == cudaSuccess && (B_k_new || B_v_new)) e = tc_prepare(c, s);
  return e == cudaSuccess ? LR_OK : LR_ERR_CUDA;
}

lr_status lr_basis_update(lr_cache* c, int32_t side, const void* blk, int32_t n, float* gram, float* R_out,
                          void* B_new, void* A_new, void* stream) {
  if (!c || !blk || !gram || !R_out || (side != 0 && side != 1)) return LR_ERR_INVALID_ARG;
  if (n < 1 || n > 128) return LR_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(blk) & 15) return LR_ERR_INVALID_ARG;
  if (c->groups > 1) return LR_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  cudaError_t e = launch_basis_update(c, side, blk, n, gram, R_out, B_new, A_new, s);
  return e == cudaSuccess ? LR_OK : cuda_status(e);
}

lr_status lr_cache_get_len(const lr_cache* c, int32_t* len, int32_t* hist_len, int32_t* win_len) {
  if (!c) return LR_ERR_INVALID_ARG;
  if (len) *len = c->len;
  if (hist_len) *hist_len = c->hist_len;
  if (win_len) *win_len = c->win_len;
  return LR_OK;
}

lr_status lr_cache_truncate(lr_cache* c, int32_t len) {
  if (!c || len < 0 || len > c->len) return LR_ERR_INVALID_ARG;
  if (c->win_slots) {
    // The ring keeps one slot beyond the window, so the last append can be undone: the
    // token it folded out of the window is still in its slot.
    if (len == c->len) return LR_OK;
    if (len != c->len - 1 || c->undo == 0) return LR_ERR_UNSUPPORTED;
    if (c->undo == 2) --c->hist_len;
    else --c->win_len;
    --c->len;
    c->undo = 0;
    return LR_OK;
  }
  c->len = c->hist_len = len;
  return LR_OK;
}

lr_status lr_cache_view_get(const lr_cache* c, lr_cache_view* v) {
  if (!c || !v) return LR_ERR_INVALID_ARG;
  std::memset(v, 0, sizeof(*v));
  v->z_k = c->z_k; v->z_v = c->z_v;
  v->codes_k = c->codes_k; v->codes_v = c->codes_v;
  v->params_k = c->params_k; v->params_v = c->params_v;
  v->win_k = c->win_k; v->win_v = c->win_v;
  v->A_k = c->A_k; v->B_k = c->B_k; v->A_v = c->A_v; v->B_v = c->B_v;
  v->groups_k = c->G_k; v->groups_v = c->G_v;
  v->capacity = c->desc.capacity; v->window_slots = c->win_slots;
  v->int4_blocks = c->latent_kind == LK_INT4 ? (int32_t)(c->lat_cap / kI4Block) : 0;
  v->n_pages = c->n_pages;
  return LR_OK;
}

lr_status lr_cache_set_block_table(lr_cache* c, const int32_t* table, void* stream) {
  if (!c) return LR_ERR_INVALID_ARG;
  if (!c->ptable) return LR_ERR_UNSUPPORTED;
  if (!table) return LR_ERR_INVALID_ARG;
  const size_t n = (size_t)c->desc.batch * c->pps;
  for (size_t i = 0; i < n; ++i)
    if (table[i] < 0 || table[i] >= c->n_pages) return LR_ERR_INVALID_ARG;
  // The copy goes from the library's own pageable buffer, which the runtime stages before
  // cudaMemcpyAsync returns: the caller's table (pinned or not) is free on return.
  c->host_table.assign(table, table + n);
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  const cudaError_t e =
      cudaMemcpyAsync(c->ptable, c->host_table.data(), n * sizeof(int32_t), cudaMemcpyHostToDevice, s);
  return e == cudaSuccess ? LR_OK : LR_ERR_CUDA;
}

lr_status lr_cache_set_block_table_device(lr_cache* c, const int32_t* table, void* stream) {
  if (!c) return LR_ERR_INVALID_ARG;
  if (!c->ptable) return LR_ERR_UNSUPPORTED;
  if (!table) return LR_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  c->last_stream = s;
  // a copy, not a kernel: the next kernel on the stream starts only after it has completed,
  // so no dependent launch reads the table early
  const cudaError_t e = cudaMemcpyAsync(c->ptable, table, (size_t)c->desc.batch * c->pps * sizeof(int32_t),
                                        cudaMemcpyDeviceToDevice, s);
  return e == cudaSuccess ? LR_OK : LR_ERR_CUDA;
}

lr_status lr_cache_set_path(lr_cache* c, int32_t path, int32_t n_splits) {
  if (!c || path < 0 || path > 2 || n_splits < 0) return LR_ERR_INVALID_ARG;
  if (path == LR_PATH_TC && !tc_supported(&c->desc)) return LR_ERR_UNSUPPORTED;
  if (n_splits > c->S_max) return LR_ERR_INVALID_ARG;
  c->path_force = path;
  c->splits_force = n_splits;
  return LR_OK;
}

lr_status lr_cache_set_kernel_events(lr_cache* c, void* ev_start, void* ev_stop) {
  if (!c || ((ev_start == nullptr) != (ev_stop == nullptr))) return LR_ERR_INVALID_ARG;
  c->ev_start = (cudaEvent_t)ev_start;
  c->ev_stop = (cudaEvent_t)ev_stop;
  return LR_OK;
}

lr_status lr_cache_set_trace(lr_cache* c, uint64_t* buf, int64_t capacity_words) {
  if (!c) return LR_ERR_INVALID_ARG;
  const int64_t cta_words = (int64_t)LR_TRACE_SLOTS * c->desc.batch * c->S_max;
  if (buf && capacity_words < cta_words + LR_TRACE_SPAN_WORDS) return LR_ERR_CAPACITY;
  c->trace = reinterpret_cast<unsigned long long*>(buf);
  c->spans = buf ? c->trace + cta_words : nullptr;
  return LR_OK;
}

void lr_abi_struct_sizes(int32_t* desc_size, int32_t* view_size, int32_t* plan_size) {
  if (desc_size) *desc_size = (int32_t)sizeof(lr_cache_desc);
  if (view_size) *view_size = (int32_t)sizeof(lr_cache_view);
  if (plan_size) *plan_size = (int32_t)sizeof(lr_plan);
}

lr_status lr_debug_inject_fault(int32_t kind, int64_t after) {
  if (kind != LR_FAULT_ALLOC && kind != LR_FAULT_LAUNCH) return LR_ERR_INVALID_ARG;
  if (after < -1) return LR_ERR_INVALID_ARG;
  g_fault_left[kind].store(after);
  return LR_OK;
}

lr_status lr_cache_set_wait_limit(lr_cache* c, int64_t ns) {
  if (!c || ns < 0) return LR_ERR_INVALID_ARG;
  c->wait_ns = (unsigned long long)ns;
  return LR_OK;
}

lr_status lr_device_error(lr_cache* c, int32_t* code) {
  if (!c || !code) return LR_ERR_INVALID_ARG;
  cudaError_t e = cudaStreamSynchronize(c->last_stream);
  if (e != cudaSuccess) return LR_ERR_CUDA;
  int h = 0;
  e = cudaMemcpy(&h, c->dev_err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(c->dev_err, 0, sizeof(int));
  *code = h;
  return e == cudaSuccess ? LR_OK : LR_ERR_CUDA;
}

}  // extern "C"
