// Decode without device allocation.
//
// Some callers cannot call cudaMalloc at decode time: serving engines that reserve
// almost all HBM up front for their own pools, and latency-critical decode loops that
// cannot afford cudaMalloc's implicit device synchronisation.  lr_attn_decode_noalloc
// runs the fp32 CUDA-core decode path (query projection, split-sequence attention,
// split merge and output projection) over caller-owned latents, with its working
// memory in one fixed static device array instead of cache-owned buffers.
#include "lr_internal.cuh"

#include <mutex>

namespace {

// The working memory: query latents [B][Hq][r_k] and per-split partial results
// ([B][S][Hq][r_v] and [B][S][Hq][2]).  Every GPU that loads the library holds it
// until process exit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the array on the current device (looked up once per device).
cudaError_t scratch_for_current_device(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

size_t scratch_bytes(const lr_cache_desc& d, int splits) {
  const size_t BH = (size_t)d.batch * d.n_q_heads;
  return sizeof(float) * (BH * d.rank_k + BH * splits * d.rank_v + BH * splits * 2);
}

}  // namespace

extern "C" lr_status lr_attn_decode_noalloc(const lr_cache_desc* desc, int32_t len, const void* z_k,
                                            const void* z_v, const void* B_k, const void* B_v, const void* q,
                                            void* out, float* lse, void* stream) {
  if (!desc || !z_k || !z_v || !B_k || !B_v || !q || !out) return LR_ERR_INVALID_ARG;
  // the bases are staged into shared memory with 16-byte copies
  if ((reinterpret_cast<uintptr_t>(B_k) | reinterpret_cast<uintptr_t>(B_v)) & 15) return LR_ERR_INVALID_ARG;
  if (desc->window != 0 || desc->quant_bits != 0 || desc->rope_in_kernel != 0 || desc->latent_groups > 1 ||
      desc->page_tokens != 0)
    return LR_ERR_UNSUPPORTED;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess) return LR_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LR_ERR_CUDA;
  lr_plan plan;
  lr_status st = lr_plan_decode(desc, len, sms, LR_PATH_SIMT, 0, &plan);
  if (st != LR_OK) return st;
  if (len < 1) return LR_ERR_INVALID_ARG;
  // fewer splits when the automatic count does not fit the array
  int splits = plan.n_splits;
  while (splits > 1 && scratch_bytes(*desc, splits) > LR_NOALLOC_SCRATCH_BYTES) splits = (splits + 1) / 2;
  if (scratch_bytes(*desc, splits) > LR_NOALLOC_SCRATCH_BYTES) return LR_ERR_CAPACITY;
  if (splits != plan.n_splits) {
    st = lr_plan_decode(desc, len, sms, LR_PATH_SIMT, splits, &plan);
    if (st != LR_OK) return st;
  }
  void* scratch = nullptr;
  if (scratch_for_current_device(&scratch) != cudaSuccess) return LR_ERR_CUDA;

  // A host-side description of the caller's buffers for the existing launchers.
  lr_cache c;
  c.desc = *desc;
  c.D = desc->n_kv_heads * desc->head_dim;
  c.G_k = c.G_v = 0;
  c.win_slots = 0;
  c.lat_cap = desc->capacity;
  c.len = c.hist_len = len;
  c.win_len = 0;
  c.esize = desc->dtype == LR_BF16 ? 2 : 4;
  c.latent_kind = desc->dtype == LR_BF16 ? LK_BF16 : LK_F32;
  const float sm_scale = desc->softmax_scale > 0.f ? desc->softmax_scale : 1.0f / sqrtf((float)desc->head_dim);
  c.scale_log2 = sm_scale * LR_LOG2E;
  c.z_k = const_cast<void*>(z_k);
  c.z_v = const_cast<void*>(z_v);
  c.B_k = const_cast<void*>(B_k);
  c.B_v = const_cast<void*>(B_v);
  const size_t BH = (size_t)desc->batch * desc->n_q_heads;
  float* base = reinterpret_cast<float*>(scratch);
  c.qt = base;
  c.part_o = base + BH * desc->rank_k;
  c.part_ml = c.part_o + BH * plan.n_splits * desc->rank_v;
  c.S_max = plan.n_splits;
  c.num_sms = sms;
  c.device = dev;
  if (decode_simt_smem(&c) > 227 * 1024) return LR_ERR_UNSUPPORTED;

  cudaStream_t s = (cudaStream_t)stream;
  // The bases belong to the caller, and the kernel just before this call may have written
  // them; the query projection stages B_k in its prologue, so it starts only after that
  // work has completed (no programmatic overlap).  The kernels after it follow their own
  // predecessor, which writes neither basis.
  cudaError_t e = launch_qproj(&c, q, s, /*pdl=*/false);
  if (e == cudaSuccess) e = launch_decode_simt(&c, plan.n_splits, plan.split_tokens, s);
  if (e == cudaSuccess) e = launch_merge(&c, plan.n_splits, out, lse, s);
  return e == cudaSuccess ? LR_OK : LR_ERR_CUDA;
}
