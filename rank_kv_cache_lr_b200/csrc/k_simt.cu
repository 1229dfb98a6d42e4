// CUDA-core kernels of the low-rank KV-cache path: query projection, the
// fp32 split-sequence decode (every configuration, the only path for fp32
// caches), the exact window, the split merge with the output projection,
// append/fold/quantise, the latent bulk fill and the basis sync.
//
// Method: TraceKV abstract (latent KV storage with quantization, low-rank
// attention kernels) and iS-KV abstract/method section (exact recent window,
// folding, historical-coordinate synchronisation).  Attention is computed in
// rank space: q~_j = s log2(e) B_k,h(j) q_j, score_t = q~_j . z_t,
// o~_j = sum_t p_t z_v,t, o_j = o~_j B_v,h(j) / l — the exact identity
// q . (z B_h) = (B_h q) . z, so the result equals attention over the
// reconstructed keys and values.
#include "lr_internal.cuh"

#include <math.h>

#include <algorithm>

namespace {

constexpr int kTileSimt = 16;     // tokens per tile in the SIMT decode
constexpr int kSyncRows = 16;     // rows per CTA in the SIMT basis sync

__device__ __forceinline__ float elem_f(const void* p, long long idx, int dtype) {
  if (dtype == LR_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[idx]);
  return reinterpret_cast<const float*>(p)[idx];
}

__device__ __forceinline__ void store_elem(void* p, long long idx, float v, int dtype) {
  if (dtype == LR_BF16) reinterpret_cast<__nv_bfloat16*>(p)[idx] = __float2bfloat16_rn(v);
  else reinterpret_cast<float*>(p)[idx] = v;
}

// One stored latent coordinate as fp32.  int4: x^ = code * scale + zero (the
// product is exact in fp32, so this is the fp32 rounding of the exact value).
__device__ __forceinline__ float latent_f(const LatentRef& L, int kind, int dtype,
                                          long long row, int i) {
  if (kind == LK_INT4) {
    const uint32_t w = L.codes[row * (L.G * 4) + (i >> 3)];
    const float code = (float)((w >> (4 * (i & 7))) & 15u);
    const uint32_t p = L.params[row * L.G + (i >> 5)];
    const float scale = __half2float(__ushort_as_half((unsigned short)(p & 0xFFFFu)));
    const float zero = __half2float(__ushort_as_half((unsigned short)(p >> 16)));
    return fmaf(code, scale, zero);
  }
  return elem_f(L.z, row * L.r + i, dtype);
}

// Warp-cooperative int4 quantisation of one group of 32 coordinates (lane = element;
// lanes with valid == false are padding).  Reading of the quantiser (the pages give
// none): zero = fp16(min), scale = fp16((max - min) / 15) in fp32, code =
// clamp(rint((x - zero) / scale), 0, 15) in IEEE fp32, 0 if scale == 0; a zero
// point of -0 is stored as +0.  Writes 4 packed words and the {scale, zero} word.
__device__ __forceinline__ void quant_group_warp(float x, bool valid, uint32_t* words,
                                                 uint32_t* param) {
  const int lane = threadIdx.x & 31;
  float mn = valid ? x : INFINITY;
  float mx = valid ? x : -INFINITY;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  __half zh = __float2half_rn(mn);
  if (__half2float(zh) == 0.0f) zh = __ushort_as_half((unsigned short)0);
  const __half sh = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
  const float zf = __half2float(zh), sf = __half2float(sh);
  uint32_t code = 0;
  if (valid && sf != 0.0f) {
    float t = rintf(__fdiv_rn(__fsub_rn(x, zf), sf));
    t = fminf(fmaxf(t, 0.0f), 15.0f);
    code = (uint32_t)t;
  }
  uint32_t v = code << (4 * (lane & 7));
  v |= __shfl_xor_sync(0xffffffffu, v, 1);
  v |= __shfl_xor_sync(0xffffffffu, v, 2);
  v |= __shfl_xor_sync(0xffffffffu, v, 4);
  if ((lane & 7) == 0) words[lane >> 3] = v;
  if (lane == 0) *param = (uint32_t)__half_as_ushort(sh) | ((uint32_t)__half_as_ushort(zh) << 16);
}

// Store one warp's 32-coordinate chunk `ch` of a latent row (lane = coordinate).
__device__ __forceinline__ void store_latent_chunk(float z, int ch, int r, int kind, int dtype,
                                                   void* Z, uint32_t* codes, uint32_t* params,
                                                   int G, long long row) {
  const int lane = threadIdx.x & 31;
  const int i = ch * 32 + lane;
  const bool valid = i < r;
  if (kind == LK_INT4) {
    quant_group_warp(z, valid, codes + row * (G * 4) + ch * 4, params + row * G + ch);
  } else if (valid) {
    store_elem(Z, row * r + i, z, dtype);
  }
}

// ---- cp.async staging (16-byte asynchronous global -> shared copies) --------------
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem)),
               "l"(gmem)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

// Copy rows [r0, r0 + nr) x columns [col0, col0 + ncol) of a row-major matrix with row
// stride ld (elements of `es` bytes) into shared memory with row pitch `pitch` bytes.
// ncol * es must be a multiple of 16 and the source 16-byte aligned.
__device__ __forceinline__ void stage_rows(uint8_t* dst, int pitch, const void* src, long long ld, int es,
                                           int r0, int nr, long long col0, int ncol) {
  const int vec_per_row = ncol * es / 16;
  const int total = nr * vec_per_row;
  const uint8_t* g = reinterpret_cast<const uint8_t*>(src);
  for (int v = threadIdx.x; v < total; v += blockDim.x) {
    const int rr = v / vec_per_row, cc = v % vec_per_row;
    cp_async16(dst + rr * pitch + cc * 16, g + (((long long)(r0 + rr) * ld + col0) * es) + cc * 16);
  }
}

__device__ __forceinline__ float smem_elem(const uint8_t* p, int dtype) {
  if (dtype == LR_BF16) return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
  return *reinterpret_cast<const float*>(p);
}

// ---------------------------------------------------------------------------
// query projection: q~ = s log2(e) B_k,h q  (latent path) and/or s log2(e) q
// ---------------------------------------------------------------------------
// One CTA per (32-row chunk of B_k,h, KV head h, sequence b).  The chunk's rows
// (32 x d) and the group's queries are staged in shared memory; thread = (rank row,
// query head): one d-long dot product each.
// qt16 (tensor-core path): rows [b][j] and [b][32 + j] of a [B][64][r_k] bf16 array get
// hi = bf16(q~) and lo = bf16(q~ - hi), so that hi + lo carries q~ to ~16 significant bits.
constexpr int kRowsQ = 32;

struct QprojArgs {
  const void* q; const void* Bk; float* qt; float* qd; __nv_bfloat16* qt16;
  int Hq, Hkv, d, D, rk, dtype;
  float scale_log2;
  int want_latent;
};

__device__ __forceinline__ void qproj_body(const QprojArgs& a, int rchunk, int h, int b, uint8_t* qsm) {
  const int Hq = a.Hq, d = a.d, D = a.D, rk = a.rk, dtype = a.dtype;
  const float scale_log2 = a.scale_log2;
  const int G = Hq / a.Hkv;
  const int r0 = rchunk * kRowsQ;
  const int j0 = h * G;
  const int es = dtype == LR_BF16 ? 2 : 4;
  const int pitch = d * es + 16;
  float* qs = reinterpret_cast<float*>(qsm);                                   // [G][d]
  uint8_t* bs = qsm + (((size_t)G * d * sizeof(float) + 15) & ~size_t(15));   // [32][pitch]
  const int nr = min(kRowsQ, rk - r0);
  if (a.want_latent && nr > 0) stage_rows(bs, pitch, a.Bk, D, es, r0, nr, (long long)h * d, d);
#pragma unroll 4
  for (int idx = threadIdx.x; idx < G * d; idx += blockDim.x) {
    const long long off = ((long long)b * Hq + j0) * d + idx;
    const float v = elem_f(a.q, off, dtype);
    qs[idx] = v;
    if (a.qd && rchunk == 0) a.qd[off] = v * scale_log2;
  }
  if (!a.want_latent) return;
  cp_async_wait_all();
  __syncthreads();
  const int lane = threadIdx.x & 31, hs0 = threadIdx.x >> 5;
  if (lane >= nr) return;
  const uint8_t* row = bs + lane * pitch;
  const int i = r0 + lane;
  for (int hs = hs0; hs < G; hs += 8) {
    const float* qr = qs + hs * d;
    float a0 = 0.f, a1 = 0.f;
    for (int c = 0; c < d; c += 8) {
      float bv[8];
      if (dtype == LR_BF16) {
        const uint4 u4 = *reinterpret_cast<const uint4*>(row + c * 2);
        const uint32_t w[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          bv[2 * k] = __uint_as_float(w[k] << 16);
          bv[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
        }
      } else {
        const float4 f0 = *reinterpret_cast<const float4*>(row + c * 4);
        const float4 f1 = *reinterpret_cast<const float4*>(row + c * 4 + 16);
        bv[0] = f0.x; bv[1] = f0.y; bv[2] = f0.z; bv[3] = f0.w;
        bv[4] = f1.x; bv[5] = f1.y; bv[6] = f1.z; bv[7] = f1.w;
      }
      const float4 q0 = *reinterpret_cast<const float4*>(qr + c);
      const float4 q1 = *reinterpret_cast<const float4*>(qr + c + 4);
      a0 = fmaf(bv[0], q0.x, a0); a1 = fmaf(bv[1], q0.y, a1);
      a0 = fmaf(bv[2], q0.z, a0); a1 = fmaf(bv[3], q0.w, a1);
      a0 = fmaf(bv[4], q1.x, a0); a1 = fmaf(bv[5], q1.y, a1);
      a0 = fmaf(bv[6], q1.z, a0); a1 = fmaf(bv[7], q1.w, a1);
    }
    const int j = j0 + hs;
    const float v = (a0 + a1) * scale_log2;
    a.qt[((long long)b * Hq + j) * rk + i] = v;
    if (a.qt16) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(v);
      const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
      a.qt16[((long long)b * 64 + j) * rk + i] = hi;
      a.qt16[((long long)b * 64 + 32 + j) * rk + i] = lo;
    }
  }
}

__global__ void __launch_bounds__(256) k_qproj(QprojArgs a) {
  extern __shared__ __align__(16) uint8_t qsm[];
  pdl_wait();
  pdl_trigger();
  qproj_body(a, blockIdx.x, blockIdx.y, blockIdx.z, qsm);
}

size_t qproj_smem(const lr_cache_desc& d, size_t es) {
  return (((size_t)(d.n_q_heads / d.n_kv_heads) * d.head_dim * sizeof(float) + 15) & ~size_t(15)) +
         (size_t)kRowsQ * (d.head_dim * es + 16);
}

// ---------------------------------------------------------------------------
// split-sequence decode on CUDA cores (fp32 arithmetic throughout)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_decode_simt(DecodeSimtArgs a, int kind) {
  extern __shared__ float sm[];
  pdl_wait();
  pdl_trigger();
  const int split = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, nt = blockDim.x;
  const int Hq = a.Hq, rk = a.k.r, rv = a.v.r;
  const int qdim = a.rope ? a.d : rk;
  const int qstride = qdim + 1;
  float* q_s = sm;                        // [Hq][qdim+1]
  float* zk_s = q_s + Hq * qstride;       // [T][rk]
  float* zv_s = zk_s + kTileSimt * rk;    // [T][rv]
  float* sc = zv_s + kTileSimt * rv;      // [T][Hq]
  float* acc = sc + kTileSimt * Hq;       // [Hq][rv]
  float* m_s = acc + Hq * rv;
  float* l_s = m_s + Hq;
  float* al_s = l_s + Hq;
  float* kh = al_s + Hq;                  // [T][D] (RoPE path)

  const float* qsrc = a.qs + (size_t)b * Hq * qdim;
  for (int idx = tid; idx < Hq * qdim; idx += nt) q_s[(idx / qdim) * qstride + idx % qdim] = qsrc[idx];
  for (int idx = tid; idx < Hq * rv; idx += nt) acc[idx] = 0.f;
  for (int j = tid; j < Hq; j += nt) { m_s[j] = -INFINITY; l_s[j] = 0.f; }
  __syncthreads();

  const int group = Hq / a.Hkv;
  const int t_begin = split * a.split_tokens;
  const int t_end = min(a.hist_len, t_begin + a.split_tokens);
  for (int t0 = t_begin; t0 < t_end; t0 += kTileSimt) {
    const int n = min(kTileSimt, t_end - t0);
    const long long row0 = (long long)b * a.k.cap + t0;
    for (int idx = tid; idx < n * rk; idx += nt) {
      const int t = idx / rk, i = idx % rk;
      zk_s[t * rk + i] = latent_f(a.k, kind, a.dtype, row0 + t, i);
    }
    for (int idx = tid; idx < n * rv; idx += nt) {
      const int t = idx / rv, i = idx % rv;
      zv_s[t * rv + i] = latent_f(a.v, kind, a.dtype, row0 + t, i);
    }
    __syncthreads();
    if (a.rope) {
      for (int c = tid; c < a.D; c += nt) {
        float accum[kTileSimt];
#pragma unroll
        for (int t = 0; t < kTileSimt; ++t) accum[t] = 0.f;
        for (int i = 0; i < rk; ++i) {
          const float bv = elem_f(a.B_k, (long long)i * a.D + c, a.dtype);
#pragma unroll
          for (int t = 0; t < kTileSimt; ++t) accum[t] = fmaf(zk_s[t * rk + i], bv, accum[t]);
        }
        for (int t = 0; t < n; ++t) kh[t * a.D + c] = accum[t];
      }
      __syncthreads();
      const int half = a.d / 2;
      for (int idx = tid; idx < n * a.Hkv * half; idx += nt) {
        const int t = idx / (a.Hkv * half);
        const int rem = idx % (a.Hkv * half);
        const int h = rem / half, i = rem % half;
        const float2 cs = a.rope_cs[(long long)(t0 + t) * half + i];
        float* row = kh + t * a.D + h * a.d;
        const float x1 = row[i], x2 = row[i + half];
        row[i] = x1 * cs.x - x2 * cs.y;
        row[i + half] = x2 * cs.x + x1 * cs.y;
      }
      __syncthreads();
    }
    for (int p = tid; p < n * Hq; p += nt) {
      const int t = p / Hq, j = p % Hq;
      const float* qv = q_s + j * qstride;
      float s = 0.f;
      if (a.rope) {
        const float* kv = kh + t * a.D + (j / group) * a.d;
        for (int c = 0; c < a.d; ++c) s = fmaf(qv[c], kv[c], s);
      } else {
        const float* zr = zk_s + t * rk;
        for (int i = 0; i < rk; ++i) s = fmaf(qv[i], zr[i], s);
      }
      sc[t * Hq + j] = s;
    }
    __syncthreads();
    for (int j = tid; j < Hq; j += nt) {
      float mt = -INFINITY;
      for (int t = 0; t < n; ++t) mt = fmaxf(mt, sc[t * Hq + j]);
      const float mo = m_s[j];
      const float mnew = fmaxf(mo, mt);
      const float alpha = (mo == -INFINITY) ? 0.f : exp2f(mo - mnew);
      float sum = 0.f;
      for (int t = 0; t < n; ++t) {
        const float p = exp2f(sc[t * Hq + j] - mnew);
        sc[t * Hq + j] = p;
        sum += p;
      }
      l_s[j] = l_s[j] * alpha + sum;
      m_s[j] = mnew;
      al_s[j] = alpha;
    }
    __syncthreads();
    for (int idx = tid; idx < Hq * rv; idx += nt) {
      const int j = idx / rv, i = idx % rv;
      float o = acc[idx] * al_s[j];
      for (int t = 0; t < n; ++t) o = fmaf(sc[t * Hq + j], zv_s[t * rv + i], o);
      acc[idx] = o;
    }
    __syncthreads();
  }
  const size_t base = ((size_t)b * a.n_splits + split) * Hq;
  for (int idx = tid; idx < Hq * rv; idx += nt) a.part_o[base * rv + idx] = acc[idx];
  for (int j = tid; j < Hq; j += nt) {
    a.part_ml[(base + j) * 2] = m_s[j];
    a.part_ml[(base + j) * 2 + 1] = l_s[j];
  }
}

// ---------------------------------------------------------------------------
// exact window (iS-KV): attention of each query head over the window tokens of
// its KV head, as one more partial (in head space, relative to its own max)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) k_window(const void* win_k, const void* win_v, const float* qd,
                                                float* win_o, float* win_ml, int Hq, int Hkv, int d,
                                                int D, int slots, int hist_len, int win_len, int dtype) {
  extern __shared__ float wsm[];
  float* q_s = wsm;           // [d]
  float* p_s = wsm + d;       // [win_len]
  __shared__ float red[2];
  pdl_wait();
  pdl_trigger();
  const int j = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  const int h = j / (Hq / Hkv);
  const int warp = tid >> 5, lane = tid & 31, nw = blockDim.x >> 5;
  for (int c = tid; c < d; c += blockDim.x) q_s[c] = qd[((long long)b * Hq + j) * d + c];
  __syncthreads();
  for (int t = warp; t < win_len; t += nw) {
    const int slot = (hist_len + t) % slots;
    const long long off = ((long long)b * slots + slot) * D + (long long)h * d;
    float s = 0.f;
    for (int c = lane; c < d; c += 32) s = fmaf(q_s[c], elem_f(win_k, off + c, dtype), s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) p_s[t] = s;
  }
  __syncthreads();
  if (tid == 0) {
    float m = -INFINITY;
    for (int t = 0; t < win_len; ++t) m = fmaxf(m, p_s[t]);
    float l = 0.f;
    for (int t = 0; t < win_len; ++t) {
      const float p = exp2f(p_s[t] - m);
      p_s[t] = p;
      l += p;
    }
    red[0] = m;
    red[1] = l;
  }
  __syncthreads();
  for (int c = tid; c < d; c += blockDim.x) {
    float o = 0.f;
    for (int t = 0; t < win_len; ++t) {
      const int slot = (hist_len + t) % slots;
      o = fmaf(p_s[t], elem_f(win_v, ((long long)b * slots + slot) * D + (long long)h * d + c, dtype), o);
    }
    win_o[((long long)b * Hq + j) * d + c] = o;
  }
  if (tid == 0) {
    win_ml[((long long)b * Hq + j) * 2] = red[0];
    win_ml[((long long)b * Hq + j) * 2 + 1] = red[1];
  }
}

// ---------------------------------------------------------------------------
// split merge (log-sum-exp) and output projection o = o~ B_v,h / l.
// One CTA (512 threads) per (KV head h, sequence b).  The B_v,h slice is prefetched
// into shared memory with asynchronous copies while the split weights and the
// combined rank-space outputs o~ of the group's query heads are formed; o~ is kept
// rank-major with the heads padded to a multiple of 4.  The projection is register
// blocked: thread = (column pair, block of 4 heads, rank slice), and the rank slices
// are summed through shared memory in a fixed order.
// ---------------------------------------------------------------------------
constexpr int kMergeThreads = 512;
constexpr size_t kMergeStage = 96 * 1024;   // bytes of B_v,h rows staged in shared memory

template <typename T>
__device__ __forceinline__ float2 load_pair(const uint8_t* p);
template <>
__device__ __forceinline__ float2 load_pair<__nv_bfloat16>(const uint8_t* p) {
  const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
template <>
__device__ __forceinline__ float2 load_pair<float>(const uint8_t* p) {
  return *reinterpret_cast<const float2*>(p);
}

template <typename T>
__global__ void __launch_bounds__(kMergeThreads) k_merge(const float* part_o, const float* part_ml,
                                                         const float* win_o, const float* win_ml,
                                                         const T* Bv, T* out, float* lse, int S, int Hq,
                                                         int Hkv, int d, int D, int rv) {
  extern __shared__ __align__(16) float msm[];
  const int G = Hq / Hkv;
  const int G4 = (G + 3) & ~3;
  const int HB = G4 / 4;
  float* ot = msm;                 // [rv][G4]  (rank-major)
  float* w_s = ot + rv * G4;       // [G][S]
  float* hdr = w_s + G * S;        // [G][3]: m*, 1/l, window weight
  float* red = hdr + G * 3;        // [RS][G4][d] partial projections
  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int j0 = h * G;
  const int warp = tid >> 5, lane = tid & 31, nw = nt >> 5;
  constexpr int es = sizeof(T);
  const int pitch = d * es;
  const int npairs = d / 2;
  const int combos = npairs * HB;
  const int RS = max(1, nt / combos);
  const size_t fl = (size_t)rv * G4 + (size_t)G * S + 3 * G + (size_t)RS * G4 * d;
  uint8_t* bs = reinterpret_cast<uint8_t*>(msm) + ((fl * sizeof(float) + 15) & ~size_t(15));   // 16-B aligned
  const int rows_staged = min(rv, (int)(kMergeStage / pitch));
  stage_rows(bs, pitch, Bv, D, es, 0, rows_staged, (long long)h * d, d);   // bases: stable data
  pdl_wait();
  pdl_trigger();
  for (int jj = warp; jj < G; jj += nw) {
    const int j = j0 + jj;
    float m = -INFINITY;
    for (int s = lane; s < S; s += 32) m = fmaxf(m, part_ml[(((size_t)b * S + s) * Hq + j) * 2]);
    const float mw = win_ml ? win_ml[((size_t)b * Hq + j) * 2] : -INFINITY;
    m = fmaxf(m, mw);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float l = 0.f;
    for (int s = lane; s < S; s += 32) {
      const size_t e = (((size_t)b * S + s) * Hq + j) * 2;
      const float ms = part_ml[e];
      const float w = (ms == -INFINITY) ? 0.f : exp2f(ms - m);
      w_s[jj * S + s] = w;
      l = fmaf(w, part_ml[e + 1], l);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      float ww = 0.f;
      if (win_ml && mw != -INFINITY) {
        ww = exp2f(mw - m);
        l = fmaf(ww, win_ml[((size_t)b * Hq + j) * 2 + 1], l);
      }
      hdr[jj * 3] = m;
      hdr[jj * 3 + 1] = 1.0f / l;
      hdr[jj * 3 + 2] = ww;
      if (lse) lse[(long long)b * Hq + j] = (m + log2f(l)) * LR_LN2;
    }
  }
  for (int idx = tid; idx < rv * (G4 - G); idx += nt) {       // zero the padding heads
    const int i = idx / (G4 - G), jj = G + idx % (G4 - G);
    ot[i * G4 + jj] = 0.f;
  }
  __syncthreads();
  // combine: thread = (rank i, head slot); the loads of 2 heads x 8 splits are issued
  // together before any is used, so each thread waits for about one memory round trip
  // per 16 partial values
  const size_t sstride = (size_t)Hq * rv;
  const int jslots = max(1, nt / rv);
  for (int t = tid; t < rv * jslots; t += nt) {
    const int i = t % rv, js = t / rv;
    for (int jj = js; jj < G; jj += 2 * jslots) {
      const int jj2 = jj + jslots;
      const bool two = jj2 < G;
      const float* src = part_o + (((size_t)b * S) * Hq + j0 + jj) * rv + i;
      const float* src2 = part_o + (((size_t)b * S) * Hq + j0 + (two ? jj2 : jj)) * rv + i;
      float acc = 0.f, acc2 = 0.f;
      for (int s0 = 0; s0 < S; s0 += 8) {
        float v[8], v2[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const bool in = s0 + k < S;
          v[k] = in ? __ldg(src + (size_t)(s0 + k) * sstride) : 0.f;
          v2[k] = (in && two) ? __ldg(src2 + (size_t)(s0 + k) * sstride) : 0.f;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (s0 + k < S) {
            acc = fmaf(w_s[jj * S + s0 + k], v[k], acc);
            if (two) acc2 = fmaf(w_s[jj2 * S + s0 + k], v2[k], acc2);
          }
        }
      }
      ot[i * G4 + jj] = acc;
      if (two) ot[i * G4 + jj2] = acc2;
    }
  }
  cp_async_wait_all();
  __syncthreads();
  // projection
  for (int t = tid; t < combos * RS; t += nt) {
    const int cp = t % npairs;
    const int hb = (t / npairs) % HB;
    const int rs = t / combos;
    const int per = (rv + RS - 1) / RS;
    const int i0 = rs * per, i1 = min(rv, i0 + per);
    float acc[4][2];
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u][0] = acc[u][1] = 0.f;
    for (int i = i0; i < i1; ++i) {
      const float2 bv = i < rows_staged
                            ? load_pair<T>(bs + i * pitch + cp * 2 * es)
                            : load_pair<T>(reinterpret_cast<const uint8_t*>(Bv + (size_t)i * D + (size_t)h * d + 2 * cp));
      const float4 o4 = *reinterpret_cast<const float4*>(ot + i * G4 + hb * 4);
      acc[0][0] = fmaf(o4.x, bv.x, acc[0][0]); acc[0][1] = fmaf(o4.x, bv.y, acc[0][1]);
      acc[1][0] = fmaf(o4.y, bv.x, acc[1][0]); acc[1][1] = fmaf(o4.y, bv.y, acc[1][1]);
      acc[2][0] = fmaf(o4.z, bv.x, acc[2][0]); acc[2][1] = fmaf(o4.z, bv.y, acc[2][1]);
      acc[3][0] = fmaf(o4.w, bv.x, acc[3][0]); acc[3][1] = fmaf(o4.w, bv.y, acc[3][1]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float* rr = red + ((size_t)rs * G4 + hb * 4 + u) * d + 2 * cp;
      rr[0] = acc[u][0];
      rr[1] = acc[u][1];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * d; idx += nt) {
    const int jj = idx / d, c = idx % d;
    float o = 0.f;
    for (int r = 0; r < RS; ++r) o += red[((size_t)r * G4 + jj) * d + c];
    const long long ooff = ((long long)b * Hq + j0 + jj) * d + c;
    if (win_o) o = fmaf(hdr[jj * 3 + 2], win_o[ooff], o);
    o *= hdr[jj * 3 + 1];
    if constexpr (sizeof(T) == 2) out[ooff] = __float2bfloat16_rn(o);
    else out[ooff] = o;
  }
}

size_t merge_smem(const lr_cache_desc& d, int S, size_t es) {
  const int G = d.n_q_heads / d.n_kv_heads;
  const int G4 = (G + 3) & ~3;
  const int combos = (d.head_dim / 2) * (G4 / 4);
  const int RS = std::max(1, kMergeThreads / combos);
  const size_t stage = std::min(kMergeStage, (size_t)d.rank_v * d.head_dim * es);
  const size_t fl = (size_t)d.rank_v * G4 + (size_t)G * S + 3 * G + (size_t)RS * G4 * d.head_dim;
  return ((fl * sizeof(float) + 15) & ~size_t(15)) + stage;
}

// ---------------------------------------------------------------------------
// append: project one token per sequence (z = x A) and store / quantise it;
// optionally write the new exact token into the window ring
// ---------------------------------------------------------------------------
struct AppendArgs {
  const void* src_k; const void* src_v;   // rows to project (input or evicted ring rows)
  long long src_bstride;                  // elements between batch rows of src
  const void* A_k; const void* A_v;
  void* Zk; void* Zv; uint32_t* codes_k; uint32_t* codes_v; uint32_t* params_k; uint32_t* params_v;
  int rk, rv, Gk, Gv, chunks_k, chunks_v;
  long long cap; int dst_slot; int project;
  const void* new_k; const void* new_v;   // exact token for the ring, or null
  void* win_k; void* win_v; int slots; int new_slot;
  int B, D, kind, dtype;
};

// One CTA per (32-coordinate chunk of K or V, sequence b).  The chunk's columns of A
// ([D][32]) and the source row are staged in shared memory with asynchronous copies;
// the 8 warps take fixed eighths of the D-long dot products and the partial sums are
// added in a fixed order, so the result does not depend on the storage kind.
__device__ __forceinline__ void append_body(const AppendArgs& a, int x, int b, uint8_t* asm_, float (*red)[32]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nproj = a.project ? (a.chunks_k + a.chunks_v) : 0;
  const int es = a.dtype == LR_BF16 ? 2 : 4;
  if (x < nproj) {
    const bool is_k = x < a.chunks_k;
    const int ch = is_k ? x : x - a.chunks_k;
    const int r = is_k ? a.rk : a.rv;
    const void* A = is_k ? a.A_k : a.A_v;
    const void* src = is_k ? a.src_k : a.src_v;
    const int ncol = min(32, r - ch * 32);         // 16 or 32 (ranks are multiples of 16)
    uint8_t* As = asm_;                            // [D][32], pitch 32 * es
    uint8_t* xs = asm_ + (size_t)a.D * 32 * es;    // [D]
    stage_rows(As, 32 * es, A, r, es, 0, a.D, (long long)ch * 32, ncol);
    const uint8_t* g = reinterpret_cast<const uint8_t*>(src) + (size_t)b * a.src_bstride * es;
    for (int v = threadIdx.x; v < a.D * es / 16; v += blockDim.x) cp_async16(xs + v * 16, g + v * 16);
    cp_async_wait_all();
    __syncthreads();
    const int per = (a.D + 7) / 8;
    const int cb = warp * per, ce = min(a.D, cb + per);
    float z0 = 0.f, z1 = 0.f;
    if (lane < ncol) {
      int c = cb;
      for (; c + 1 < ce; c += 2) {
        z0 = fmaf(smem_elem(xs + c * es, a.dtype), smem_elem(As + (c * 32 + lane) * es, a.dtype), z0);
        z1 = fmaf(smem_elem(xs + (c + 1) * es, a.dtype), smem_elem(As + ((c + 1) * 32 + lane) * es, a.dtype), z1);
      }
      if (c < ce) z0 = fmaf(smem_elem(xs + c * es, a.dtype), smem_elem(As + (c * 32 + lane) * es, a.dtype), z0);
    }
    red[warp][lane] = z0 + z1;
    __syncthreads();
    if (warp == 0) {
      float z = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) z += red[w][lane];
      const long long row = (long long)b * a.cap + a.dst_slot;
      store_latent_chunk(z, ch, r, a.kind, a.dtype, is_k ? a.Zk : a.Zv, is_k ? a.codes_k : a.codes_v,
                         is_k ? a.params_k : a.params_v, is_k ? a.Gk : a.Gv, row);
    }
    return;
  }
  // ring write of the exact new token of sequence b
  const bool is_k = (x - nproj) == 0;
  const void* src = is_k ? a.new_k : a.new_v;
  void* dst = is_k ? a.win_k : a.win_v;
  for (int c = threadIdx.x; c < a.D; c += blockDim.x) {
    const long long so = (long long)b * a.D + c;
    const long long dof = ((long long)b * a.slots + a.new_slot) * a.D + c;
    if (a.dtype == LR_BF16) reinterpret_cast<uint16_t*>(dst)[dof] = reinterpret_cast<const uint16_t*>(src)[so];
    else reinterpret_cast<uint32_t*>(dst)[dof] = reinterpret_cast<const uint32_t*>(src)[so];
  }
}

__global__ void __launch_bounds__(256) k_append(AppendArgs a) {
  extern __shared__ __align__(16) uint8_t asm_[];
  __shared__ float red[8][32];
  pdl_wait();
  pdl_trigger();
  append_body(a, blockIdx.x, blockIdx.y, asm_, red);
}

// One decode step's independent first half in one grid: CTAs [0, x_app) of each row
// are the append of the new token (projection / ring write), the others the query
// projection (rank chunk, KV head).
__global__ void __launch_bounds__(256) k_step_pre(AppendArgs aa, QprojArgs qa, int x_app, int nchunks_q) {
  extern __shared__ __align__(16) uint8_t psm[];
  __shared__ float red[8][32];
  pdl_wait();
  pdl_trigger();
  const int x = blockIdx.x, b = blockIdx.y;
  if (x < x_app) append_body(aa, x, b, psm, red);
  else qproj_body(qa, (x - x_app) % nchunks_q, (x - x_app) / nchunks_q, b, psm);
}

// bulk latent fill: one warp per (token, 32-coordinate chunk)
__global__ void __launch_bounds__(256) k_append_latent(const float* zk, const float* zv, int n, int B,
                                                       int rk, int rv, int chunks_k, int chunks_v,
                                                       void* Zk, void* Zv, uint32_t* codes_k,
                                                       uint32_t* codes_v, uint32_t* params_k,
                                                       uint32_t* params_v, int Gk, int Gv,
                                                       long long cap, int slot0, int kind, int dtype) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long pi = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
  const int per_tok = chunks_k + chunks_v;
  const int b = blockIdx.y;
  if (pi >= (long long)n * per_tok) return;
  const int t = (int)(pi / per_tok), c = (int)(pi % per_tok);
  const bool is_k = c < chunks_k;
  const int ch = is_k ? c : c - chunks_k;
  const int r = is_k ? rk : rv;
  const float* src = is_k ? zk : zv;
  const int i = ch * 32 + lane;
  const float z = i < r ? src[((long long)b * n + t) * r + i] : 0.f;
  const long long row = (long long)b * cap + slot0 + t;
  store_latent_chunk(z, ch, r, kind, dtype, is_k ? Zk : Zv, is_k ? codes_k : codes_v,
                     is_k ? params_k : params_v, is_k ? Gk : Gv, row);
}

// basis sync on CUDA cores: Z[b][t][:] <- Z[b][t][:] R for t < hist_len (in place)
__global__ void __launch_bounds__(256) k_sync_simt(void* Z, const float* R, int r, long long cap,
                                                   int hist_len, int dtype) {
  extern __shared__ float zs[];   // [kSyncRows][r]
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int t0 = blockIdx.x * kSyncRows;
  const int n = min(kSyncRows, hist_len - t0);
  for (int idx = threadIdx.x; idx < n * r; idx += blockDim.x) {
    const int t = idx / r, k = idx % r;
    zs[t * r + k] = elem_f(Z, ((long long)b * cap + t0 + t) * r + k, dtype);
  }
  __syncthreads();
  for (int col = threadIdx.x; col < r; col += blockDim.x) {
    float acc[kSyncRows];
#pragma unroll
    for (int t = 0; t < kSyncRows; ++t) acc[t] = 0.f;
    for (int k = 0; k < r; ++k) {
      const float rv = R[(long long)k * r + col];
#pragma unroll
      for (int t = 0; t < kSyncRows; ++t) acc[t] = fmaf(zs[t * r + k], rv, acc[t]);
    }
    for (int t = 0; t < n; ++t) store_elem(Z, ((long long)b * cap + t0 + t) * r + col, acc[t], dtype);
  }
}

LatentRef latent_ref(const lr_cache* c, bool k) {
  LatentRef L;
  L.z = k ? c->z_k : c->z_v;
  L.codes = k ? c->codes_k : c->codes_v;
  L.params = k ? c->params_k : c->params_v;
  L.r = k ? c->desc.rank_k : c->desc.rank_v;
  L.G = k ? c->G_k : c->G_v;
  L.cap = c->desc.capacity;
  return L;
}

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

static QprojArgs make_qproj_args(const lr_cache* c, const void* q, bool tc) {
  const lr_cache_desc& d = c->desc;
  const bool rope = d.rope_in_kernel != 0;
  QprojArgs a;
  a.q = q;
  a.Bk = c->B_k;
  a.qt = c->qt;
  a.qd = (rope || c->win_slots) ? (rope ? c->qt : c->qt + (size_t)d.batch * d.n_q_heads * d.rank_k) : nullptr;
  a.qt16 = tc ? (__nv_bfloat16*)c->qt16 : nullptr;
  a.Hq = d.n_q_heads; a.Hkv = d.n_kv_heads; a.d = d.head_dim; a.D = c->D; a.rk = d.rank_k; a.dtype = d.dtype;
  a.scale_log2 = c->scale_log2;
  a.want_latent = rope ? 0 : 1;
  return a;
}

static int qproj_chunks(const lr_cache* c) {
  return c->desc.rope_in_kernel ? 1 : (c->desc.rank_k + kRowsQ - 1) / kRowsQ;
}

static cudaError_t qproj(const lr_cache* c, const void* q, cudaStream_t s, bool tc) {
  const lr_cache_desc& d = c->desc;
  dim3 grid(qproj_chunks(c), d.n_kv_heads, d.batch);
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_qproj, optin_done);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_qproj, grid, dim3(256), qproj_smem(d, c->esize), s, make_qproj_args(c, q, tc));
}

cudaError_t launch_qproj(const lr_cache* c, const void* q, cudaStream_t s) { return qproj(c, q, s, false); }

cudaError_t launch_qproj_tc(const lr_cache* c, const void* q, cudaStream_t s) {
  if (!c->qt16) return cudaErrorNotSupported;
  return qproj(c, q, s, true);
}

size_t decode_simt_smem(const lr_cache* c) {
  const lr_cache_desc& d = c->desc;
  const int qdim = d.rope_in_kernel ? d.head_dim : d.rank_k;
  size_t f = (size_t)d.n_q_heads * (qdim + 1) + (size_t)kTileSimt * d.rank_k + (size_t)kTileSimt * d.rank_v +
             (size_t)kTileSimt * d.n_q_heads + (size_t)d.n_q_heads * d.rank_v + 3 * (size_t)d.n_q_heads;
  if (d.rope_in_kernel) f += (size_t)kTileSimt * c->D;
  return f * sizeof(float);
}

cudaError_t launch_decode_simt(const lr_cache* c, int n_splits, int split_tokens, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  DecodeSimtArgs a;
  a.k = latent_ref(c, true);
  a.v = latent_ref(c, false);
  a.qs = c->qt;
  a.B_k = c->B_k;
  a.rope_cs = c->rope_cs;
  a.part_o = c->part_o;
  a.part_ml = c->part_ml;
  a.Hq = d.n_q_heads; a.Hkv = d.n_kv_heads; a.d = d.head_dim; a.D = c->D;
  a.hist_len = c->hist_len; a.split_tokens = split_tokens; a.n_splits = n_splits;
  a.rope = d.rope_in_kernel; a.dtype = d.dtype;
  const size_t smem = decode_simt_smem(c);
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_decode_simt, optin_done);
  if (e != cudaSuccess) return e;
  dim3 grid(n_splits, d.batch);
  return launch_pdl(k_decode_simt, grid, dim3(256), smem, s, a, c->latent_kind);
}

cudaError_t launch_window(const lr_cache* c, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  const float* qd = d.rope_in_kernel ? c->qt : c->qt + (size_t)d.batch * d.n_q_heads * d.rank_k;
  const size_t smem = (size_t)(d.head_dim + c->win_len + 1) * sizeof(float);
  dim3 grid(d.n_q_heads, d.batch);
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_window, optin_done);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_window, grid, dim3(128), smem, s, c->win_k, c->win_v, qd, c->win_o, c->win_ml, d.n_q_heads, d.n_kv_heads,
                                   d.head_dim, c->D, c->win_slots, c->hist_len, c->win_len, d.dtype);
}

cudaError_t launch_merge(const lr_cache* c, int n_splits, void* out, float* lse, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  const bool win = c->win_slots > 0;
  const size_t smem = merge_smem(d, n_splits, c->esize);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  dim3 grid(d.n_kv_heads, d.batch);
  const float* wo = win ? c->win_o : nullptr;
  const float* wm = win ? c->win_ml : nullptr;
  if (d.dtype == LR_BF16) {
    static std::atomic<uint32_t> optin_done{0};
    cudaError_t e = smem_optin(k_merge<__nv_bfloat16>, optin_done);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_merge<__nv_bfloat16>, grid, dim3(kMergeThreads), smem, s, c->part_o, c->part_ml, wo, wm,
                      (const __nv_bfloat16*)c->B_v, (__nv_bfloat16*)out, lse, n_splits, d.n_q_heads, d.n_kv_heads,
                      d.head_dim, c->D, d.rank_v);
  }
  static std::atomic<uint32_t> optin_done32{0};
  cudaError_t e = smem_optin(k_merge<float>, optin_done32);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_merge<float>, grid, dim3(kMergeThreads), smem, s, c->part_o, c->part_ml, wo, wm,
                    (const float*)c->B_v, (float*)out, lse, n_splits, d.n_q_heads, d.n_kv_heads, d.head_dim, c->D,
                    d.rank_v);
}

static AppendArgs make_append_args(const lr_cache* c, const void* k, const void* v) {
  const lr_cache_desc& d = c->desc;
  AppendArgs a;
  const bool win = c->win_slots > 0;
  const bool fold = win && c->win_len == d.window;
  a.project = win ? (fold ? 1 : 0) : 1;
  if (win) {
    const int old_slot = c->hist_len % c->win_slots;
    const size_t es = c->esize;
    a.src_k = (const char*)c->win_k + (size_t)old_slot * c->D * es;
    a.src_v = (const char*)c->win_v + (size_t)old_slot * c->D * es;
    a.src_bstride = (long long)c->win_slots * c->D;
  } else {
    a.src_k = k; a.src_v = v; a.src_bstride = c->D;
  }
  a.A_k = c->A_k; a.A_v = c->A_v;
  a.Zk = c->z_k; a.Zv = c->z_v; a.codes_k = c->codes_k; a.codes_v = c->codes_v;
  a.params_k = c->params_k; a.params_v = c->params_v;
  a.rk = d.rank_k; a.rv = d.rank_v; a.Gk = c->G_k; a.Gv = c->G_v;
  a.chunks_k = (d.rank_k + 31) / 32; a.chunks_v = (d.rank_v + 31) / 32;
  a.cap = d.capacity; a.dst_slot = c->hist_len;
  a.new_k = win ? k : nullptr; a.new_v = win ? v : nullptr;
  a.win_k = c->win_k; a.win_v = c->win_v; a.slots = c->win_slots;
  a.new_slot = win ? (c->len % c->win_slots) : 0;
  a.B = d.batch; a.D = c->D; a.kind = c->latent_kind; a.dtype = d.dtype;
  return a;
}

static int append_ctas(const AppendArgs& a) {
  return (a.project ? a.chunks_k + a.chunks_v : 0) + (a.new_k ? 2 : 0);
}

static size_t append_smem(const lr_cache* c) {
  return (size_t)c->D * 32 * c->esize + (size_t)c->D * c->esize;
}

cudaError_t launch_append(lr_cache* c, const void* k, const void* v, cudaStream_t s) {
  const AppendArgs a = make_append_args(c, k, v);
  dim3 grid(append_ctas(a), c->desc.batch);
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_append, optin_done);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_append, grid, dim3(256), append_smem(c), s, a);
}

cudaError_t launch_step_pre(lr_cache* c, const void* k, const void* v, const void* q, bool tc, cudaStream_t s) {
  const AppendArgs aa = make_append_args(c, k, v);
  const QprojArgs qa = make_qproj_args(c, q, tc);
  const int x_app = append_ctas(aa);
  const int nq = qproj_chunks(c);
  dim3 grid(x_app + nq * c->desc.n_kv_heads, c->desc.batch);
  const size_t smem = std::max(append_smem(c), qproj_smem(c->desc, c->esize));
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_step_pre, optin_done);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_step_pre, grid, dim3(256), smem, s, aa, qa, x_app, nq);
}

cudaError_t launch_append_latent(lr_cache* c, const float* zk, const float* zv, int n, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  const int chunks_k = (d.rank_k + 31) / 32, chunks_v = (d.rank_v + 31) / 32;
  const long long pairs = (long long)n * (chunks_k + chunks_v);
  dim3 grid((unsigned)((pairs + 7) / 8), d.batch);
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_append_latent, optin_done);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_append_latent, grid, dim3(256), 0, s, zk, zv, n, d.batch, d.rank_k, d.rank_v, chunks_k, chunks_v, c->z_k,
                                       c->z_v, c->codes_k, c->codes_v, c->params_k, c->params_v, c->G_k,
                                       c->G_v, d.capacity, c->hist_len, c->latent_kind, d.dtype);
}

cudaError_t launch_sync_simt(lr_cache* c, const float* R, int which, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  const int r = which == 0 ? d.rank_k : d.rank_v;
  void* Z = which == 0 ? c->z_k : c->z_v;
  if (c->hist_len == 0) return cudaSuccess;
  const size_t smem = (size_t)kSyncRows * r * sizeof(float);
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_sync_simt, optin_done);
  if (e != cudaSuccess) return e;
  dim3 grid((c->hist_len + kSyncRows - 1) / kSyncRows, d.batch);
  return launch_pdl(k_sync_simt, grid, dim3(256), smem, s, Z, R, r, d.capacity, c->hist_len, d.dtype);
}
