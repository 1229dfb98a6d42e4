// The small kernels around the decode: query projection (q~ = s log2(e) B_k,h q), the
// append of one token (z = k A, stored / quantised, window ring and fold), both fused
// in one grid for lr_decode_step, and the split merge with the output projection
// (o = o~ B_v,h / l).
//
// Method: TraceKV abstract (latent KV storage, low-rank attention kernels); iS-KV
// abstract and method section (exact window, folding).
//
// These kernels move little data (bases, one token, one query), so they are built for
// issue efficiency: the element type is a template parameter, shared-memory reads are
// 16-byte vectors, each thread computes a rank row for every query head of its group,
// and the bases — which no in-flight kernel writes — are staged with cp.async before
// the grid-dependency wait, overlapping the preceding kernel.
#include "lr_internal.cuh"
#include "k_common.cuh"

#include <algorithm>

namespace {

// ---- element helpers ---------------------------------------------------------------
template <typename T>
struct El;
template <>
struct El<__nv_bfloat16> {
  static __device__ __forceinline__ float ld(const void* p, size_t i) {
    return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  }
  static __device__ __forceinline__ void st(void* p, size_t i, float v) {
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  }
  // 8 consecutive elements from 16-byte aligned shared memory
  static __device__ __forceinline__ void lds8(const uint8_t* s, float (&v)[8]) {
    const uint4 u = *reinterpret_cast<const uint4*>(s);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = __uint_as_float(w[k] << 16);
      v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  }
  static __device__ __forceinline__ float lds1(const uint8_t* s) {
    return __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t*>(s)) << 16);
  }
  // 4 consecutive elements from 8-byte aligned shared memory
  static __device__ __forceinline__ void lds4(const uint8_t* s, float (&v)[4]) {
    const uint2 u = *reinterpret_cast<const uint2*>(s);
    v[0] = __uint_as_float(u.x << 16);
    v[1] = __uint_as_float(u.x & 0xFFFF0000u);
    v[2] = __uint_as_float(u.y << 16);
    v[3] = __uint_as_float(u.y & 0xFFFF0000u);
  }
};
template <>
struct El<float> {
  static __device__ __forceinline__ float ld(const void* p, size_t i) { return reinterpret_cast<const float*>(p)[i]; }
  static __device__ __forceinline__ void st(void* p, size_t i, float v) { reinterpret_cast<float*>(p)[i] = v; }
  static __device__ __forceinline__ void lds8(const uint8_t* s, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(s);
    const float4 b = *reinterpret_cast<const float4*>(s + 16);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ float lds1(const uint8_t* s) { return *reinterpret_cast<const float*>(s); }
  static __device__ __forceinline__ void lds4(const uint8_t* s, float (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(s);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  }
};

// ---- query projection -----------------------------------------------------------
// One CTA per (32 rank rows of B_k,h, KV head h, group of kRows sequences), 256 threads;
// thread = (rank row i, query head j of the group; heads beyond 8 in further passes), each
// for every sequence of the CTA: q~_j[i] = s log2(e) sum_c B_k[i][h d + c] q_j[c].  The rows
// of B_k are staged once for the CTA's sequences.
// qt16 (tensor-core path), bf16 latents: rows [b][j] and [b][32 + j] of a [B][64][r_k]
// bf16 array get hi = bf16(q~) and lo = bf16(q~ - hi), so that hi + lo carries q~ to ~16
// significant bits.  int4 latents: row [b][j] of a [B][32][r_k] fp16 array gets fp16(q~),
// each 8-rank run in the order 0,4,1,5,2,6,3,7 in which the int4 kernel expands codes.
constexpr int kQRowsCta = 32;
constexpr int kRows = 2;   // sequences per CTA of the small kernels

struct QprojArgs {
  const void* q; const void* Bk; float* qt; float* qd; void* qt16;
  int qt16_fp16;          // 1: fp16 rows in int4 run order; 0: bf16 hi / lo rows
  int Hq, Hkv, d, D, rk, B;
  float scale_log2;
  int want_latent;
  unsigned long long* span;   // timeline span, or null
};

template <typename T>
__device__ __forceinline__ int qproj_pitch(int d) { return d * (int)sizeof(T) + 16; }

template <typename T>
__device__ __forceinline__ void qproj_stage(const QprojArgs& a, int rchunk, int h, uint8_t* smem) {
  const int r0 = rchunk * kQRowsCta;
  const int nr = min(kQRowsCta, a.rk - r0);
  if (a.want_latent && nr > 0)
    stage_rows(smem, qproj_pitch<T>(a.d), a.Bk, a.D, sizeof(T), r0, nr, (long long)h * a.d, a.d);
}

template <typename T>
__device__ __forceinline__ void qproj_main(const QprojArgs& a, int rchunk, int h, int b0, int B, uint8_t* smem) {
  const int d = a.d, G = a.Hq / a.Hkv, j0 = h * G;
  const int pitch = qproj_pitch<T>(d);
  const int nb = min(kRows, B - b0);
  float* qs_all = reinterpret_cast<float*>(smem + (size_t)kQRowsCta * pitch);   // [nb][G][d]
  // the query rows of the group, 16-byte vectors, all of a thread's loads issued before its
  // first store (a store between dependent loads would serialise their latencies)
  {
    constexpr int kVec = 16 / sizeof(T);                // elements per vector
    constexpr int kPer = 4;                             // vectors in flight per thread
    const int nvec = nb * G * d / kVec;                 // G d is a multiple of 8
    for (int v0 = threadIdx.x; v0 < nvec; v0 += kPer * blockDim.x) {
      uint4 raw[kPer];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int v = v0 + k * blockDim.x;
        if (v < nvec) {
          const int e0 = v * kVec, bb = e0 / (G * d), e = e0 - bb * (G * d);
          raw[k] = __ldg(reinterpret_cast<const uint4*>(static_cast<const T*>(a.q) + ((size_t)(b0 + bb) * a.Hq + j0) * d + e));
        }
      }
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int v = v0 + k * blockDim.x;
        if (v < nvec) {
          const int e0 = v * kVec, bb = e0 / (G * d), e = e0 - bb * (G * d);
          float f[8];
          if constexpr (sizeof(T) == 2) {
            El<T>::lds8(reinterpret_cast<const uint8_t*>(&raw[k]), f);
          } else {
            f[0] = __uint_as_float(raw[k].x);
            f[1] = __uint_as_float(raw[k].y);
            f[2] = __uint_as_float(raw[k].z);
            f[3] = __uint_as_float(raw[k].w);
          }
#pragma unroll
          for (int m = 0; m < kVec; ++m) qs_all[e0 + m] = f[m];
          if (a.qd && rchunk == 0) {
            float* qd = a.qd + ((size_t)(b0 + bb) * a.Hq + j0) * d + e;
#pragma unroll
            for (int m = 0; m < kVec; ++m) qd[m] = f[m] * a.scale_log2;
          }
        }
      }
    }
  }
  if (!a.want_latent) return;
  cp_async_wait_all();
  __syncthreads();
  // thread = (rank row, query head); each 8-element run of the B_k row is read and converted
  // once for the CTA's sequences (the per-output sums keep their order)
  const int r0 = rchunk * kQRowsCta;
  const int nr = min(kQRowsCta, a.rk - r0);
  const int t = threadIdx.x & 31;            // rank row within the chunk
  const int i = r0 + t;
  const uint8_t* row = smem + (size_t)t * pitch;
  for (int u = threadIdx.x >> 5; u < G && t < nr; u += (int)(blockDim.x >> 5)) {
    float acc0[kRows], acc1[kRows];
#pragma unroll
    for (int bb = 0; bb < kRows; ++bb) acc0[bb] = acc1[bb] = 0.f;
    for (int c = 0; c < d; c += 8) {
      float bv[8];
      El<T>::lds8(row + (size_t)c * sizeof(T), bv);
#pragma unroll
      for (int bb = 0; bb < kRows; ++bb) {
        if (bb < nb) {
          const float* qj = qs_all + ((size_t)bb * G + u) * d;
          const float4 q0 = *reinterpret_cast<const float4*>(qj + c);
          const float4 q1 = *reinterpret_cast<const float4*>(qj + c + 4);
          acc0[bb] = fmaf(bv[0], q0.x, acc0[bb]);
          acc1[bb] = fmaf(bv[1], q0.y, acc1[bb]);
          acc0[bb] = fmaf(bv[2], q0.z, acc0[bb]);
          acc1[bb] = fmaf(bv[3], q0.w, acc1[bb]);
          acc0[bb] = fmaf(bv[4], q1.x, acc0[bb]);
          acc1[bb] = fmaf(bv[5], q1.y, acc1[bb]);
          acc0[bb] = fmaf(bv[6], q1.z, acc0[bb]);
          acc1[bb] = fmaf(bv[7], q1.w, acc1[bb]);
        }
      }
    }
    const int j = j0 + u;
#pragma unroll
    for (int bb = 0; bb < kRows; ++bb) {
      if (bb >= nb) continue;
      const int b = b0 + bb;
      const float v = (acc0[bb] + acc1[bb]) * a.scale_log2;
      a.qt[((size_t)b * a.Hq + j) * a.rk + i] = v;
      if (a.qt16 && a.qt16_fp16) {
        const int pos = (i & ~7) | ((i & 3) << 1) | ((i >> 2) & 1);
        reinterpret_cast<__half*>(a.qt16)[((size_t)b * 32 + j) * a.rk + pos] = __float2half_rn(v);
      } else if (a.qt16) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(v);
        const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
        __nv_bfloat16* q16 = reinterpret_cast<__nv_bfloat16*>(a.qt16);
        q16[((size_t)b * 64 + j) * a.rk + i] = hi;
        q16[((size_t)b * 64 + 32 + j) * a.rk + i] = lo;
      }
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_qproj(QprojArgs a) {
  extern __shared__ __align__(16) uint8_t qsm[];
  span_begin(a.span);
  qproj_stage<T>(a, blockIdx.x, blockIdx.y, qsm);      // bases: stable data
  pdl_wait();
  pdl_trigger();
  qproj_main<T>(a, blockIdx.x, blockIdx.y, blockIdx.z * kRows, a.B, qsm);
  span_end(a.span);
}

size_t qproj_smem(const lr_cache_desc& d, size_t es) {
  return (size_t)kQRowsCta * (d.head_dim * es + 16) +
         (size_t)kRows * (d.n_q_heads / d.n_kv_heads) * d.head_dim * sizeof(float);
}

// ---- append -----------------------------------------------------------------------
// One CTA per (32-coordinate chunk of K or V, group of kRows sequences):
// z_b[i] = sum_c x_b[c] A[c][i].  The chunk's columns of A ([D][32]) are staged before the
// grid-dependency wait (once for the CTA's sequences), the source rows after it.  The 8
// warps take fixed eighths of D, each A element read once for all the rows, and the
// partial sums are added in a fixed order, so the projection does not depend on the
// storage kind.
struct AppendArgs {
  const void* src_k; const void* src_v;   // rows to project (input or evicted ring rows)
  long long src_bstride;                  // elements between batch rows of src
  const void* A_k; const void* A_v;
  void* Zk; void* Zv; uint32_t* codes_k; uint32_t* codes_v; uint32_t* params_k; uint32_t* params_v;
  int rk, rv, Gk, Gv, chunks_k, chunks_v;
  RowMap map; int dst_slot; int project;
  const int32_t* row_pos;                 // per-row destination slots (device), or null: dst_slot
  int cap;                                // slots per sequence (a row_pos outside [0, cap) writes nothing)
  const void* new_k; const void* new_v;   // exact token for the ring, or null
  void* win_k; void* win_v; int slots; int new_slot;
  unsigned long long* span;   // timeline span, or null
  int B, D, kind, dtype;
};

template <typename T>
__device__ __forceinline__ void append_stage(const AppendArgs& a, int x, uint8_t* smem) {
  const int nproj = a.project ? (a.chunks_k + a.chunks_v) : 0;
  if (x >= nproj) return;
  const bool is_k = x < a.chunks_k;
  const int ch = is_k ? x : x - a.chunks_k;
  const int r = is_k ? a.rk : a.rv;
  const int ncol = min(32, r - ch * 32);         // 16 or 32 (ranks are multiples of 16)
  stage_rows(smem, 32 * sizeof(T), is_k ? a.A_k : a.A_v, r, sizeof(T), 0, a.D, (long long)ch * 32, ncol);
}

template <typename T>
__device__ __forceinline__ void append_main(const AppendArgs& a, int x, int b0, uint8_t* smem,
                                            float (*red)[kRows][32]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nproj = a.project ? (a.chunks_k + a.chunks_v) : 0;
  const int nb = min(kRows, a.B - b0);
  constexpr int es = sizeof(T);
  if (x < nproj) {
    const bool is_k = x < a.chunks_k;
    const int ch = is_k ? x : x - a.chunks_k;
    const int r = is_k ? a.rk : a.rv;
    const void* src = is_k ? a.src_k : a.src_v;
    const int ncol = min(32, r - ch * 32);
    const uint8_t* As = smem;                            // [D][32]
    uint8_t* xs = smem + (size_t)a.D * 32 * es;          // [nb][D]
    const int vrow = a.D * es / 16;
    for (int v = threadIdx.x; v < nb * vrow; v += blockDim.x) {
      const int bb = v / vrow, vv = v - bb * vrow;
      const uint8_t* g = reinterpret_cast<const uint8_t*>(src) + (size_t)(b0 + bb) * a.src_bstride * es;
      cp_async16(xs + (size_t)bb * a.D * es + vv * 16, g + vv * 16);
    }
    cp_async_wait_all();
    __syncthreads();
    const int per = (((a.D + 7) / 8) + 7) & ~7;          // multiple of 8 (vector reads of x)
    const int cb = warp * per, ce = min(a.D, cb + per);
    float z[kRows];
#pragma unroll
    for (int bb = 0; bb < kRows; ++bb) z[bb] = 0.f;
    if (lane < ncol) {
      for (int c = cb; c < ce; c += 8) {
        float av[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) av[e] = El<T>::lds1(As + ((size_t)(c + e) * 32 + lane) * es);
#pragma unroll
        for (int bb = 0; bb < kRows; ++bb) {
          if (bb < nb) {
            float xv[8];
            El<T>::lds8(xs + ((size_t)bb * a.D + c) * es, xv);
#pragma unroll
            for (int e = 0; e < 8; ++e) z[bb] = fmaf(xv[e], av[e], z[bb]);
          }
        }
      }
    }
#pragma unroll
    for (int bb = 0; bb < kRows; ++bb) red[warp][bb][lane] = z[bb];
    __syncthreads();
    // warp w stores row w (the quantiser works on the 32 lanes of one chunk)
    if (warp < nb) {
      float zz = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) zz += red[w][warp][lane];
      const int slot = a.row_pos ? __ldg(a.row_pos + b0 + warp) : a.dst_slot;
      if (slot >= 0 && slot < a.cap) {
        const long long row = a.map.row(b0 + warp, slot);
        store_latent_chunk(zz, ch, r, a.kind, a.dtype, is_k ? a.Zk : a.Zv, is_k ? a.codes_k : a.codes_v,
                           is_k ? a.params_k : a.params_v, is_k ? a.Gk : a.Gv, row, !is_k);
      }
    }
    return;
  }
  // ring write of the exact new token of each sequence
  const bool is_k = (x - nproj) == 0;
  const int vrow = a.D * es / 16;
  for (int v = threadIdx.x; v < nb * vrow; v += blockDim.x) {
    const int bb = v / vrow, vv = v - bb * vrow;
    const uint8_t* src = reinterpret_cast<const uint8_t*>(is_k ? a.new_k : a.new_v) + (size_t)(b0 + bb) * a.D * es;
    uint8_t* dst =
        reinterpret_cast<uint8_t*>(is_k ? a.win_k : a.win_v) + ((size_t)(b0 + bb) * a.slots + a.new_slot) * a.D * es;
    reinterpret_cast<uint4*>(dst)[vv] = reinterpret_cast<const uint4*>(src)[vv];
  }
}

template <typename T>
__global__ void __launch_bounds__(256) k_append(AppendArgs a) {
  extern __shared__ __align__(16) uint8_t asm_[];
  __shared__ float red[8][kRows][32];
  span_begin(a.span);
  append_stage<T>(a, blockIdx.x, asm_);                 // bases: stable data
  pdl_wait();
  pdl_trigger();
  append_main<T>(a, blockIdx.x, blockIdx.y * kRows, asm_, red);
  span_end(a.span);
}

// The independent first half of a decode step in one grid: CTAs [0, x_app) of each
// row are the append of the new token, the others the query projection.
template <typename T>
__global__ void __launch_bounds__(256) k_step_pre(AppendArgs aa, QprojArgs qa, int x_app, int nchunks_q) {
  extern __shared__ __align__(16) uint8_t psm[];
  __shared__ float red[8][kRows][32];
  const int x = blockIdx.x, b0 = blockIdx.y * kRows;
  const int qx = x - x_app;
  span_begin(aa.span);
  if (x < x_app) append_stage<T>(aa, x, psm);
  else qproj_stage<T>(qa, qx % nchunks_q, qx / nchunks_q, psm);
  pdl_wait();
  pdl_trigger();
  if (x < x_app) append_main<T>(aa, x, b0, psm, red);
  else qproj_main<T>(qa, qx % nchunks_q, qx / nchunks_q, b0, qa.B, psm);
  span_end(aa.span);
}

// ---- split merge and output projection ------------------------------------------
// A cluster of ncb = ceil(d / 32) CTAs per (KV head h, sequence b), 256 threads each; CTA p
// of the cluster owns output columns [32 p, +32) of the group's heads and ranks
// [p rp, +rp) of the merge.  Per pass of up to 8 query heads:
//   1. the split weights (log-sum-exp over the splits and the window partial; a warp per
//      head in turn) while each thread's first split loads are already in flight;
//   2. the merged rank-space outputs o~_j = sum_s w_s o~_s,j of the CTA's ranks (thread =
//      (head, 4 ranks), float4 loads of up to 16 splits in flight);
//   3. the parts are exchanged through distributed shared memory, so every CTA holds the
//      whole o~_j of the pass, and projected: o_j = o~_j B_v,h / l_j for its columns
//      (thread = column x eighth of the ranks, eighths added in a fixed order).
// The columns of B_v,h (no in-flight kernel writes them) are staged before the
// grid-dependency wait.  The exchange keeps every load of the partials issued once per
// cluster and the dependent global-load rounds at two (the (m, l) pairs and the partials,
// issued together).
constexpr int kMergeThreads = 256;
constexpr int kMergeHeads = 8;       // query heads per pass
constexpr int kMergeCols = 32;       // output columns per CTA
constexpr int kMergeLoads = 12;      // split loads in flight per thread

struct MergeArgs {
  const float* part_o; const float* part_ml; const float* win_o; const float* win_ml;
  const void* Bv; void* out; float* lse;
  int S, Hq, Hkv, d, D, rv;
  int ncb, rp;                // CTAs per cluster; ranks per CTA (multiple of 4)
  // partial (b, s) starts at head row (b * b_stride + s * s_stride) * Hq of part_o / part_ml:
  // the cache's [B][S][Hq] has b_stride = S, s_stride = 1; gathered shards [S][B][Hq] have
  // b_stride = 1, s_stride = B
  long long b_stride, s_stride;
  // rank-space output instead of the projection: the merged o~ (relative to the merged
  // max) [B][Hq][rv] and (m, l) [B][Hq][2]; or null
  float* rs_o; float* rs_ml;
  unsigned long long* span;   // timeline span, or null
};

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t cluster_addr(const void* smem_ptr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(r)
               : "r"((uint32_t)__cvta_generic_to_shared(smem_ptr)), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

struct MergeSmem {
  size_t bs, otp, otf, mls, wsm, red, hdr, total;
};
__host__ __device__ inline MergeSmem merge_layout(int rv, int rp, int S, int es) {
  MergeSmem L;
  size_t o = 0;
  L.bs = o;  o += ((size_t)rv * kMergeCols * es + 15) / 16 * 16;            // [rv][ncols] B_v columns
  L.otp = o; o += (size_t)kMergeHeads * (rp + 4) * 4;                        // [8][rp + 4] this part
  L.otf = o; o += (size_t)kMergeHeads * (rv + 4) * 4;                        // [8][rv + 4] whole o~
  L.mls = o; o += (size_t)kMergeHeads * S * 8;                               // [8][S] (m, l)
  L.wsm = o; o += ((size_t)kMergeHeads * S * 4 + 15) / 16 * 16;              // [8][S] weights
  L.red = o; o += (size_t)(kMergeThreads / 32) * kMergeHeads * kMergeCols * 4;   // [8][8][32]
  L.hdr = o; o += (size_t)kMergeHeads * 4 * 4;                               // [8]{m, 1/l, w_win, l}
  L.total = o;
  return L;
}

template <typename T>
__global__ void __launch_bounds__(kMergeThreads, 2) k_merge(MergeArgs a) {
  extern __shared__ __align__(16) uint8_t msm[];
  constexpr int es = sizeof(T);
  const int p = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int G = a.Hq / a.Hkv, S = a.S, rv = a.rv, rp = a.rp;
  const int c0 = p * kMergeCols, ncols = min(kMergeCols, a.d - c0);
  const int i0 = min(rv, p * rp), np = min(rv, i0 + rp) - i0;   // this CTA's ranks
  const MergeSmem L = merge_layout(rv, rp, S, es);
  uint8_t* bs = msm + L.bs;
  float* otp = reinterpret_cast<float*>(msm + L.otp);
  float* otf = reinterpret_cast<float*>(msm + L.otf);
  float2* mls = reinterpret_cast<float2*>(msm + L.mls);
  float* wsm = reinterpret_cast<float*>(msm + L.wsm);
  float* red = reinterpret_cast<float*>(msm + L.red);
  float* hdr = reinterpret_cast<float*>(msm + L.hdr);
  const bool project = a.rs_o == nullptr;
  span_begin(a.span);
  if (project) stage_rows(bs, ncols * es, a.Bv, a.D, es, 0, rv, (long long)h * a.d + c0, ncols);   // stable data
  pdl_wait();
  pdl_trigger();
  const size_t sstride = (size_t)a.s_stride * a.Hq * rv;   // floats between splits of one head row
  auto row_of = [&](int s) -> size_t { return (size_t)b * a.b_stride + (size_t)s * a.s_stride; };
  const int nq = np / 4;                                    // rank quads of this CTA
  bool staged = false;
  for (int jb = 0; jb < G; jb += kMergeHeads) {
    const int nh = min(kMergeHeads, G - jb);
    const int nitems = nh * nq;
    // 1. this thread's first item: its first kMergeLoads split loads go out now.  An item
    //    (head, 4 ranks) is shared by tpi adjacent threads (the CTA's threads spread over
    //    the items), thread `sub` of them taking splits sub, sub + tpi, ...
    const int tpi = nitems * 4 <= kMergeThreads ? 4 : (nitems * 2 <= kMergeThreads ? 2 : 1);
    const int sub = tid & (tpi - 1), it0 = tid / tpi, it_step = kMergeThreads / tpi;
    const int u0 = it0 < nitems ? it0 / nq : 0, q0 = it0 < nitems ? it0 - u0 * nq : 0;
    const float* src0 = a.part_o + ((size_t)b * a.b_stride * a.Hq + h * G + jb + u0) * rv + i0 + 4 * q0;
    // the (m, l) pairs first: the weights wait only for them, the partials keep coming
    float2 mlv[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int e = tid + k * kMergeThreads;
      if (e < nh * S) {
        const int u = e / S, s = e - (e / S) * S;
        mlv[k] = __ldg(reinterpret_cast<const float2*>(a.part_ml) + row_of(s) * a.Hq + h * G + jb + u);
      }
    }
    float4 v[kMergeLoads];
#pragma unroll
    for (int k = 0; k < kMergeLoads; ++k) {
      const int s = sub + k * tpi;
      v[k] = (it0 < nitems && s < S) ? __ldg(reinterpret_cast<const float4*>(src0 + (size_t)s * sstride))
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k)
      if (tid + k * kMergeThreads < nh * S) mls[tid + k * kMergeThreads] = mlv[k];
    for (int e = tid + 2 * kMergeThreads; e < nh * S; e += kMergeThreads) {
      const int u = e / S, s = e - (e / S) * S;
      mls[e] = __ldg(reinterpret_cast<const float2*>(a.part_ml) + row_of(s) * a.Hq + h * G + jb + u);
    }
    __syncthreads();
    for (int u = warp; u < nh; u += kMergeThreads / 32) {
      // split weights of head u (a split with no tokens has m = -inf: weight 0)
      const int j = h * G + jb + u;
      float m = -INFINITY;
      for (int s = lane; s < S; s += 32) m = fmaxf(m, mls[u * S + s].x);
      const float mw = a.win_ml ? a.win_ml[((size_t)b * a.Hq + j) * 2] : -INFINITY;
      m = fmaxf(m, mw);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      float l = 0.f;
      for (int s = lane; s < S; s += 32) {
        const float2 ml = mls[u * S + s];
        const float w = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - m);
        wsm[u * S + s] = w;
        l = fmaf(w, ml.y, l);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
      if (lane == 0) {
        float ww = 0.f;
        if (a.win_ml && mw != -INFINITY) {
          ww = exp2f(mw - m);
          l = fmaf(ww, a.win_ml[((size_t)b * a.Hq + j) * 2 + 1], l);
        }
        hdr[u * 4 + 0] = m;
        hdr[u * 4 + 1] = 1.0f / l;
        hdr[u * 4 + 2] = ww;
        hdr[u * 4 + 3] = l;
        if (a.lse && p == 0) a.lse[(size_t)b * a.Hq + j] = (m + log2f(l)) * LR_LN2;
      }
    }
    __syncthreads();
    // 2. merged o~ of this CTA's ranks: each thread sums its splits in a fixed order
    //    (zero-weight splits skipped: their outputs are not written), then the item's tpi
    //    threads add their sums (lanes sub ^ 1, then sub ^ 2)
    for (int it = it0; it < nitems; it += it_step) {
      const int u = it / nq, q = it - (it / nq) * nq;
      const float* src = a.part_o + ((size_t)b * a.b_stride * a.Hq + h * G + jb + u) * rv + i0 + 4 * q;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int s0 = 0; s0 < S; s0 += kMergeLoads * tpi) {
        if (it != it0 || s0 > 0) {
#pragma unroll
          for (int k = 0; k < kMergeLoads; ++k) {
            const int s = s0 + sub + k * tpi;
            v[k] = s < S ? __ldg(reinterpret_cast<const float4*>(src + (size_t)s * sstride))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
#pragma unroll
        for (int k = 0; k < kMergeLoads; ++k) {
          const int s = s0 + sub + k * tpi;
          const float w = s < S ? wsm[u * S + s] : 0.f;
          if (w != 0.f) {
            acc.x = fmaf(w, v[k].x, acc.x);
            acc.y = fmaf(w, v[k].y, acc.y);
            acc.z = fmaf(w, v[k].z, acc.z);
            acc.w = fmaf(w, v[k].w, acc.w);
          }
        }
      }
      if (tpi > 1) {
        const unsigned mask = ((1u << tpi) - 1u) << (lane & ~(tpi - 1));
        for (int o = 1; o < tpi; o <<= 1) {
          acc.x += __shfl_xor_sync(mask, acc.x, o);
          acc.y += __shfl_xor_sync(mask, acc.y, o);
          acc.z += __shfl_xor_sync(mask, acc.z, o);
          acc.w += __shfl_xor_sync(mask, acc.w, o);
        }
      }
      if (sub == 0) *reinterpret_cast<float4*>(otp + u * (rp + 4) + 4 * q) = acc;
    }
    if (!project) {
      // rank-space partial of this shard: the merged o~ (relative to m) and (m, l)
      __syncthreads();
      for (int it = tid; it < nitems; it += kMergeThreads) {
        const int u = it / nq, q = it - (it / nq) * nq;
        *reinterpret_cast<float4*>(a.rs_o + ((size_t)b * a.Hq + h * G + jb + u) * rv + i0 + 4 * q) =
            *reinterpret_cast<const float4*>(otp + u * (rp + 4) + 4 * q);
      }
      if (p == 0 && tid < nh) {
        a.rs_ml[((size_t)b * a.Hq + h * G + jb + tid) * 2] = hdr[tid * 4 + 0];
        a.rs_ml[((size_t)b * a.Hq + h * G + jb + tid) * 2 + 1] = hdr[tid * 4 + 3];
      }
      __syncthreads();
      continue;
    }
    // 3. every CTA gathers the whole o~ of the pass from the cluster's parts
    cluster_sync_all();
    {
      // items (part, head, 4 ranks), kGather remote loads in flight per thread before the
      // stores (a part's last quads may lie past rv: skipped)
      constexpr int kGather = 4;
      const int rq = rp / 4, per_part = nh * rq, total = a.ncb * per_part;
      for (int ib = tid; ib < total; ib += kGather * kMergeThreads) {
        float4 g[kGather];
        int dst[kGather];
#pragma unroll
        for (int k = 0; k < kGather; ++k) {
          const int it = ib + k * kMergeThreads;
          dst[k] = -1;
          if (it < total) {
            const int part = it / per_part, r = it - part * per_part;
            const int u = r / rq, q = r - (r / rq) * rq;
            const int i = part * rp + 4 * q;
            if (i < rv) {
              g[k] = ld_cluster_f4(cluster_addr(otp, (uint32_t)part) + (uint32_t)((u * (rp + 4) + 4 * q) * 4));
              dst[k] = u * (rv + 4) + i;
            }
          }
        }
#pragma unroll
        for (int k = 0; k < kGather; ++k)
          if (dst[k] >= 0) *reinterpret_cast<float4*>(otf + dst[k]) = g[k];
      }
    }
    if (!staged) {
      cp_async_wait_all();
      staged = true;
    }
    // the parts have been read everywhere before any CTA overwrites its own (next pass) or
    // exits; the gathered rows and the staged columns are visible to the whole CTA
    cluster_sync_all();
    // projection partial sums: column c, eighth rq of the ranks, every head of the pass
    {
      constexpr int kParts = kMergeThreads / 32;
      const int c = tid & 31, rq = tid >> 5;
      const int rql = ((rv + 4 * kParts - 1) / (4 * kParts)) * 4;   // ranks per part, multiple of 4
      const int r0 = min(rv, rq * rql), r1 = min(rv, r0 + rql);
      float acc[kMergeHeads];
#pragma unroll
      for (int u = 0; u < kMergeHeads; ++u) acc[u] = 0.f;
      if (c < ncols) {
        for (int i = r0; i < r1; i += 4) {
          float bv[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) bv[k] = El<T>::lds1(bs + ((size_t)(i + k) * ncols + c) * es);
#pragma unroll
          for (int u = 0; u < kMergeHeads; ++u) {
            if (u < nh) {
              const float4 o4 = *reinterpret_cast<const float4*>(otf + u * (rv + 4) + i);
              acc[u] = fmaf(o4.x, bv[0], acc[u]);
              acc[u] = fmaf(o4.y, bv[1], acc[u]);
              acc[u] = fmaf(o4.z, bv[2], acc[u]);
              acc[u] = fmaf(o4.w, bv[3], acc[u]);
            }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kMergeHeads; ++u) red[(rq * kMergeHeads + u) * kMergeCols + c] = acc[u];
    }
    __syncthreads();
    // parts added in order; window partial; normalisation; store
    for (int e = tid; e < nh * kMergeCols; e += kMergeThreads) {
      const int u = e / kMergeCols, cc = e % kMergeCols;
      if (cc >= ncols) continue;
      float o = red[u * kMergeCols + cc];
#pragma unroll
      for (int q = 1; q < kMergeThreads / 32; ++q) o += red[(q * kMergeHeads + u) * kMergeCols + cc];
      const int j = h * G + jb + u;
      const size_t oi = ((size_t)b * a.Hq + j) * a.d + c0 + cc;
      if (a.win_o) o = fmaf(hdr[u * 4 + 2], a.win_o[oi], o);
      El<T>::st(a.out, oi, o * hdr[u * 4 + 1]);
    }
    __syncthreads();
  }
  if (!staged) cp_async_wait_all();
  span_end(a.span);
}

// Ranks per CTA of the merge cluster: the rank range split evenly over the column blocks, in
// multiples of 4 (ranks are multiples of 16).
int merge_ncb(int d) { return (d + kMergeCols - 1) / kMergeCols; }
int merge_rp(int rv, int ncb) { return ((rv + 4 * ncb - 1) / (4 * ncb)) * 4; }

size_t merge_smem(const lr_cache_desc& d, int S, size_t es) {
  const int ncb = merge_ncb(d.head_dim);
  return merge_layout(d.rank_v, merge_rp(d.rank_v, ncb), S, (int)es).total;
}

// ---- argument construction ------------------------------------------------------------
QprojArgs make_qproj_args(const lr_cache* c, const void* q, bool tc) {
  const lr_cache_desc& d = c->desc;
  const bool rope = d.rope_in_kernel != 0;
  QprojArgs a;
  a.q = q;
  a.Bk = c->B_k;
  a.qt = c->qt;
  a.qd = (rope || c->win_slots) ? (rope ? c->qt : c->qt + (size_t)d.batch * d.n_q_heads * d.rank_k) : nullptr;
  a.qt16 = tc ? c->qt16 : nullptr;
  a.qt16_fp16 = c->latent_kind == LK_INT4 ? 1 : 0;
  a.Hq = d.n_q_heads; a.Hkv = d.n_kv_heads; a.d = d.head_dim; a.D = c->D; a.rk = d.rank_k; a.B = d.batch;
  a.scale_log2 = c->scale_log2;
  a.want_latent = rope ? 0 : 1;
  a.span = span_of(c->spans, SPAN_PRE);
  return a;
}

int qproj_chunks(const lr_cache* c) {
  return c->desc.rope_in_kernel ? 1 : (c->desc.rank_k + kQRowsCta - 1) / kQRowsCta;
}

AppendArgs make_append_args(const lr_cache* c, const void* k, const void* v) {
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
  a.map = row_map(c); a.dst_slot = c->hist_len;
  a.row_pos = nullptr; a.cap = d.capacity;
  a.new_k = win ? k : nullptr; a.new_v = win ? v : nullptr;
  a.win_k = c->win_k; a.win_v = c->win_v; a.slots = c->win_slots;
  a.new_slot = win ? (c->len % c->win_slots) : 0;
  a.B = d.batch; a.D = c->D; a.kind = c->latent_kind; a.dtype = d.dtype;
  a.span = span_of(c->spans, SPAN_PRE);
  return a;
}

int append_ctas(const AppendArgs& a) { return (a.project ? a.chunks_k + a.chunks_v : 0) + (a.new_k ? 2 : 0); }

size_t append_smem(const lr_cache* c) { return (size_t)c->D * 32 * c->esize + (size_t)kRows * c->D * c->esize; }

template <typename T>
cudaError_t qproj_t(const lr_cache* c, const void* q, cudaStream_t s, bool tc, bool pdl = true) {
  const lr_cache_desc& d = c->desc;
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_qproj<T>, optin_done);
  if (e != cudaSuccess) return e;
  const dim3 grid(qproj_chunks(c), d.n_kv_heads, (d.batch + kRows - 1) / kRows);
  if (!pdl) return launch_serial(k_qproj<T>, grid, dim3(256), qproj_smem(d, sizeof(T)), s, make_qproj_args(c, q, tc));
  return launch_pdl(k_qproj<T>, grid, dim3(256), qproj_smem(d, sizeof(T)), s, make_qproj_args(c, q, tc));
}

template <typename T>
cudaError_t merge_t(const lr_cache* c, int n_splits, void* out, float* lse, cudaStream_t s,
                    const MergeSource* src = nullptr) {
  const lr_cache_desc& d = c->desc;
  const bool win = c->win_slots > 0 && !src;
  const size_t smem = merge_smem(d, n_splits, sizeof(T));
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_merge<T>, optin_done);
  if (e != cudaSuccess) return e;
  MergeArgs a;
  a.part_o = src ? src->part_o : c->part_o;
  a.part_ml = src ? src->part_ml : c->part_ml;
  a.b_stride = src ? src->b_stride : n_splits;
  a.s_stride = src ? src->s_stride : 1;
  a.rs_o = src ? src->rs_o : nullptr;
  a.rs_ml = src ? src->rs_ml : nullptr;
  a.win_o = win ? c->win_o : nullptr;
  a.win_ml = win ? c->win_ml : nullptr;
  a.Bv = c->B_v;
  a.out = out;
  a.lse = lse;
  a.S = n_splits;
  a.Hq = d.n_q_heads;
  a.Hkv = d.n_kv_heads;
  a.d = d.head_dim;
  a.D = c->D;
  a.rv = d.rank_v;
  a.ncb = merge_ncb(d.head_dim);
  a.rp = merge_rp(d.rank_v, a.ncb);
  a.span = span_of(c->spans, SPAN_MERGE);
  return launch_pdl_cluster(k_merge<T>, dim3(a.ncb, d.n_kv_heads, d.batch), dim3(kMergeThreads), a.ncb, smem, s, a);
}

template <typename T>
cudaError_t append_t(lr_cache* c, const void* k, const void* v, cudaStream_t s, long long bstride,
                     const int32_t* row_pos) {
  AppendArgs a = make_append_args(c, k, v);
  if (bstride && !c->win_slots) a.src_bstride = bstride;
  if (!c->win_slots) a.row_pos = row_pos;
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_append<T>, optin_done);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_append<T>, dim3(append_ctas(a), (c->desc.batch + kRows - 1) / kRows), dim3(256), append_smem(c), s, a);
}

template <typename T>
cudaError_t step_pre_t(lr_cache* c, const void* k, const void* v, const void* q, bool tc, cudaStream_t s) {
  const AppendArgs aa = make_append_args(c, k, v);
  const QprojArgs qa = make_qproj_args(c, q, tc);
  const int x_app = append_ctas(aa);
  const int nq = qproj_chunks(c);
  const size_t smem = std::max(append_smem(c), qproj_smem(c->desc, sizeof(T)));
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_step_pre<T>, optin_done);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_step_pre<T>, dim3(x_app + nq * c->desc.n_kv_heads, (c->desc.batch + kRows - 1) / kRows), dim3(256),
                    smem, s, aa, qa,
                    x_app, nq);
}

}  // namespace

cudaError_t launch_qproj(const lr_cache* c, const void* q, cudaStream_t s, bool pdl) {
  return c->desc.dtype == LR_BF16 ? qproj_t<__nv_bfloat16>(c, q, s, false, pdl)
                                  : qproj_t<float>(c, q, s, false, pdl);
}

cudaError_t launch_qproj_tc(const lr_cache* c, const void* q, cudaStream_t s) {
  // keys before RoPE: the decode reads the scaled fp32 queries, no 16-bit latents
  if (c->desc.dtype != LR_BF16 || (!c->qt16 && !c->desc.rope_in_kernel)) return cudaErrorNotSupported;
  return qproj_t<__nv_bfloat16>(c, q, s, true);
}

cudaError_t launch_merge(const lr_cache* c, int n_splits, void* out, float* lse, cudaStream_t s,
                         const MergeSource* src) {
  return c->desc.dtype == LR_BF16 ? merge_t<__nv_bfloat16>(c, n_splits, out, lse, s, src)
                                  : merge_t<float>(c, n_splits, out, lse, s, src);
}

cudaError_t launch_append(lr_cache* c, const void* k, const void* v, cudaStream_t s, long long bstride,
                          const int32_t* row_pos) {
  return c->desc.dtype == LR_BF16 ? append_t<__nv_bfloat16>(c, k, v, s, bstride, row_pos)
                                  : append_t<float>(c, k, v, s, bstride, row_pos);
}

cudaError_t launch_step_pre(lr_cache* c, const void* k, const void* v, const void* q, bool tc, cudaStream_t s) {
  if (tc && c->desc.dtype != LR_BF16) return cudaErrorNotSupported;
  return c->desc.dtype == LR_BF16 ? step_pre_t<__nv_bfloat16>(c, k, v, q, tc, s)
                                  : step_pre_t<float>(c, k, v, q, false, s);
}
