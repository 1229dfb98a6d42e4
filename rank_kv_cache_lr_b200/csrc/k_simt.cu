// CUDA-core kernels of the low-rank KV-cache path: the fp32 split-sequence decode
// (every configuration; the only path for fp32, int4 and keys-before-RoPE caches),
// the exact window, the latent bulk fill and the basis sync.
//
// Method: TraceKV abstract (latent KV storage with quantization, low-rank
// attention kernels) and iS-KV abstract/method section (exact recent window,
// folding, historical-coordinate synchronisation).  Attention is computed in
// rank space: q~_j = s log2(e) B_k,h(j) q_j, score_t = q~_j . z_t,
// o~_j = sum_t p_t z_v,t, o_j = o~_j B_v,h(j) / l — the exact identity
// q . (z B_h) = (B_h q) . z, so the result equals attention over the
// reconstructed keys and values.
#include "lr_internal.cuh"
#include "k_common.cuh"

#include <math.h>

#include <algorithm>

namespace {

constexpr int kTileSimt = 16;     // tokens per tile in the SIMT decode
constexpr int kSyncRows = 16;     // rows per CTA in the SIMT basis sync

// ---------------------------------------------------------------------------
// split-sequence decode on CUDA cores (fp32 arithmetic throughout)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_decode_simt(DecodeSimtArgs a, int kind) {
  extern __shared__ float sm[];
  span_begin(a.span);
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
  const int t_end = min(row_hist(a.row_len, b, a.hist_len), t_begin + a.split_tokens);
  for (int t0 = t_begin; t0 < t_end; t0 += kTileSimt) {
    const int n = min(kTileSimt, t_end - t0);
    const long long row0 = a.k.map.row(b, t0);   // a 16-token tile lies inside one page
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
        const float2 cs = a.rope_cs[rope_cs_index(t0 + t, i, half)];
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
  span_end(a.span);
}

// ---------------------------------------------------------------------------
// exact window (iS-KV): attention of each query head over its KV head's window tokens, as
// one more partial (in head space, relative to its own max).  One CTA per (KV head,
// sequence, query head of the group), 128 threads; the window rows come kWinTok tokens at a
// time with every row of the round in flight at once (16-byte cp.async into padded rows),
// then thread per token for the scores, a block-wide max and sum, and thread per column
// for the output.
// ---------------------------------------------------------------------------
constexpr int kWinTok = 128;
constexpr int kWinThreads = 128;

__host__ __device__ inline int window_pitch(int d, int es) { return d * es + 16; }   // staged row, bytes

size_t window_smem(int G, int d, int es) {
  (void)G;
  return (size_t)2 * d * sizeof(float) + (size_t)2 * kWinTok * window_pitch(d, es) +
         (size_t)(kWinTok + 16) * sizeof(float);
}

__device__ __forceinline__ void load8(const uint8_t* s, int dtype, float (&v)[8]) {
  if (dtype == LR_BF16) {
    const uint4 u = *reinterpret_cast<const uint4*>(s);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = __uint_as_float(w[k] << 16);
      v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
  } else {
    const float4 a = *reinterpret_cast<const float4*>(s);
    const float4 b = *reinterpret_cast<const float4*>(s + 16);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

template <typename T> __device__ __forceinline__ float win_elem(const uint8_t* p);
template <> __device__ __forceinline__ float win_elem<float>(const uint8_t* p) { return *reinterpret_cast<const float*>(p); }
template <> __device__ __forceinline__ float win_elem<__nv_bfloat16>(const uint8_t* p) {
  return __uint_as_float((uint32_t)(*reinterpret_cast<const uint16_t*>(p)) << 16);
}

// Window attention arguments.  Two modes:
//  - after the latent decode (lr_attn_decode): q_in is null; the query comes scaled from qd
//    (written by the query projection) and the newest token from its ring slot, both after
//    the dependency wait;
//  - right after the step's append and query projection (lr_decode_step): q_in, k_new, v_new
//    are the step's inputs; the newest window token is read from k_new / v_new (the append
//    copies those rows into its ring slot unchanged) and the query is scaled here as the
//    projection scales it, so the result is the same; hist_len / win_len are the counters
//    after the append.  Nothing here reads what that kernel writes, so the whole window runs
//    before the dependency wait, alongside it; the wait comes last, because the decode after
//    this kernel waits only for this grid, and through it for the append and projection.
// In both, the window tokens before the newest were written by earlier steps' kernels, which
// completed before the kernel just before this one passed its own wait (and this grid starts
// only after that kernel's CTAs have), so their rows are copied before this kernel's wait.
struct WinArgs {
  const void* win_k; const void* win_v; const float* qd;
  const void* q_in; const void* k_new; const void* v_new; float scale_log2;
  float* win_o; float* win_ml;
  int Hq, Hkv, d, D, slots, hist_len, win_len;
  unsigned long long* span;
};

template <typename T>
__global__ void __launch_bounds__(kWinThreads) k_window(const WinArgs a) {
  extern __shared__ __align__(16) uint8_t wsm_raw[];
  constexpr int es = sizeof(T);
  constexpr int dtype = es == 2 ? LR_BF16 : LR_F32;
  const int Hq = a.Hq, d = a.d, D = a.D, slots = a.slots, hist_len = a.hist_len, win_len = a.win_len;
  const int G = Hq / a.Hkv;
  const bool step = a.q_in != nullptr;
  const int pitch = window_pitch(d, es);
  float* q_s = reinterpret_cast<float*>(wsm_raw);          // [d]
  float* o_s = q_s + d;                                    // [d] (unused slot kept for alignment)
  uint8_t* k_s = reinterpret_cast<uint8_t*>(o_s + d);      // [kWinTok] rows of `pitch` bytes
  uint8_t* v_s = k_s + kWinTok * pitch;
  float* p_s = reinterpret_cast<float*>(v_s + kWinTok * pitch);   // [kWinTok]
  float* red = p_s + kWinTok;                              // [8]: warp maxima, then warp sums
  span_begin(a.span);
  pdl_trigger();   // the next kernel may start its own prologue
  const int h = blockIdx.x, b = blockIdx.y, u = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  constexpr int nw = kWinThreads / 32;
  const int j = h * G + u;                                 // query head
  const int vpr = d * es / 16;                             // 16-byte vectors per row
  // copy positions: with vpr dividing the block, a thread keeps one vector column and steps
  // over rows (no division per copy); otherwise (odd head dims) the general walk
  const bool fixed = (kWinThreads % vpr) == 0;
  const int rstep = fixed ? kWinThreads / vpr : 0;
  const uint8_t* gk = reinterpret_cast<const uint8_t*>(a.win_k) + ((long long)b * slots * D + (long long)h * d) * es;
  const uint8_t* gv = reinterpret_cast<const uint8_t*>(a.win_v) + ((long long)b * slots * D + (long long)h * d) * es;
  // rows [t0, t0 + n) of the window into staging rows 0.. (ring slot of window position t:
  // (hist_len + t) % slots), except position `skip`
  auto issue = [&](int t0, int n, int skip) {
    if (fixed) {
      const int v = tid % vpr;
      int t = tid / vpr;
      int slot = (hist_len + t0 + t) % slots;
      const int sstep = rstep % slots;
      for (; t < n; t += rstep) {
        if (t0 + t != skip) {
          const long long off = (long long)slot * D * es + v * 16;
          cp_async16(k_s + t * pitch + v * 16, gk + off);
          cp_async16(v_s + t * pitch + v * 16, gv + off);
        }
        slot += sstep;
        if (slot >= slots) slot -= slots;
      }
    } else {
      for (int idx = tid; idx < n * vpr; idx += kWinThreads) {
        const int t = idx / vpr, v = idx - (idx / vpr) * vpr;
        if (t0 + t == skip) continue;
        const long long off = (long long)((hist_len + t0 + t) % slots) * D * es + v * 16;
        cp_async16(k_s + t * pitch + v * 16, gk + off);
        cp_async16(v_s + t * pitch + v * 16, gv + off);
      }
    }
  };
  // the newest window token (position win_len - 1) into its staging row when it falls in the
  // round [t0, t0 + n): from the step's input rows, or from its ring slot
  const int newest = win_len - 1;
  auto issue_newest = [&](int t0, int n) {
    if (newest < t0 || newest >= t0 + n) return;
    const uint8_t* sk = step ? reinterpret_cast<const uint8_t*>(a.k_new) + ((long long)b * D + (long long)h * d) * es
                             : gk + (long long)((hist_len + newest) % slots) * D * es;
    const uint8_t* sv = step ? reinterpret_cast<const uint8_t*>(a.v_new) + ((long long)b * D + (long long)h * d) * es
                             : gv + (long long)((hist_len + newest) % slots) * D * es;
    const int t = newest - t0;
    for (int v = tid; v < vpr; v += kWinThreads) {
      cp_async16(k_s + t * pitch + v * 16, sk + v * 16);
      cp_async16(v_s + t * pitch + v * 16, sv + v * 16);
    }
  };
  const int n_first = min(kWinTok, win_len);
  issue(0, n_first, newest);
  if (!step) pdl_wait();
  if (step) {
    // the query, scaled as the query projection scales it (fp32 product of the stored value)
    const T* qb = static_cast<const T*>(a.q_in) + ((long long)b * Hq + j) * d;
    for (int e = tid; e < d; e += kWinThreads) q_s[e] = win_elem<T>(reinterpret_cast<const uint8_t*>(qb + e)) * a.scale_log2;
  } else {
    for (int v = tid; v < d / 4; v += kWinThreads)
      cp_async16(q_s + 4 * v, a.qd + ((long long)b * Hq + j) * d + 4 * v);
  }
  issue_newest(0, n_first);
  float m = -INFINITY, l = 0.f;
  float o = 0.f;                                           // output column tid (d <= 128 here: tid < d)
  float o2 = 0.f;                                          // column tid + 128 (d > 128)
  for (int t0 = 0; t0 < win_len; t0 += kWinTok) {
    const int n = min(kWinTok, win_len - t0);
    if (t0 > 0) {
      __syncthreads();   // the previous round's rows and weights are no longer read
      issue(t0, n, newest);
      issue_newest(t0, n);
    }
    cp_async_wait_all();
    __syncthreads();
    // score of token tid (kWinTok = blockDim: one token per thread)
    float sc = -INFINITY;
    if (tid < n) {
      const uint8_t* kr = k_s + tid * pitch;
      float s0 = 0.f, s1 = 0.f;
      for (int c = 0; c < d; c += 8) {
        float kf[8];
        load8(kr + c * es, dtype, kf);
        const float4 qa = *reinterpret_cast<const float4*>(q_s + c);
        const float4 qb = *reinterpret_cast<const float4*>(q_s + c + 4);
        s0 = fmaf(qa.x, kf[0], s0); s1 = fmaf(qa.y, kf[1], s1);
        s0 = fmaf(qa.z, kf[2], s0); s1 = fmaf(qa.w, kf[3], s1);
        s0 = fmaf(qb.x, kf[4], s0); s1 = fmaf(qb.y, kf[5], s1);
        s0 = fmaf(qb.z, kf[6], s0); s1 = fmaf(qb.w, kf[7], s1);
      }
      sc = s0 + s1;
    }
    // block max, weights, block sum (every thread keeps the same m and l)
    float mx = sc;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    mx = red[0];
#pragma unroll
    for (int w = 1; w < nw; ++w) mx = fmaxf(mx, red[w]);
    const float mn = fmaxf(m, mx);
    const float pv = tid < n ? exp2f(sc - mn) : 0.f;
    p_s[tid] = pv;
    float sum = pv;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    __syncthreads();   // red[] maxima read by everyone; p_s complete
    if (lane == 0) red[nw + warp] = sum;
    __syncthreads();
    float st = red[nw];
#pragma unroll
    for (int w = 1; w < nw; ++w) st += red[nw + w];
    const float alpha = m == -INFINITY ? 0.f : exp2f(m - mn);
    l = l * alpha + st;
    m = mn;
    // output columns tid (and tid + 128): tokens in order, four per step
    o *= alpha;
    o2 *= alpha;
    const uint8_t* vc = v_s + tid * es;
    const uint8_t* vc2 = v_s + (tid + kWinThreads) * es;
    if (tid < d) {
      int t = 0;
      for (; t + 4 <= n; t += 4) {
        const float4 p4 = *reinterpret_cast<const float4*>(p_s + t);
        o = fmaf(p4.x, win_elem<T>(vc + (t + 0) * pitch), o);
        o = fmaf(p4.y, win_elem<T>(vc + (t + 1) * pitch), o);
        o = fmaf(p4.z, win_elem<T>(vc + (t + 2) * pitch), o);
        o = fmaf(p4.w, win_elem<T>(vc + (t + 3) * pitch), o);
      }
      for (; t < n; ++t) o = fmaf(p_s[t], win_elem<T>(vc + t * pitch), o);
    }
    if (tid + kWinThreads < d)
      for (int t = 0; t < n; ++t) o2 = fmaf(p_s[t], win_elem<T>(vc2 + t * pitch), o2);
  }
  cp_async_wait_all();   // (no window tokens: the query copies still complete)
  if (step) pdl_wait();  // (the previous step's merge completed before the projection's wait)
  const long long ob = ((long long)b * Hq + j) * d;
  if (tid < d) a.win_o[ob + tid] = o;
  if (tid + kWinThreads < d) a.win_o[ob + tid + kWinThreads] = o2;
  if (tid == 0) {
    a.win_ml[((long long)b * Hq + j) * 2] = m;
    a.win_ml[((long long)b * Hq + j) * 2 + 1] = l;
  }
  span_end(a.span);
}

// bulk latent fill: one warp per (token, 32-coordinate chunk)
__global__ void __launch_bounds__(256) k_append_latent(const float* zk, const float* zv, int n, int B,
                                                       int rk, int rv, int chunks_k, int chunks_v,
                                                       void* Zk, void* Zv, uint32_t* codes_k,
                                                       uint32_t* codes_v, uint32_t* params_k,
                                                       uint32_t* params_v, int Gk, int Gv,
                                                       RowMap map, int slot0, int kind, int dtype) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long pi = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
  const int per_tok = chunks_k + chunks_v;
  const int b = blockIdx.y;
  if (pi >= (long long)n * per_tok) return;
  const int t = (int)(pi / per_tok), c = (int)(pi % per_tok);
  const bool is_k = c < chunks_k;
  if (!is_k && kind == LK_INT4) return;   // int4 values: k_append_latent_v
  const int ch = is_k ? c : c - chunks_k;
  const int r = is_k ? rk : rv;
  const float* src = is_k ? zk : zv;
  const int i = ch * 32 + lane;
  const float z = i < r ? src[((long long)b * n + t) * r + i] : 0.f;
  const long long row = map.row(b, slot0 + t);
  store_latent_chunk(z, ch, r, kind, dtype, is_k ? Zk : Zv, is_k ? codes_k : codes_v,
                     is_k ? params_k : params_v, is_k ? Gk : Gv, row);
}

// bulk fill of int4 values in the rank-major layout: one warp per (8-token word, group),
// lane = rank.  The warp quantises the word's tokens one after another and writes each
// rank's word once; a word the fill covers only in part (the ends of the range) keeps its
// other tokens' nibbles (cleared and set with atomics, which touch only the filled bits).
__global__ void __launch_bounds__(256) k_append_latent_v(const float* zv, int n, int rv, int Gv, uint32_t* codes,
                                                         uint32_t* params, RowMap map, int slot0) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int w0 = slot0 >> 3, nwords = ((slot0 + n - 1) >> 3) - w0 + 1;
  const long long pi = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
  if (pi >= (long long)nwords * Gv) return;
  const int wq = w0 + (int)(pi / Gv), g = (int)(pi % Gv);
  const int b = blockIdx.y;
  const int i = g * 32 + lane;
  const bool valid = i < rv;
  uint32_t word = 0, mask = 0;
  unsigned short* h = reinterpret_cast<unsigned short*>(params);
  for (int k = 0; k < 8; ++k) {
    const int t = wq * 8 + k;
    if (t < slot0 || t >= slot0 + n) continue;   // warp-uniform
    const float z = valid ? zv[((long long)b * n + (t - slot0)) * rv + i] : 0.f;
    const QuantOut q = quant_group_codes(z, valid);
    const long long row = map.row(b, t);
    const int sh = 4 * i4v_nibble(row);
    word |= q.code << sh;
    mask |= 15u << sh;
    if (lane == 0) {
      const long long si = i4v_scale_index(row, Gv, g);
      h[si] = q.sh;
      h[si + 128] = q.zh;
    }
  }
  uint32_t* w = codes + i4v_code_index(map.row(b, wq * 8), Gv, i);   // 8 tokens: one page
  if (mask == 0xFFFFFFFFu) {
    *w = word;
  } else {
    atomicAnd(w, ~mask);
    if (word) atomicOr(w, word);
  }
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
  L.map = row_map(c);
  L.rank_major = (!k && c->latent_kind == LK_INT4) ? 1 : 0;
  return L;
}

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------

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
  a.row_len = c->row_len;
  a.span = span_of(c->spans, SPAN_DECODE);
  const size_t smem = decode_simt_smem(c);
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_decode_simt, optin_done);
  if (e != cudaSuccess) return e;
  dim3 grid(n_splits, d.batch);
  return launch_pdl(k_decode_simt, grid, dim3(256), smem, s, a, c->latent_kind);
}

cudaError_t launch_window(const lr_cache* c, cudaStream_t s, const WindowStep* st) {
  const lr_cache_desc& d = c->desc;
  const size_t smem = window_smem(d.n_q_heads / d.n_kv_heads, d.head_dim, (int)c->esize);
  if (smem > 227 * 1024) return cudaErrorInvalidConfiguration;
  dim3 grid(d.n_kv_heads, d.batch, d.n_q_heads / d.n_kv_heads);
  WinArgs a;
  a.win_k = c->win_k;
  a.win_v = c->win_v;
  a.qd = d.rope_in_kernel ? c->qt : c->qt + (size_t)d.batch * d.n_q_heads * d.rank_k;
  a.q_in = st ? st->q : nullptr;
  a.k_new = st ? st->k : nullptr;
  a.v_new = st ? st->v : nullptr;
  a.scale_log2 = c->scale_log2;
  a.win_o = c->win_o;
  a.win_ml = c->win_ml;
  a.Hq = d.n_q_heads; a.Hkv = d.n_kv_heads; a.d = d.head_dim; a.D = c->D; a.slots = c->win_slots;
  a.hist_len = st ? st->hist_len : c->hist_len;
  a.win_len = st ? st->win_len : c->win_len;
  a.span = span_of(c->spans, SPAN_WINDOW);
  const bool bf = d.dtype == LR_BF16;
  using Kern = void (*)(const WinArgs);
  const Kern kern = bf ? k_window<__nv_bfloat16> : k_window<float>;
  static std::atomic<uint32_t> optin_done[2] = {0, 0};
  cudaError_t e = smem_optin(kern, optin_done[bf ? 1 : 0]);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, grid, dim3(kWinThreads), smem, s, a);
}

cudaError_t launch_append_latent(lr_cache* c, const float* zk, const float* zv, int n, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  const int chunks_k = (d.rank_k + 31) / 32, chunks_v = (d.rank_v + 31) / 32;
  const long long pairs = (long long)n * (chunks_k + chunks_v);
  dim3 grid((unsigned)((pairs + 7) / 8), d.batch);
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_append_latent, optin_done);
  if (e != cudaSuccess) return e;
  e = launch_pdl(k_append_latent, grid, dim3(256), 0, s, zk, zv, n, d.batch, d.rank_k, d.rank_v, chunks_k, chunks_v,
                 c->z_k, c->z_v, c->codes_k, c->codes_v, c->params_k, c->params_v, c->G_k, c->G_v, row_map(c),
                 c->hist_len, c->latent_kind, d.dtype);
  if (e != cudaSuccess || c->latent_kind != LK_INT4 || n == 0) return e;
  const int slot0 = c->hist_len;
  const long long units = (long long)(((slot0 + n - 1) >> 3) - (slot0 >> 3) + 1) * c->G_v;
  static std::atomic<uint32_t> optin_v{0};
  e = smem_optin(k_append_latent_v, optin_v);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_append_latent_v, dim3((unsigned)((units + 7) / 8), d.batch), dim3(256), 0, s, zv, n, d.rank_v,
                    c->G_v, c->codes_v, c->params_v, row_map(c), slot0);
}

cudaError_t launch_sync_simt(lr_cache* c, const float* R, int which, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  const int r = which == 0 ? d.rank_k : d.rank_v;
  void* Z = which == 0 ? c->z_k : c->z_v;
  // a paged pool is rotated whole, as one run of rows: every page once, whatever maps it
  const int rows = c->ptable ? c->n_pages * kPageTokens : c->hist_len;
  const int nseq = c->ptable ? 1 : d.batch;
  if (rows == 0) return cudaSuccess;
  const size_t smem = (size_t)kSyncRows * r * sizeof(float);
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_sync_simt, optin_done);
  if (e != cudaSuccess) return e;
  dim3 grid((rows + kSyncRows - 1) / kSyncRows, nseq);
  return launch_pdl(k_sync_simt, grid, dim3(256), smem, s, Z, R, r, (long long)(c->ptable ? rows : d.capacity), rows,
                    d.dtype);
}
