// Device utilities shared by the CUDA-core kernels of the library: element access by
// runtime dtype, the int4 group quantiser (store path of the append), and cp.async
// staging of row blocks into shared memory.
#pragma once

#include "lr_internal.cuh"

namespace {

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
  if (kind == LK_INT4 && L.rank_major) {
    const uint32_t w = L.codes[i4v_code_index(row, L.G, i)];
    const float code = (float)((w >> (4 * i4v_nibble(row))) & 15u);
    const unsigned short* h = reinterpret_cast<const unsigned short*>(L.params);
    const long long si = i4v_scale_index(row, L.G, i >> 5);
    return fmaf(code, __half2float(__ushort_as_half(h[si])), __half2float(__ushort_as_half(h[si + 128])));
  }
  if (kind == LK_INT4) {
    const uint32_t w = L.codes[i4_code_index(row, L.G, i >> 5, (i >> 3) & 3)];
    const float code = (float)((w >> (4 * (i & 7))) & 15u);
    const uint32_t p = L.params[i4_param_index(row, L.G, i >> 5)];
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
struct QuantOut {
  uint32_t code;           // this lane's code (0 for padding lanes)
  unsigned short sh, zh;   // fp16 bits of the group's scale and zero
};
__device__ __forceinline__ QuantOut quant_group_codes(float x, bool valid) {
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
  QuantOut q;
  q.code = code;
  q.sh = __half_as_ushort(sh);
  q.zh = __half_as_ushort(zh);
  return q;
}

// Token-major packing of one quantised group (keys): 4 words and the {scale, zero} word.
__device__ __forceinline__ void quant_group_warp(float x, bool valid, uint32_t* words,
                                                 uint32_t* param) {
  const int lane = threadIdx.x & 31;
  const QuantOut q = quant_group_codes(x, valid);
  uint32_t v = q.code << (4 * (lane & 7));
  v |= __shfl_xor_sync(0xffffffffu, v, 1);
  v |= __shfl_xor_sync(0xffffffffu, v, 2);
  v |= __shfl_xor_sync(0xffffffffu, v, 4);
  if ((lane & 7) == 0) words[lane >> 3] = v;
  if (lane == 0) *param = (uint32_t)q.sh | ((uint32_t)q.zh << 16);
}

// Rank-major store of one quantised group of one value token (lane = rank 32 g + lane):
// each lane replaces its token's nibble in its rank's word.  The words are shared with
// seven other tokens, which other warps of the same launch may be writing, so the nibble
// is cleared and set with atomics (the two touch only this token's bits).
__device__ __forceinline__ void quant_group_warp_v(float x, bool valid, uint32_t* codes, uint32_t* params,
                                                   int G, int g, long long row) {
  const int lane = threadIdx.x & 31;
  const QuantOut q = quant_group_codes(x, valid);
  const int sh = 4 * i4v_nibble(row);
  uint32_t* w = codes + i4v_code_index(row, G, g * 32 + lane);
  atomicAnd(w, ~(15u << sh));
  if (q.code) atomicOr(w, q.code << sh);
  if (lane == 0) {
    unsigned short* h = reinterpret_cast<unsigned short*>(params);
    const long long si = i4v_scale_index(row, G, g);
    h[si] = q.sh;
    h[si + 128] = q.zh;
  }
}

// Store one warp's 32-coordinate chunk `ch` of a latent row (lane = coordinate); int4
// values (rank_major) take the rank-major block layout.
__device__ __forceinline__ void store_latent_chunk(float z, int ch, int r, int kind, int dtype,
                                                   void* Z, uint32_t* codes, uint32_t* params,
                                                   int G, long long row, bool rank_major = false) {
  const int lane = threadIdx.x & 31;
  const int i = ch * 32 + lane;
  const bool valid = i < r;
  if (kind == LK_INT4 && rank_major) {
    quant_group_warp_v(z, valid, codes, params, G, ch, row);
  } else if (kind == LK_INT4) {
    quant_group_warp(z, valid, codes + i4_code_index(row, G, ch, 0), params + i4_param_index(row, G, ch));
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
// ncol * es must be a multiple of 16 and the source 16-byte aligned.  Thread t copies
// vectors t, t + blockDim, ...; the (row, vector) position advances without division.
__device__ __forceinline__ void stage_rows(uint8_t* dst, int pitch, const void* src, long long ld, int es,
                                           int r0, int nr, long long col0, int ncol) {
  const int vpr = ncol * es / 16;                 // 16-byte vectors per row
  if (vpr <= 0 || nr <= 0) return;
  const int nt = blockDim.x;
  int rr = threadIdx.x / vpr, cc = threadIdx.x - (threadIdx.x / vpr) * vpr;
  const int rstep = nt / vpr, cstep = nt - (nt / vpr) * vpr;
  const size_t gpitch = (size_t)ld * es;
  const uint8_t* gbase = reinterpret_cast<const uint8_t*>(src) + ((size_t)r0 * ld + col0) * es;
  while (rr < nr) {
    cp_async16(dst + rr * pitch + cc * 16, gbase + rr * gpitch + cc * 16);
    rr += rstep;
    cc += cstep;
    if (cc >= vpr) {
      cc -= vpr;
      ++rr;
    }
  }
}

__device__ __forceinline__ float smem_elem(const uint8_t* p, int dtype) {
  if (dtype == LR_BF16) return __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(p));
  return *reinterpret_cast<const float*>(p);
}


}  // namespace
