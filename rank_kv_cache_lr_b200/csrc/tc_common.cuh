// Pieces shared by the tensor-core decode kernels (bf16 latents and int4 latents):
// bounded mbarrier waits with a per-CTA abort flag, the warp butterfly reduce-scatter,
// the optional per-CTA timeline, and the host-side tensor-map encoder.
#pragma once

#include "lr_internal.cuh"
#include "ptx.cuh"

#include <cudaTypedefs.h>

#include <mutex>

namespace tc {

constexpr int kTile = 128;                 // tokens per tile (the MMA's M for the scores)
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr int kSmemLimit = 232448;         // 227 KB opt-in per block
constexpr int kTraceSlots = LR_TRACE_SLOTS; // 0 start, 1 setup done, 2 query latents in,
                                           // 3+4i: key tile i consumed, 4+4i: scores of tile i read,
                                           // 5+4i: probabilities of tile i written,
                                           // 6+4i: value mix of tile i issued (i < 16), last: end
constexpr float kLazy = 8.0f;              // log2 of the allowed running-max growth before a rescale

// The wait limit of a launch: the cache's test setting (lr_cache_set_wait_limit), or
// kTimeoutNs when that is 0.
__host__ __device__ __forceinline__ uint64_t wait_limit(unsigned long long ns) { return ns ? ns : kTimeoutNs; }

// Wait for phase `parity` of `bar`.  Gives up when another thread of the CTA has
// aborted, or after `limit_ns`, in which case it records LR_ERR_TIMEOUT in the device
// error word and raises the CTA's abort flag.  Returns false when it gave up.
// (A phase already complete passes the first, non-blocking test.  After that every round of
// the loop checks the abort flag and the clock, then sleeps in the barrier until the phase
// completes or kSuspendNs pass: a waiting thread costs no issue slots that the working warps
// of its sub-partition need, and still sees an abort or its limit within kSuspendNs.)
constexpr uint32_t kSuspendNs = 20000;
__device__ __forceinline__ bool wait_b(uint64_t* bar, uint32_t parity, int* abort_flag, int* err,
                                       uint64_t limit_ns = kTimeoutNs) {
  if (ptx::mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  const uint32_t hint = limit_ns < kSuspendNs ? (uint32_t)limit_ns : kSuspendNs;
  for (;;) {
    if (*(volatile int*)abort_flag) return false;
    if (ptx::globaltimer() - t0 > limit_ns) {
      *(volatile int*)abort_flag = 1;
      atomicExch(err, (int)LR_ERR_TIMEOUT);
      return false;
    }
    if (ptx::mbar_try_wait_hint(bar, parity, hint)) return true;
  }
}

// Wait that ignores the abort flag (used to drain in-flight copies and MMAs after an
// abort); still bounded, always by kTimeoutNs (a short test limit applies only to the
// waits above).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = ptx::globaltimer();
  while (!ptx::mbar_try_wait_hint(bar, parity, kSuspendNs))
    if (ptx::globaltimer() - t0 > kTimeoutNs) return;
}

__device__ __forceinline__ void trace_stamp(unsigned long long* trace, int slot) {
  if (trace)
    trace[(((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * kTraceSlots + slot] =
        ptx::globaltimer();
}

// Unit u of the pipelined tile order, in which the scores of tile s+1 are computed before
// the value mix of tile s (each unit is the K or the V side of one tile):
//   u = 0 -> K(0); u = 2s - 1 -> K(s) for 1 <= s < n; u = 2s -> V(s - 1); the last unit,
//   u = 2n - 1, is V(n - 1).
__device__ __forceinline__ void unit_of(int u, int n, int* tile, bool* is_v) {
  if (u == 0) {
    *tile = 0;
    *is_v = false;
  } else if (u == 2 * n - 1) {
    *tile = n - 1;
    *is_v = true;
  } else if (u & 1) {
    *tile = (u + 1) >> 1;
    *is_v = false;
  } else {
    *tile = (u >> 1) - 1;
    *is_v = true;
  }
}

// Butterfly reduce-scatter over a warp: on return lane l holds op over all lanes of
// v[l] (v is destroyed).
template <bool kMax>
__device__ __forceinline__ float warp_reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int k = 0; k < w; ++k) {
      const float keep = up ? v[k + w] : v[k];
      const float send = up ? v[k] : v[k + w];
      const float got = __shfl_xor_sync(0xffffffffu, send, w);
      v[k] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  return v[0];
}

// ---- host ------------------------------------------------------------------------

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// A tiled map with 128-byte swizzle over 16-bit elements.
inline bool make_map(CUtensorMap* m, CUtensorMapDataType type, const void* ptr, int rank, const cuuint64_t* dims,
                     const cuuint64_t* strides, const cuuint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, type, rank, const_cast<void*>(ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace tc
