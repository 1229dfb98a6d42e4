// Basis synchronisation on tensor cores: Z_hist <- Z_hist R for the key and the value
// latents (iS-KV abstract and method section: stored historical coordinates are
// synchronised when the basis changes).
//
// Z is bf16 [B][cap][r] (r <= 256), R fp32 [r][r].  R is first split into two bf16
// halves, R = R_hi + R_lo (R_lo = bf16(R - R_hi)), so Z R_hi + Z R_lo carries R to ~16
// significant bits and the only material rounding is the final bf16 store, as on the
// CUDA-core path.  The product is a dense contraction per 128-token tile:
//   D[t, n] = sum_k Z[t, k] R[k, n]     M = 128 tokens, N = r, K = r (16 per MMA, hi and lo)
// with the tile (A, K-major, 128-byte swizzle) loaded by TMA into one of two tile buffers,
// R streamed through a ring of three slots of 32 k-rows (B, MN-major, hi then lo), D in one
// of two TMEM accumulators, and an epilogue that rounds D to bf16 into the tile's own buffer
// (same swizzle) and stores it back in place with a TMA store.  Each CTA loops over (side,
// sequence, tile) units; with two tile buffers and two accumulators the load of unit i + 1
// and the store of unit i - 1 overlap the MMAs of unit i.
//
// Roles (224 threads): warp 0 loads the tiles, warp 6 streams R (one thread each), warp 1
// owns TMEM and issues the MMAs (the whole warp runs the loop, one elected lane issues),
// warps 2..5 run the epilogue (thread = token row = TMEM lane).  Every wait is bounded; on
// timeout the kernel records LR_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and
// returns.
#include "tc_common.cuh"

#include <algorithm>

namespace {

using tc::drain_wait;
using tc::kSmemLimit;
using tc::kTile;

constexpr int kThreads = 224;
constexpr int kSubBytes = 128 * 128;      // Z tile: 128 tokens x 64 ranks x 2 B
constexpr int kRRows = 32;                // k-rows of R per ring slot
constexpr int kRBox = kRRows * 128;       // R box: 32 k-rows x 64 n-columns x 2 B
constexpr int kRSlots = 3;
constexpr int kAccCols = 256;             // TMEM columns per accumulator (N = r <= 256)
constexpr int kAuxBytes = 1024;

struct SyncParams {
  unsigned long long wait_ns;   // bounded-wait limit (0: the default)
  int r, kb, nch, B, ntile, units, hist;
  uint32_t z_bytes, r_half, r_slot;   // tile bytes; bytes of one of hi/lo per chunk; slot bytes
  int* err;
};

// Barriers (arrival count; who arrives -> who waits); a barrier used by every other unit
// (index i & 1) is waited for unit i with parity (i >> 1) & 1, a ring slot used for the
// n-th time with parity n & 1.
//   z_full[2]         1 + tx   tile loader's TMA boxes of one Z tile -> MMA issuer
//   z_empty[2]        1        the storing thread, once its TMA store has read the tile -> tile loader
//   r_full[kRSlots]   1 + tx   R streamer's chunk (hi and lo rows) -> MMA issuer
//   r_empty[kRSlots]  1        MMA commit -> R streamer
//   d_full[2]         1        MMA commit of a tile's product -> epilogue warps
//   d_empty[2]        4        epilogue warps (product read from TMEM) -> MMA issuer
struct Aux {
  uint64_t z_full[2], z_empty[2], d_full[2], d_empty[2];
  uint64_t r_full[kRSlots], r_empty[kRSlots];
  uint64_t fin;                 // one MMA commit after the last unit: every MMA has completed
  uint32_t tmem_base;
  int abort_flag;
  unsigned long long wait_ns;   // this launch's wait limit
};
static_assert(sizeof(Aux) <= kAuxBytes, "aux block");

struct SyncState {
  CUtensorMap zk, zv, rk, rv;
  __nv_bfloat16* rbuf = nullptr;   // [2 sides][2r rows: hi then lo][r] bf16
  int r = 0;
};

__device__ __forceinline__ bool wait_b(uint64_t* bar, uint32_t parity, Aux* aux, int* err) {
  return tc::wait_b(bar, parity, &aux->abort_flag, err, aux->wait_ns);
}
// The same, by a whole warp with one verdict for all its lanes.
__device__ __forceinline__ bool wait_w(uint64_t* bar, uint32_t parity, Aux* aux, int* err) {
  return __all_sync(0xffffffffu, wait_b(bar, parity, aux, err));
}

// unit u -> (side, sequence, first token)
__device__ __forceinline__ void unit_of(const SyncParams& p, int u, int* side, int* b, int* t0) {
  const int per_side = p.B * p.ntile;
  *side = u / per_side;
  const int rem = u - *side * per_side;
  *b = rem / p.ntile;
  *t0 = (rem - *b * p.ntile) * kTile;
}
// Shared memory: [aux 1 KB][2 Z tiles of kb x 16 KB][R ring kRSlots x (hi | lo) x kb x 4 KB]
__global__ void __launch_bounds__(kThreads, 1)
    k_sync_tc(const __grid_constant__ CUtensorMap tm_zk, const __grid_constant__ CUtensorMap tm_zv,
              const __grid_constant__ CUtensorMap tm_rk, const __grid_constant__ CUtensorMap tm_rv,
              const SyncParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (ptx::smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicExch(p.err, (int)LR_ERR_UNSUPPORTED);
    return;
  }
  Aux* aux = reinterpret_cast<Aux*>(smem_raw);
  uint8_t* z_s = smem_raw + kAuxBytes;          // tile buffer j at z_s + j * z_bytes
  uint8_t* r_s = z_s + 2 * p.z_bytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int my_units = p.units > (int)blockIdx.x ? (p.units - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    for (int j = 0; j < 2; ++j) {
      ptx::mbar_init(&aux->z_full[j], 1);
      ptx::mbar_init(&aux->z_empty[j], 1);
      ptx::mbar_init(&aux->d_full[j], 1);
      ptx::mbar_init(&aux->d_empty[j], 4);   // one arrival per epilogue warp
    }
    ptx::mbar_init(&aux->fin, 1);
    for (int k = 0; k < kRSlots; ++k) {
      ptx::mbar_init(&aux->r_full[k], 1);
      ptx::mbar_init(&aux->r_empty[k], 1);
    }
    aux->abort_flag = 0;
    aux->wait_ns = tc::wait_limit(p.wait_ns);
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_zk);
    ptx::prefetch_tmap(&tm_zv);
  }
  if (warp == 6 && lane == 0) {
    ptx::prefetch_tmap(&tm_rk);
    ptx::prefetch_tmap(&tm_rv);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&aux->tmem_base, 2 * kAccCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = aux->tmem_base;
  pdl_wait();      // the latents and R were written by earlier work on the stream
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------- tile loader
    if (lane == 0 && my_units > 0) {
      int z_issued = 0;
      for (int i = 0; i < my_units; ++i) {
        const int j = i & 1;
        int side, b, t0;
        unit_of(p, (int)blockIdx.x + i * (int)gridDim.x, &side, &b, &t0);
        // the buffer's previous tile (unit i - 2) has been read by its store
        if (i >= 2 && !wait_b(&aux->z_empty[j], ((i >> 1) - 1) & 1, aux, p.err)) break;
        uint8_t* dst = z_s + j * p.z_bytes;
        ptx::mbar_arrive_expect_tx(&aux->z_full[j], p.z_bytes);
        for (int sb = 0; sb < p.kb; ++sb)
          ptx::tma_load_3d(dst + sb * kSubBytes, side ? &tm_zv : &tm_zk, &aux->z_full[j], sb * 64, t0, b);
        z_issued = i + 1;
      }
      // Every copy this thread issued has landed before the CTA can exit, whether or not
      // the CTA aborted (an abort in another role may come after this loop); the last
      // phase of each buffer's barrier is its latest, and in a normal run it has been
      // waited already.
      for (int i = std::max(0, z_issued - 2); i < z_issued; ++i) drain_wait(&aux->z_full[i & 1], (i >> 1) & 1);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------- R streamer
    if (lane == 0 && my_units > 0) {
      int rpos = 0, r_issued = 0;
      bool ok = true;
      for (int i = 0; i < my_units && ok; ++i) {
        int side, b, t0;
        unit_of(p, (int)blockIdx.x + i * (int)gridDim.x, &side, &b, &t0);
        for (int kc = 0; kc < p.nch; ++kc, ++rpos) {
          const int slot = rpos % kRSlots, round = rpos / kRSlots;
          if (round > 0 && !(ok = wait_b(&aux->r_empty[slot], (round - 1) & 1, aux, p.err))) break;
          uint8_t* dst = r_s + slot * p.r_slot;
          ptx::mbar_arrive_expect_tx(&aux->r_full[slot], p.r_slot);
          for (int hl = 0; hl < 2; ++hl)
            for (int nb = 0; nb < p.kb; ++nb)
              ptx::tma_load_2d(dst + hl * p.r_half + nb * kRBox, side ? &tm_rv : &tm_rk, &aux->r_full[slot],
                               nb * 64, hl * p.r + kc * kRRows);
          r_issued = rpos + 1;
        }
      }
      for (int k = std::max(0, r_issued - kRSlots); k < r_issued; ++k)
        drain_wait(&aux->r_full[k % kRSlots], (k / kRSlots) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    if (my_units > 0) {   // the whole warp runs the loop; an elected lane issues
      const uint32_t id = ptx::idesc_f16(1, 0, 1, 128, (uint32_t)p.r);   // bf16; A K-major, B MN-major
      const uint64_t adesc0 = ptx::smem_desc(ptx::smem_u32(z_s), 16, 1024, 2);
      const uint64_t bdesc0 = ptx::smem_desc(ptx::smem_u32(r_s), kRBox, 1024, 2);
      bool ok = true;
      int rpos = 0;
      for (int i = 0; i < my_units && ok; ++i) {
        const int j = i & 1;
        if (!(ok = wait_w(&aux->z_full[j], (i >> 1) & 1, aux, p.err))) break;
        if (i >= 2 && !(ok = wait_w(&aux->d_empty[j], ((i >> 1) - 1) & 1, aux, p.err))) break;
        ptx::tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)(j * kAccCols);
        const uint64_t az = adesc0 + (uint64_t)((j * p.z_bytes) >> 4);
        for (int kc = 0; kc < p.nch && ok; ++kc, ++rpos) {
          const int slot = rpos % kRSlots;
          if (!(ok = wait_w(&aux->r_full[slot], (rpos / kRSlots) & 1, aux, p.err))) break;
          ptx::tc_fence_after();
          const uint64_t bs = bdesc0 + (uint64_t)((slot * p.r_slot) >> 4);
          const int nk = std::min(kRRows / 16, (p.r - kc * kRRows) >> 4);
          // k-rows kc*32 .. of the tile: 64-rank sub-tile kc / 2, byte 64 (kc & 1) of its rows
          const uint32_t abase = (uint32_t)((kc >> 1) * kSubBytes + (kc & 1) * 64);
          for (int kk = 0; kk < nk; ++kk) {
            const uint64_t ad = az + (uint64_t)((abase + kk * 32) >> 4);
            const uint64_t bd = bs + (uint64_t)((kk * 2048) >> 4);   // 16 k-rows of 128 B
            ptx::mma_f16_elect(acc, ad, bd, id, (kc | kk) ? 1u : 0u);
            ptx::mma_f16_elect(acc, ad, bd + (uint64_t)(p.r_half >> 4), id, 1u);
          }
          ptx::mma_commit_elect(&aux->r_empty[slot]);
        }
        if (!ok) break;
        ptx::mma_commit_elect(&aux->d_full[j]);
      }
      // every MMA issued so far completes before TMEM is freed, even if the epilogue aborted
      ptx::mma_commit_elect(&aux->fin);
      drain_wait(&aux->fin, 0);
    }
    __syncwarp();
  } else if (my_units > 0) {
    // ------------------------------------------------------------- epilogue
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const int sw = row & 7;
    bool ok = true;
    for (int i = 0; i < my_units; ++i) {
      const int j = i & 1;
      ok = ptx::named_bar_and(1, 128, wait_b(&aux->d_full[j], (i >> 1) & 1, aux, p.err));
      if (!ok) break;
      ptx::tc_fence_after();
      // D row -> bf16 into the tile's own buffer (the MMAs that read it have completed)
      uint8_t* zt = z_s + j * p.z_bytes;
      const uint32_t zrow = ptx::smem_u32(zt) + row * 128;
      const uint32_t acc = tmem + lane_off + (uint32_t)(j * kAccCols);
      for (int c0 = 0; c0 < p.r; c0 += 32) {
        uint32_t v[32];
        ptx::tmem_ld32(acc + c0, v);
        ptx::tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
          w[e] = *reinterpret_cast<const uint32_t*>(&h);
        }
        const uint32_t sub = zrow + (c0 >> 6) * kSubBytes;
        const int ch0 = (c0 & 63) >> 3;   // first 16-byte column of these 32 values
#pragma unroll
        for (int q = 0; q < 4; ++q)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(sub + (((ch0 + q) ^ sw) << 4)),
                       "r"(w[4 * q]), "r"(w[4 * q + 1]), "r"(w[4 * q + 2]), "r"(w[4 * q + 3])
                       : "memory");
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&aux->d_empty[j]);   // this accumulator may be overwritten
      ptx::fence_proxy_async_smem();
      ptx::named_bar_sync(1, 128);
      if (threadIdx.x == 64) {
        int side, b, t0;
        unit_of(p, (int)blockIdx.x + i * (int)gridDim.x, &side, &b, &t0);
        for (int sb = 0; sb < p.kb; ++sb) ptx::tma_store_3d(side ? &tm_zv : &tm_zk, zt + sb * kSubBytes, sb * 64, t0, b);
        ptx::bulk_commit_group();
        ptx::bulk_wait_group_read0();   // the tile buffer may be refilled
        ptx::mbar_arrive(&aux->z_empty[j]);
      }
    }
    if (threadIdx.x == 64) ptx::bulk_wait_group0();   // stores complete before the kernel ends
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 2 * kAccCols);
  }
}

// R (fp32, caller-owned) -> bf16 hi and lo halves, rows [k] then [r + k] of one side.
__global__ void k_sync_prep(const float* R, __nv_bfloat16* out, int r) {
  const int n = r * r;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float x = R[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
    out[i] = hi;
    out[n + i] = __float2bfloat16_rn(x - __bfloat162float(hi));
  }
}

bool map_bf16(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
              const cuuint32_t* box) {
  return tc::make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, rank, dims, strides, box);
}

size_t sync_smem(int r) {
  const int kb = (r + 63) / 64;
  return (size_t)kAuxBytes + 2 * (size_t)kb * kSubBytes + kRSlots * (2 * (size_t)kb * kRBox);
}

}  // namespace

bool sync_tc_supported(const lr_cache_desc* d) {
  return d->dtype == LR_BF16 && d->quant_bits == 0 && d->rank_k == d->rank_v && d->rank_k <= 256 &&
         sync_smem(d->rank_k) <= (size_t)kSmemLimit;
}

void sync_tc_release(lr_cache* c) {
  SyncState* st = reinterpret_cast<SyncState*>(c->sync_state);
  if (st) {
    if (st->rbuf) cudaFree(st->rbuf);
    delete st;
  }
  c->sync_state = nullptr;
}

// Z <- Z R for the sides whose R is given (both R are r x r, fp32, device).
cudaError_t launch_sync_tc(lr_cache* c, const float* R_k, const float* R_v, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  const int r = d.rank_k;
  SyncState* st = reinterpret_cast<SyncState*>(c->sync_state);
  if (!st) {
    st = new (std::nothrow) SyncState();
    if (!st) return cudaErrorMemoryAllocation;
    cudaError_t e = lr_dev_malloc(&st->rbuf, (size_t)2 * 2 * r * r * sizeof(__nv_bfloat16));
    if (e != cudaSuccess) {   // nothing is kept, so the next call starts over
      delete st;
      return e;
    }
    c->sync_state = st;
    st->r = r;
    // [B][capacity][r], or a paged pool as one run of n_pages * 128 rows
    const cuuint64_t cap = c->ptable ? (cuuint64_t)c->n_pages * kPageTokens : d.capacity;
    const cuuint64_t B = c->ptable ? 1 : d.batch;
    cuuint64_t zdims[3] = {(cuuint64_t)r, cap, B};
    cuuint64_t zstr[2] = {(cuuint64_t)r * 2, cap * r * 2};
    cuuint32_t zbox[3] = {64, (cuuint32_t)kTile, 1};
    if (!map_bf16(&st->zk, c->z_k, 3, zdims, zstr, zbox) || !map_bf16(&st->zv, c->z_v, 3, zdims, zstr, zbox))
      return cudaErrorInvalidValue;
    cuuint64_t rdims[2] = {(cuuint64_t)r, (cuuint64_t)2 * r};
    cuuint64_t rstr[1] = {(cuuint64_t)r * 2};
    cuuint32_t rbox[2] = {64, (cuuint32_t)kRRows};
    if (!map_bf16(&st->rk, st->rbuf, 2, rdims, rstr, rbox) ||
        !map_bf16(&st->rv, st->rbuf + (size_t)2 * r * r, 2, rdims, rstr, rbox))
      return cudaErrorInvalidValue;
  }
  // a paged pool is rotated whole: every page once, whatever maps it
  const int rows = c->ptable ? c->n_pages * kPageTokens : c->hist_len;
  const int nseq = c->ptable ? 1 : d.batch;
  const int ntile = (rows + kTile - 1) / kTile;
  if (ntile == 0 || (!R_k && !R_v)) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  const dim3 pgrid(std::min(256, (r * r + 255) / 256));
  if (R_k) e = launch_serial(k_sync_prep, pgrid, dim3(256), 0, s, R_k, st->rbuf, r);
  if (e == cudaSuccess && R_v) e = launch_serial(k_sync_prep, pgrid, dim3(256), 0, s, R_v, st->rbuf + (size_t)2 * r * r, r);
  if (e != cudaSuccess) return e;
  SyncParams p;
  p.wait_ns = c->wait_ns;
  p.r = r;
  p.kb = (r + 63) / 64;
  p.nch = (r + kRRows - 1) / kRRows;
  p.B = nseq;
  p.ntile = ntile;
  p.hist = rows;
  p.z_bytes = (uint32_t)p.kb * kSubBytes;
  p.r_half = (uint32_t)p.kb * kRBox;
  p.r_slot = 2 * p.r_half;
  p.err = c->dev_err;
  // units: the K side first (if R_k), then the V side (if R_v)
  const int sides = (R_k ? 1 : 0) + (R_v ? 1 : 0);
  p.units = sides * nseq * ntile;
  CUtensorMap zk = st->zk, zv = st->zv, rk = st->rk, rv = st->rv;
  if (!R_k) {   // V only: unit side 0 must address the value latents
    zk = st->zv;
    rk = st->rv;
  }
  static std::atomic<uint32_t> optin_done{0};
  e = smem_optin(k_sync_tc, optin_done);
  if (e != cudaSuccess) return e;
  const int grid = std::min(p.units, std::max(1, c->num_sms));
  return launch_pdl(k_sync_tc, dim3(grid), dim3(kThreads), sync_smem(r), s, zk, zv, rk, rv, p);
}
