// Bulk prefill on tensor cores: the latents of a whole prompt, Z = X A (X = the tokens'
// exact keys or values), rounded to bf16 or int4-quantised, written at the cache's next
// slots.
//
// Method: TraceKV abstract (the cache holds low-dimensional latents of the KV states,
// optionally combined with quantization); the latents of n new tokens are n rows of one
// dense contraction, so the projection is a GEMM:
//   Z[t, i] = sum_c X[t, c] A[c, i]     M = 128 tokens, N = r (<= 256 per MMA), K = D
// One CTA per (128-token tile, sequence, side): warp 0 TMA-loads the tile's X (K-major,
// 128-byte swizzle) and the matching rows of A (MN-major: 64 ranks per 128-byte row) per
// 64-wide slice of D through a ring of stages; warp 1 issues the MMAs (bf16, fp32
// accumulation in TMEM); the epilogue warps (kEpiPerQuarter per TMEM lane quarter, taking
// 32-rank groups in turn; thread = token row = TMEM lane) read each 32-rank group of the row and store it: bf16 rows, or the int4 group quantiser of the
// append path (the same fp32 operations, so a given fp32 latent gets the same codes) in the
// token-major key layout or the rank-major value layout (eight tokens' nibbles of one rank
// gathered across eight lanes with shuffles).
//
// Every wait is bounded: on timeout the kernel records LR_ERR_TIMEOUT, drains its own copies
// and MMAs, frees TMEM and returns.
#include "tc_common.cuh"
#include "k_common.cuh"

#include <algorithm>

namespace {

using tc::drain_wait;
using tc::kSmemLimit;
using tc::kTile;

constexpr int kEpiPerQuarter = 4;          // epilogue warps per TMEM lane quarter
constexpr int kThreads = 64 + 128 * kEpiPerQuarter;   // producer, MMA, the epilogue warps
constexpr int kAuxBytes = 1024;
constexpr int kXBytes = 128 * 128;         // X stage: 128 tokens x 64 dims x 2 B
constexpr int kWBox = 64 * 128;            // A box: 64 dims (rows) x 64 ranks x 2 B
constexpr int kMaxStages = 4;

struct PfParams {
  unsigned long long wait_ns;
  int n, D, r_k, r_v, G_k, G_v, slot0, kind, nstage;
  RowMap map;                              // token -> latent row
  void* Zk; void* Zv;                      // bf16 latents (kind LK_BF16)
  uint32_t* codes_k; uint32_t* codes_v; uint32_t* params_k; uint32_t* params_v;
  int* err;
};

// The code min(max(rint(x / sf), 0), 15) with the quotient rounded to fp32 as the division
// rounds it (the append path's quantiser), at the cost of a multiply: y = x * (1/sf) lies within
// 3 ulp of that rounded quotient, so it rounds to the same integer unless it is within a few
// ulp of a half-integer, where the division itself decides.  |y| <= 20 keeps 4 ulp below
// 1e-5; beyond that the clamp decides whatever the rounding.
__device__ __forceinline__ uint32_t quant_code(float x, float sf, float rs) {
  const float y = x * rs;
  const float half_off = fabsf(y - floorf(y) - 0.5f);
  const float q = half_off < 1e-5f ? rintf(__fdiv_rn(x, sf)) : rintf(y);
  return (uint32_t)fminf(fmaxf(q, 0.0f), 15.0f);
}

//   full[s]   1 + tx   producer's TMA boxes of stage s -> MMA issuer
//   empty[s]  1        MMA commit -> producer
//   d_full    1        MMA commit after the last K block -> epilogue warps
struct Aux {
  uint64_t full[kMaxStages], empty[kMaxStages], d_full;
  uint32_t tmem_base;
  int abort_flag;
  unsigned long long wait_ns;
};
static_assert(sizeof(Aux) <= kAuxBytes, "aux block");

__device__ __forceinline__ bool wait_b(uint64_t* bar, uint32_t parity, Aux* aux, int* err) {
  return tc::wait_b(bar, parity, &aux->abort_flag, err, aux->wait_ns);
}
// The same, by a whole warp with one verdict for all its lanes.
__device__ __forceinline__ bool wait_w(uint64_t* bar, uint32_t parity, Aux* aux, int* err) {
  return __all_sync(0xffffffffu, wait_b(bar, parity, aux, err));
}

__device__ __forceinline__ uint32_t tmem_cols_for(int r) { return r <= 256 ? 256u : 512u; }

// Shared memory: [aux 1 KB][stages: X (16 KB) then A (r/64 boxes of 8 KB)]
__global__ void __launch_bounds__(kThreads, 1)
    k_prefill_tc(const __grid_constant__ CUtensorMap tm_xk, const __grid_constant__ CUtensorMap tm_xv,
                 const __grid_constant__ CUtensorMap tm_ak, const __grid_constant__ CUtensorMap tm_av,
                 const PfParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (ptx::smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicExch(p.err, (int)LR_ERR_UNSUPPORTED);
    return;
  }
  Aux* aux = reinterpret_cast<Aux*>(smem_raw);
  uint8_t* stages = smem_raw + kAuxBytes;
  const int tile = blockIdx.x, b = blockIdx.y;
  const bool is_v = blockIdx.z == 1;
  const int r = is_v ? p.r_v : p.r_k;
  const int nwb = (r + 63) / 64;                       // A boxes per stage
  const uint32_t stage_bytes = kXBytes + (uint32_t)nwb * kWBox;
  const int kb = p.D / 64;                             // K blocks of 64 dims
  const uint32_t tcols = tmem_cols_for(r);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.nstage; ++s) {
      ptx::mbar_init(&aux->full[s], 1);
      ptx::mbar_init(&aux->empty[s], 1);
    }
    ptx::mbar_init(&aux->d_full, 1);
    aux->abort_flag = 0;
    aux->wait_ns = tc::wait_limit(p.wait_ns);
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(is_v ? &tm_xv : &tm_xk);
    ptx::prefetch_tmap(is_v ? &tm_av : &tm_ak);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&aux->tmem_base, tcols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = aux->tmem_base;
  pdl_wait();      // the tokens were written by earlier work on the stream
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      const CUtensorMap* tx = is_v ? &tm_xv : &tm_xk;
      const CUtensorMap* ta = is_v ? &tm_av : &tm_ak;
      bool ok = true;
      int issued = 0;
      for (int k = 0; k < kb && ok; ++k) {
        const int s = k % p.nstage, round = k / p.nstage;
        if (round > 0 && !(ok = wait_b(&aux->empty[s], (round - 1) & 1, aux, p.err))) break;
        uint8_t* st = stages + s * stage_bytes;
        ptx::mbar_arrive_expect_tx(&aux->full[s], stage_bytes);
        ptx::tma_load_3d(st, tx, &aux->full[s], k * 64, tile * kTile, b);   // tokens past n read as 0
        for (int w = 0; w < nwb; ++w) ptx::tma_load_2d(st + kXBytes + w * kWBox, ta, &aux->full[s], w * 64, k * 64);
        issued = k + 1;
      }
      // every copy has landed before the CTA can exit (see the decode kernels)
      for (int k = std::max(0, issued - p.nstage); k < issued; ++k)
        drain_wait(&aux->full[k % p.nstage], (k / p.nstage) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    {   // the whole warp runs the loop; an elected lane issues
      // N per MMA: the whole rank, or 256 then the rest above 256 (the second MMA's B starts
      // at the fifth 64-rank box, its D at TMEM column 256)
      const int nh = r > 256 ? 2 : 1;
      const uint32_t id0 = ptx::idesc_f16(1, 0, 1, 128, (uint32_t)std::min(r, 256));   // bf16; X K-major, A MN-major
      const uint32_t id1 = ptx::idesc_f16(1, 0, 1, 128, (uint32_t)std::max(16, r - 256));
      const uint64_t xdesc0 = ptx::smem_desc(ptx::smem_u32(stages), 16, 1024, 2);
      const uint64_t adesc0 = ptx::smem_desc(ptx::smem_u32(stages + kXBytes), kWBox, 1024, 2);
      bool ok = true;
      for (int k = 0; k < kb && ok; ++k) {
        const int s = k % p.nstage;
        if (!(ok = wait_w(&aux->full[s], (k / p.nstage) & 1, aux, p.err))) break;
        ptx::tc_fence_after();
        const uint64_t xs = xdesc0 + (uint64_t)((s * stage_bytes) >> 4);
        const uint64_t as = adesc0 + (uint64_t)((s * stage_bytes) >> 4);
        for (int kk = 0; kk < 4; ++kk) {                // 16 dims per MMA: 32 B on X, 16 rows on A
          for (int hh = 0; hh < nh; ++hh)
            ptx::mma_f16_elect(tmem + hh * 256, xs + (uint64_t)(kk * 2),
                         as + (uint64_t)((hh * 4 * kWBox + kk * 16 * 128) >> 4), hh ? id1 : id0, (k | kk) ? 1u : 0u);
        }
        ptx::mma_commit_elect(&aux->empty[s]);
      }
      ptx::mma_commit_elect(&aux->d_full);
      drain_wait(&aux->d_full, 0);                      // every MMA done before TMEM is freed
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------- epilogue
    // kEpiPerQuarter warps per TMEM lane quarter, taking 32-rank groups in turn: one warp
    // per sub-partition left the epilogue's dependent chains (shuffles, index arithmetic)
    // without another warp to hide their latency
    const int qd = warp & 3;
    const int part = (warp - 2) >> 2;
    const int m = qd * 32 + lane;                       // token row of the tile
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    const int t = tile * kTile + m;
    const bool valid = t < p.n;
    const long long row = valid ? p.map.row(b, p.slot0 + t) : 0;   // the table has no row past n
    const bool ok = ptx::named_bar_and(1, 128 * kEpiPerQuarter, wait_b(&aux->d_full, 0, aux, p.err));
    if (ok) {
      ptx::tc_fence_after();
      const int G = (r + 31) / 32;
      const bool aligned = (p.slot0 & 7) == 0;
      for (int g = part; g < G; g += kEpiPerQuarter) {
        uint32_t v[32];
        ptx::tmem_ld32(tmem + lane_off + g * 32, v);
        ptx::tmem_wait_ld();
        const int nvalid = min(32, r - g * 32);        // 16 in a final half group
        if (p.kind == LK_BF16) {
          if (valid) {
            __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(is_v ? p.Zv : p.Zk) + row * r + g * 32;
            for (int e = 0; e < nvalid; e += 8) {
              uint4 w;
              uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const __nv_bfloat162 h2 =
                    __floats2bfloat162_rn(__uint_as_float(v[e + 2 * k]), __uint_as_float(v[e + 2 * k + 1]));
                wp[k] = *reinterpret_cast<const uint32_t*>(&h2);
              }
              *reinterpret_cast<uint4*>(dst + e) = w;
            }
          }
          continue;
        }
        // int4: the group quantiser of the append path, one thread per token row
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e < nvalid) {
            mn = fminf(mn, __uint_as_float(v[e]));
            mx = fmaxf(mx, __uint_as_float(v[e]));
          }
        __half zh = __float2half_rn(mn);
        if (__half2float(zh) == 0.0f) zh = __ushort_as_half((unsigned short)0);
        const __half sh = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
        const float zf = __half2float(zh), sf = __half2float(sh);
        const float rs = sf != 0.0f ? __frcp_rn(sf) : 0.0f;
        uint32_t code[32];
#pragma unroll
        for (int e = 0; e < 32; ++e)
          code[e] = (e < nvalid && sf != 0.0f) ? quant_code(__fsub_rn(__uint_as_float(v[e]), zf), sf, rs) : 0u;
        const int G_s = is_v ? p.G_v : p.G_k;
        if (!is_v) {
          if (valid) {
            uint4 w = make_uint4(0u, 0u, 0u, 0u);
            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
            for (int e = 0; e < 32; ++e) wp[e >> 3] |= code[e] << (4 * (e & 7));
            *reinterpret_cast<uint4*>(p.codes_k + i4_code_index(row, G_s, g, 0)) = w;
            p.params_k[i4_param_index(row, G_s, g)] =
                (uint32_t)__half_as_ushort(sh) | ((uint32_t)__half_as_ushort(zh) << 16);
          }
        } else {
          unsigned short* h = reinterpret_cast<unsigned short*>(p.params_v);
          if (valid) {
            const long long si = i4v_scale_index(row, G_s, g);
            h[si] = __half_as_ushort(sh);
            h[si + 128] = __half_as_ushort(zh);
          }
          const int sh4 = 4 * i4v_nibble(row);
          if (aligned) {
            // lanes 8w .. 8w+7 hold the eight tokens of one word of every rank: OR their
            // nibbles together, then lane k stores the words of ranks k, k + 8, k + 16, k + 24.
            // Tokens past n contribute 0 (their slots hold no data); a word whose first token
            // is past n is not stored at all (its slots may lie beyond the storage).
            const int tb = t & ~7;
            const long long row_w = tb < p.n ? p.map.row(b, p.slot0 + tb) : 0;
            // the word of rank g * 32 + e: its rank row's base, then the 16-byte column
            // (token quarter ^ ((e / 2) % 4)) and the word in it (g * 32 is a multiple of 8,
            // so the rotation depends on e alone)
            uint32_t* vrow = p.codes_v + i4v_code_index(row_w, G_s, g * 32) - ((((row_w & 127) >> 5)) << 2);
            const uint32_t tq = (uint32_t)((row_w & 127) >> 5);
            // per block of 8 ranks, a butterfly reduce-scatter over the word's 8 lanes: lane
            // m of the word ends with the OR of all 8 lanes' nibbles of rank 8 jb + m (seven
            // shuffles per block instead of three per rank)
            const int m8 = lane & 7;
            uint32_t* vlane = vrow + m8 * 16 + ((tq ^ (uint32_t)((m8 >> 1) & 3)) << 2);
#pragma unroll
            for (int jb = 0; jb < 4; ++jb) {
              uint32_t x[8];
#pragma unroll
              for (int m = 0; m < 8; ++m) x[m] = valid ? code[8 * jb + m] << sh4 : 0u;
#pragma unroll
              for (int dd = 4; dd >= 1; dd >>= 1) {
                const bool up = (lane & dd) != 0;
#pragma unroll
                for (int k = 0; k < dd; ++k) {
                  const uint32_t keep = up ? x[k + dd] : x[k];
                  const uint32_t send = up ? x[k] : x[k + dd];
                  x[k] = keep | __shfl_xor_sync(0xffffffffu, send, dd);
                }
              }
              if (8 * jb + m8 < nvalid && tb < p.n) vlane[jb * 128] = x[0];
            }
          } else if (valid) {
            // a fill that starts inside a word shares it with older tokens: this token's
            // nibbles only (the two atomics touch only its bits).  The loop runs to 32 with a
            // guard so that code[] keeps constant indices and stays in registers.
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              if (e < nvalid) {
                uint32_t* w = p.codes_v + i4v_code_index(row, G_s, g * 32 + e);
                atomicAnd(w, ~(15u << sh4));
                if (code[e]) atomicOr(w, code[e] << sh4);
              }
            }
          }
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, tcols);
  }
}

}  // namespace

bool prefill_tc_supported(const lr_cache_desc* d, int D) {
  return d->dtype == LR_BF16 && d->window == 0 && D % 64 == 0;
}

cudaError_t launch_prefill_tc(lr_cache* c, const void* k, const void* v, int n, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  const int D = c->D;
  if (!prefill_tc_supported(&d, D)) return cudaErrorNotSupported;
  CUtensorMap xk, xv, ak, av;
  cuuint64_t xdims[3] = {(cuuint64_t)D, (cuuint64_t)n, (cuuint64_t)d.batch};
  cuuint64_t xstr[2] = {(cuuint64_t)D * 2, (cuuint64_t)n * D * 2};
  cuuint32_t xbox[3] = {64, (cuuint32_t)kTile, 1};
  if (!tc::make_map(&xk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, 3, xdims, xstr, xbox) ||
      !tc::make_map(&xv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, v, 3, xdims, xstr, xbox))
    return cudaErrorInvalidValue;
  cuuint64_t akd[2] = {(cuuint64_t)d.rank_k, (cuuint64_t)D}, avd[2] = {(cuuint64_t)d.rank_v, (cuuint64_t)D};
  cuuint64_t aks[1] = {(cuuint64_t)d.rank_k * 2}, avs[1] = {(cuuint64_t)d.rank_v * 2};
  cuuint32_t abox[2] = {64, 64};
  if (!tc::make_map(&ak, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c->A_k, 2, akd, aks, abox) ||
      !tc::make_map(&av, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, c->A_v, 2, avd, avs, abox))
    return cudaErrorInvalidValue;
  PfParams p;
  p.wait_ns = c->wait_ns;
  p.n = n;
  p.D = D;
  p.r_k = d.rank_k;
  p.r_v = d.rank_v;
  p.G_k = c->G_k;
  p.G_v = c->G_v;
  p.slot0 = c->hist_len;
  p.kind = c->latent_kind;
  p.map = row_map(c);
  p.Zk = c->z_k;
  p.Zv = c->z_v;
  p.codes_k = c->codes_k;
  p.codes_v = c->codes_v;
  p.params_k = c->params_k;
  p.params_v = c->params_v;
  p.err = c->dev_err;
  const int rmax = std::max(d.rank_k, d.rank_v);
  const size_t stage = (size_t)kXBytes + (size_t)((rmax + 63) / 64) * kWBox;
  p.nstage = std::min(kMaxStages, (int)(((size_t)kSmemLimit - kAuxBytes) / stage));
  if (p.nstage < 2) return cudaErrorNotSupported;
  const size_t smem = kAuxBytes + (size_t)p.nstage * stage;
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_prefill_tc, optin_done);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_prefill_tc, dim3((n + kTile - 1) / kTile, d.batch, 2), dim3(kThreads), smem, s, xk, xv, ak,
                    av, p);
}
