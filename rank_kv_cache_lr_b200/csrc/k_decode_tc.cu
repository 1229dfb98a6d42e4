// Tensor-core (tcgen05) split-sequence decode over bf16 latents.
//
// Method: TraceKV abstract ("optimized low-rank attention kernels" over latent KV
// states).  Attention runs in rank space (exact identity q . (z B_h) = (B_h q) . z):
//   S[t, j]  = z_k,t . q~_j          GEMM1: M = 128 tokens, N = 64, K = r_k
//   p[t, j]  = exp2(S[t, j] - m_j)   online softmax, lazy max (rescale only when the
//                                    running max grows by more than 2^8)
//   O~[e, j] += sum_t z_v,t[e] p[t,j] GEMM2: M = 128 ranks per chunk, N = 64, K = 128 tokens
// The ring and the MMAs follow the order K(0), K(1), V(0), K(2), V(1), ..., so the scores
// of tile s+1 are computed while the softmax of tile s runs (S double-buffered in TMEM).
// The query latent q~ (scaled by s log2 e) enters GEMM1 as two bf16 halves, hi and
// lo = q~ - hi, stacked on N (B rows 0..31 and 32..63), so the scores carry almost
// fp32 precision while the stored latents stay bf16.  The probabilities enter GEMM2
// the same way (p = p_hi + p_lo), so the value mix and the normaliser l are both
// computed from ~fp32 weights; a single bf16 rounding of p would bias l when the
// weights cluster (near-uniform softmax).  One N = 64 MMA costs what an N = 32 MMA
// costs on this tensor core, so the halves go through N rather than through a second
// MMA; the softmax and the epilogue add the two 32-column halves of each accumulator.
// Accumulators live in TMEM: S in two buffers of 64 columns (hi | lo), O~ in
// ceil(r_v/128) chunks of 64 columns (hi | lo).
//
// Roles (192 threads): warp 0 issues TMA tile loads (128 tokens x 64 ranks boxes,
// 128-byte swizzle, no multicast) into a ring of 32 KB slots (one 128-rank chunk of
// K or V for one 128-token tile); warp 1 owns TMEM and issues tcgen05.mma from one
// thread; warps 2..5 run the softmax (thread = token row = TMEM lane) and the
// epilogue (thread = rank row).  Every wait is bounded: on timeout the kernel records
// LR_ERR_TIMEOUT, drains its own copies and MMAs, frees TMEM and returns.
#include "tc_common.cuh"

#include <algorithm>

namespace {

using tc::drain_wait;
using tc::kLazy;
using tc::kSmemLimit;
using tc::kTile;
using tc::kTraceSlots;
using tc::warp_reduce_scatter32;

constexpr int kThreads = 192;
constexpr int kSubBytes = 128 * 128;       // 128 tokens x 64 ranks x 2 B
constexpr int kSlotBytes = 2 * kSubBytes;  // 128 tokens x 128 ranks
constexpr int kQRows = 64;                 // 32 head rows (hi) + 32 head rows (lo)
constexpr int kQSubBytes = kQRows * 128;   // 64 rows x 64 ranks x 2 B
constexpr int kPHalfBytes = 128 * 32 * 2;  // 128 tokens x 32 heads x 2 B (one of hi, lo)
constexpr int kPBytes = 2 * kPHalfBytes;
constexpr int kAuxBytes = 1024;            // barriers and reduction scratch, first in smem
constexpr int kSCol = 0;                   // TMEM: S of tile s in columns [64 (s % 2), +64) (hi | lo)
constexpr int kOCol = 128;                 // TMEM: O~ chunk c in columns [128 + 64c, +64) (hi | lo)
constexpr int kMaxSlots = 8;
constexpr int kSmemPair = 115712;          // per block when two blocks share an SM (228 KB - 2 x 1 KB)

struct TcParams {
  unsigned long long wait_ns;   // bounded-wait limit (0: the default)
  const int32_t* row_len;       // per-row history lengths (device), or null
  unsigned long long* span;     // timeline span, or null
  RowMap map;                   // paged caches: the block table (maps address pages), else table null
  int r_k, r_v, ck, cv, kb_k, tmem_cols;
  int Hq, hist_len, stable_len, split_tokens, n_splits, nslot;
  uint32_t q_bytes;
  float* part_o;
  float* part_ml;
  int* err;
  unsigned long long* trace;   // optional per-CTA timeline (kTraceSlots stamps per CTA), or null
};

// Barriers (arrival count; who arrives -> who waits); phase k is waited with parity k & 1.
//   slot_full[nslot]  1 + tx   producer's TMA boxes of one 128-rank chunk -> MMA issuer
//   slot_empty[nslot] 1        MMA commit -> producer
//   q_full            1 + tx   producer (after the grid-dependency wait) -> MMA issuer
//   s_full[2]         1        MMA commit of GEMM1 -> softmax warps
//   s_empty[2]        4        softmax warps (scores read) -> MMA issuer
//   p_full            4        softmax warps (fenced P stores) -> MMA issuer
//   p_empty           1        MMA commit of GEMM2 -> softmax warps (P reuse, O~ rescale)
//   o_final           1        MMA commit after the last unit -> softmax warps (epilogue)
struct Aux {
  uint64_t slot_full[kMaxSlots];
  uint64_t slot_empty[kMaxSlots];
  uint64_t s_full[2], s_empty[2];
  uint64_t q_full, p_full, p_empty, o_final;
  uint32_t tmem_base;
  int abort_flag;
  unsigned long long wait_ns;   // this launch's wait limit
  float red[4][32];
  float m_s[32];
  float alpha_s[32];
};
static_assert(sizeof(Aux) <= kAuxBytes, "aux block");

struct TcState {
  CUtensorMap q, zk, zv;
  int nslot_pair, nslot_single;   // ring slots with two blocks per SM (0: not possible) / with one
  size_t smem_pair, smem_single;
};

// Row `lane_off` of an N = 64 accumulator at column `col`: hi (columns 0..31) + lo
// (32..63), 16 columns at a time.
__device__ __forceinline__ void tmem_ld_sum(uint32_t taddr, float (&v)[32]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t a[16], b[16];
    ptx::tmem_ld16(taddr + 16 * h, a);
    ptx::tmem_ld16(taddr + 32 + 16 * h, b);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int j = 0; j < 16; ++j) v[16 * h + j] = __uint_as_float(a[j]) + __uint_as_float(b[j]);
  }
}

__device__ __forceinline__ bool wait_b(uint64_t* bar, uint32_t parity, Aux* aux, int* err) {
  return tc::wait_b(bar, parity, &aux->abort_flag, err, aux->wait_ns);
}
// The same, by a whole warp with one verdict for all its lanes.
__device__ __forceinline__ bool wait_w(uint64_t* bar, uint32_t parity, Aux* aux, int* err) {
  return __all_sync(0xffffffffu, wait_b(bar, parity, aux, err));
}

__device__ __forceinline__ void trace_stamp(const TcParams& p, int slot) { tc::trace_stamp(p.trace, slot); }

// Shared memory: [aux 1 KB][q~ hi|lo per 64-rank sub-block][ring of nslot x 32 KB][P hi | P lo].
// The dynamic shared-memory window starts 1024-byte aligned (checked); the swizzled
// operands sit at 1024-byte multiples.
__global__ void __launch_bounds__(kThreads, 2)
    k_decode_tc(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_zk,
                const __grid_constant__ CUtensorMap tm_zv, const TcParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (ptx::smem_u32(smem_raw) & 1023) {      // layout precondition; uniform for the whole CTA
    if (threadIdx.x == 0) atomicExch(p.err, (int)LR_ERR_UNSUPPORTED);
    return;
  }
  span_begin(p.span);
  Aux* aux = reinterpret_cast<Aux*>(smem_raw);
  uint8_t* q_s = smem_raw + kAuxBytes;
  uint8_t* ring = q_s + p.q_bytes;
  uint8_t* p_s = ring + p.nslot * kSlotBytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x, b = blockIdx.y;
  const int tok_begin = split * p.split_tokens;
  const int tok_end = min(row_hist(p.row_len, b, p.hist_len), tok_begin + p.split_tokens);
  const int ntiles = tok_end > tok_begin ? (tok_end - tok_begin + kTile - 1) / kTile : 0;
  const int nunits = 2 * ntiles;

  if (threadIdx.x == 0) {
    trace_stamp(p, 0);
    for (int s = 0; s < p.nslot; ++s) {
      ptx::mbar_init(&aux->slot_full[s], 1);
      ptx::mbar_init(&aux->slot_empty[s], 1);
    }
    ptx::mbar_init(&aux->q_full, 1);
    for (int k = 0; k < 2; ++k) {
      ptx::mbar_init(&aux->s_full[k], 1);
      ptx::mbar_init(&aux->s_empty[k], 4);     // one arrival per softmax warp
    }
    ptx::mbar_init(&aux->p_full, 4);
    ptx::mbar_init(&aux->p_empty, 1);
    ptx::mbar_init(&aux->o_final, 1);
    aux->abort_flag = 0;
    aux->wait_ns = tc::wait_limit(p.wait_ns);
    for (int j = 0; j < 32; ++j) aux->m_s[j] = -INFINITY;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    ptx::prefetch_tmap(&tm_q);
    ptx::prefetch_tmap(&tm_zk);
    ptx::prefetch_tmap(&tm_zv);
  }
  if (warp == 1) {
    ptx::tmem_alloc(&aux->tmem_base, p.tmem_cols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = aux->tmem_base;
  if (!(warp == 0 && lane == 0)) pdl_wait();   // the producer waits after its first loads
  pdl_trigger();
  if (threadIdx.x == 32) trace_stamp(p, 1);

  if (warp == 0) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0 && ntiles > 0) {
      // The first round of the ring is issued before the grid-dependency wait when every
      // token of its tiles lies below stable_len: those rows were written by kernels that
      // completed before the preceding kernel allowed this one to start.  The query
      // latents, and rows the preceding kernel appends, come after the wait.
      int issued = 0, pos = 0;
      bool ok = true;
      bool q_issued = false;
      for (int u = 0; u < nunits && ok; ++u) {
        int tile;
        bool isv;
        tc::unit_of(u, ntiles, &tile, &isv);
        const int t0 = tok_begin + tile * kTile;
        // box origin: (token, sequence), or (0, page) in a paged pool (a tile is one page)
        const int ty = p.map.table ? 0 : t0;
        const int tz = p.map.table ? p.map.page(b, t0) : b;
        const int nch = isv ? p.cv : p.ck;
        const int r = isv ? p.r_v : p.r_k;
        for (int c = 0; c < nch; ++c, ++pos) {
          const int slot = pos % p.nslot, round = pos / p.nslot;
          if (!q_issued && (round > 0 || t0 + kTile > p.stable_len)) {
            pdl_wait();
            ptx::mbar_arrive_expect_tx(&aux->q_full, p.q_bytes);
            for (int sb = 0; sb < p.kb_k; ++sb)
              ptx::tma_load_2d(q_s + sb * kQSubBytes, &tm_q, &aux->q_full, sb * 64, b * kQRows);
            q_issued = true;
          }
          if (round > 0 && !wait_b(&aux->slot_empty[slot], (round - 1) & 1, aux, p.err)) {
            ok = false;
            break;
          }
          const int nsub = (c * 128 + 64 < r) ? 2 : 1;
          uint8_t* dst = ring + slot * kSlotBytes;
          ptx::mbar_arrive_expect_tx(&aux->slot_full[slot], nsub * kSubBytes);
          for (int sb = 0; sb < nsub; ++sb)
            ptx::tma_load_3d(dst + sb * kSubBytes, isv ? &tm_zv : &tm_zk, &aux->slot_full[slot],
                             c * 128 + sb * 64, ty, tz);
          issued = pos + 1;
        }
      }
      if (!q_issued) {
        pdl_wait();
        ptx::mbar_arrive_expect_tx(&aux->q_full, p.q_bytes);
        for (int sb = 0; sb < p.kb_k; ++sb)
          ptx::tma_load_2d(q_s + sb * kQSubBytes, &tm_q, &aux->q_full, sb * 64, b * kQRows);
      }
      // Every copy this thread issued has landed before the CTA can exit: after an abort
      // (here or in another role, which may come after this loop) the consumers stop
      // waiting for them.  In a normal run these are the phases the consumers already
      // waited for, so the waits return at once.
      drain_wait(&aux->q_full, 0);
      for (int pos = max(0, issued - p.nslot); pos < issued; ++pos)
        drain_wait(&aux->slot_full[pos % p.nslot], (pos / p.nslot) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------- MMA issuer
    // The whole warp runs the loop (operands warp-uniform, K steps unrolled) and one
    // elected lane issues each MMA: far faster issue than a loop run by one lane.
    if (ntiles > 0) {
      const uint32_t id = ptx::idesc_f16(1, 0, 0, 128, 64);    // GEMM1: K-major x K-major, N = 64 (hi | lo)
      const uint32_t id2 = ptx::idesc_f16(1, 1, 1, 128, 64);   // GEMM2: MN-major x MN-major, N = 64 (hi | lo)
      // Descriptors are built once; a step along K or to another slot adds its byte
      // offset >> 4 to the start-address field (no carry: shared memory < 256 KB).
      const uint64_t kdesc0 = ptx::smem_desc(ptx::smem_u32(ring), 16, 1024, 2);
      const uint64_t qdesc0 = ptx::smem_desc(ptx::smem_u32(q_s), 16, 1024, 2);
      const uint64_t vdesc0 = ptx::smem_desc(ptx::smem_u32(ring), kSubBytes, 1024, 2);
      const uint64_t pdesc0 = ptx::smem_desc(ptx::smem_u32(p_s), 128, 2048, 0);
      bool ok = wait_w(&aux->q_full, 0, aux, p.err);
      ptx::tc_fence_after();
      if (lane == 0) trace_stamp(p, 2);
      int pos = 0;
      for (int u = 0; u < nunits && ok; ++u) {
        int tile;
        bool isv;
        tc::unit_of(u, ntiles, &tile, &isv);
        if (!isv) {
          // GEMM1(tile): S[tile % 2] = Z_k [q~_hi | q~_lo]^T
          const int sb2 = tile & 1;
          if (tile >= 2 && !(ok = wait_w(&aux->s_empty[sb2], ((tile - 2) >> 1) & 1, aux, p.err))) break;
          ptx::tc_fence_after();
          const uint32_t d_s = tmem + kSCol + 64 * sb2;
          for (int c = 0; c < p.ck && ok; ++c, ++pos) {
            const int slot = pos % p.nslot;
            if (!(ok = wait_w(&aux->slot_full[slot], (pos / p.nslot) & 1, aux, p.err))) break;
            ptx::tc_fence_after();
            const uint64_t a0 = kdesc0 + (uint64_t)((slot * kSlotBytes) >> 4);
            const uint64_t b0 = qdesc0 + (uint64_t)((c * 2 * kQSubBytes) >> 4);
            const int nk = min(8, (p.r_k - c * 128) >> 4);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint64_t ad = a0 + (uint64_t)((kk >> 2) * (kSubBytes >> 4) + (kk & 3) * 2);
              const uint64_t bd = b0 + (uint64_t)((kk >> 2) * (kQSubBytes >> 4) + (kk & 3) * 2);
              if (kk < nk) ptx::mma_f16_elect(d_s, ad, bd, id, (c | kk) ? 1u : 0u);
            }
            ptx::mma_commit_elect(&aux->slot_empty[slot]);
          }
          if (!ok) break;
          ptx::mma_commit_elect(&aux->s_full[sb2]);
          if (tile < 16 && lane == 0) trace_stamp(p, 3 + 4 * tile);
        } else {
          // GEMM2(tile): O~ += Z_v^T [P_hi | P_lo]
          if (!(ok = wait_w(&aux->p_full, tile & 1, aux, p.err))) break;
          ptx::tc_fence_after();
          for (int c = 0; c < p.cv && ok; ++c, ++pos) {
            const int slot = pos % p.nslot;
            if (!(ok = wait_w(&aux->slot_full[slot], (pos / p.nslot) & 1, aux, p.err))) break;
            ptx::tc_fence_after();
            const uint64_t a0 = vdesc0 + (uint64_t)((slot * kSlotBytes) >> 4);
            const uint32_t d_o = tmem + kOCol + c * 64;
#pragma unroll
            for (int kt = 0; kt < 8; ++kt) {
              const uint64_t ad = a0 + (uint64_t)(kt * 128);
              const uint64_t bd = pdesc0 + (uint64_t)(kt * 16);
              ptx::mma_f16_elect(d_o, ad, bd, id2, (tile | kt) ? 1u : 0u);
            }
            ptx::mma_commit_elect(&aux->slot_empty[slot]);
          }
          if (!ok) break;
          ptx::mma_commit_elect(&aux->p_empty);
          if (tile < 16 && lane == 0) trace_stamp(p, 6 + 4 * tile);
        }
      }
      ptx::mma_commit_elect(&aux->o_final);
      // the MMAs have completed before TMEM is freed, even if the epilogue aborted
      drain_wait(&aux->o_final, 0);
    }
    __syncwarp();
  } else if (ntiles > 0) {
    // ------------------------------------------------------------- softmax / epilogue
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
    float l[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) l[j] = 0.f;
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const bool valid = tok_begin + i * kTile + row < tok_end;
      const int k2 = i & 1;
      const uint32_t s_col = tmem + lane_off + kSCol + 64 * k2;
      ok = ptx::named_bar_and(1, 128, wait_b(&aux->s_full[k2], (i >> 1) & 1, aux, p.err));
      if (!ok) break;
      ptx::tc_fence_after();
      if (i < 16 && threadIdx.x == 64) trace_stamp(p, 4 + 4 * i);
      float s[32];
      tmem_ld_sum(s_col, s);
#pragma unroll
      for (int j = 0; j < 32; ++j) s[j] = valid ? s[j] : -INFINITY;

      bool ex = false;
#pragma unroll
      for (int j = 0; j < 32; ++j) ex |= s[j] > aux->m_s[j] + kLazy;
      ex = ptx::named_bar_or(1, 128, ex);
      if (i >= 1) {   // the value mix of tile i - 1 has completed: P may be rewritten, O~ rescaled
        ok = ptx::named_bar_and(1, 128, wait_b(&aux->p_empty, (i - 1) & 1, aux, p.err));
        if (!ok) break;
        ptx::tc_fence_after();
      }
      if (ex) {
        // reduce in place, then read the scores again (S stays intact until s_empty)
        aux->red[qd][lane] = warp_reduce_scatter32<true>(s, lane);
        tmem_ld_sum(s_col, s);
#pragma unroll
        for (int j = 0; j < 32; ++j) s[j] = valid ? s[j] : -INFINITY;
        ptx::named_bar_sync(1, 128);
        if (qd == 0) {
          const float mt = fmaxf(fmaxf(aux->red[0][lane], aux->red[1][lane]), fmaxf(aux->red[2][lane], aux->red[3][lane]));
          const float mo = aux->m_s[lane];
          const float mn = fmaxf(mo, mt);
          aux->alpha_s[lane] = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
          aux->m_s[lane] = mn;
        }
        ptx::named_bar_sync(1, 128);
        bool need_o = false;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float a = aux->alpha_s[j];
          l[j] *= a;
          need_o |= a < 1.f;
        }
        if (need_o && i > 0) {
          for (int c = 0; c < 2 * p.cv; ++c) {   // both halves of every chunk
            uint32_t v2[32];
            ptx::tmem_ld32(tmem + lane_off + kOCol + c * 32, v2);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) v2[j] = __float_as_uint(__uint_as_float(v2[j]) * aux->alpha_s[j]);
            ptx::tmem_st32(tmem + lane_off + kOCol + c * 32, v2);
          }
          ptx::tmem_wait_st();
        }
      }
      // probabilities in two bf16 halves: p = hi + lo, hi = bf16(p), lo = bf16(p - hi)
      const uint32_t prow = ptx::smem_u32(p_s + row * 16);
#pragma unroll
      for (int hg = 0; hg < 4; ++hg) {
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = hg * 8 + 2 * e;
          const float p0 = exp2f(s[j] - aux->m_s[j]);
          const float p1 = exp2f(s[j + 1] - aux->m_s[j + 1]);
          const __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
          const __nv_bfloat162 lo2 = __floats2bfloat162_rn(p0 - __low2float(h), p1 - __high2float(h));
          l[j] += p0;
          l[j + 1] += p1;
          hw[e] = *reinterpret_cast<const uint32_t*>(&h);
          lw[e] = *reinterpret_cast<const uint32_t*>(&lo2);
        }
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + hg * 2048), "r"(hw[0]), "r"(hw[1]),
                     "r"(hw[2]), "r"(hw[3])
                     : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + kPHalfBytes + hg * 2048), "r"(lw[0]),
                     "r"(lw[1]), "r"(lw[2]), "r"(lw[3])
                     : "memory");
      }
      // every lane makes its own P stores visible to the tensor core, then one arrival per warp
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&aux->s_empty[k2]);
        ptx::mbar_arrive(&aux->p_full);
      }
      if (i < 16 && threadIdx.x == 64) trace_stamp(p, 5 + 4 * i);
    }
    if (ok) ok = ptx::named_bar_and(1, 128, wait_b(&aux->o_final, 0, aux, p.err));
    if (ok) {
      ptx::tc_fence_after();
      const size_t base_out = ((size_t)b * p.n_splits + split) * p.Hq;
      // the normaliser first, so its 32 registers are free for the two accumulator halves
      aux->red[qd][lane] = warp_reduce_scatter32<false>(l, lane);
      ptx::named_bar_sync(1, 128);
      if (qd == 0 && lane < p.Hq) {
        const float lt = (aux->red[0][lane] + aux->red[1][lane]) + (aux->red[2][lane] + aux->red[3][lane]);
        p.part_ml[(base_out + lane) * 2] = aux->m_s[lane];
        p.part_ml[(base_out + lane) * 2 + 1] = lt;
      }
      for (int c = 0; c < p.cv; ++c) {
        float o[32];
        tmem_ld_sum(tmem + lane_off + kOCol + c * 64, o);
        const int e = c * 128 + qd * 32 + lane;
        if (e < p.r_v) {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < p.Hq) p.part_o[(base_out + j) * p.r_v + e] = o[j];
        }
      }
      if (threadIdx.x == 64) trace_stamp(p, kTraceSlots - 1);
    }
  } else if (warp == 2) {
    // a split that starts beyond its row's length: zero weight in the merge
    const size_t base_out = ((size_t)b * p.n_splits + split) * p.Hq;
    if (lane < p.Hq) {
      p.part_ml[(base_out + lane) * 2] = -INFINITY;
      p.part_ml[(base_out + lane) * 2 + 1] = 0.f;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, p.tmem_cols);
  }
  span_end(p.span);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

bool make_map(CUtensorMap* m, const void* ptr, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
              const cuuint32_t* box) {
  return tc::make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, ptr, rank, dims, strides, box);
}

int q_bytes_for(int r_k) { return ((r_k + 63) / 64) * kQSubBytes; }

size_t smem_for(int r_k, int nslot) { return (size_t)kAuxBytes + q_bytes_for(r_k) + (size_t)nslot * kSlotBytes + kPBytes; }

int tmem_cols_for(int r_v) {
  const int cols = kOCol + 64 * ((r_v + 127) / 128);
  return cols <= 128 ? 128 : (cols <= 256 ? 256 : 512);
}

// Ring slots with two blocks per SM (a 2-slot ring in half the SM; 0 if the block does not
// fit) and with one block per SM (as many slots as fit).
int slots_pair(const lr_cache_desc* d) {
  return (smem_for(d->rank_k, 2) <= (size_t)kSmemPair && tmem_cols_for(d->rank_v) <= 256) ? 2 : 0;
}
int slots_single(const lr_cache_desc* d) {
  int n = 0;
  while (n + 1 <= kMaxSlots && smem_for(d->rank_k, n + 1) <= (size_t)kSmemLimit) ++n;
  return n;
}

}  // namespace

bool tc_supported(const lr_cache_desc* d) {
  if (d->quant_bits == 4) return tc_i4_supported(d);
  if (d->dtype != LR_BF16 || d->quant_bits != 0 || d->rope_in_kernel) return false;
  if (d->n_q_heads > 32) return false;
  return slots_single(d) >= 1;
}

// Two blocks per SM whenever they fit: each block's tile chain (scores, softmax, value
// mix) is serial, and a second block overlaps it on the same SM; measured faster than one
// block with a deep ring both at 4K and at 16K tokens.
int tc_ctas_per_sm(const lr_cache_desc* d, int hist_len, int num_sms) {
  (void)hist_len;
  (void)num_sms;
  if (d->quant_bits == 4) return 1;
  return slots_pair(d) ? 2 : 1;
}

int tc_split_ctas(const lr_cache_desc* d) { return d->quant_bits == 4 ? tc_i4_split_ctas(d) : 1; }

cudaError_t tc_prepare(lr_cache* c, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  if (!tc_supported(&d)) return cudaSuccess;
  if (d.quant_bits == 4) return tc_i4_prepare(c, s);
  TcState* st = reinterpret_cast<TcState*>(c->tc_state);
  if (!st) {
    st = new (std::nothrow) TcState();
    if (!st) return cudaErrorMemoryAllocation;
    c->tc_state = st;
  }
  if (!c->qt16) {
    cudaError_t e = lr_dev_malloc(&c->qt16, (size_t)d.batch * kQRows * d.rank_k * 2);
    if (e != cudaSuccess) return e;
    e = cudaMemset(c->qt16, 0, (size_t)d.batch * kQRows * d.rank_k * 2);
    if (e != cudaSuccess) return e;
  }
  // latent maps: [B][capacity][r], or the paged pool [n_pages][128][r]
  const cuuint64_t B = d.batch;
  const cuuint64_t rows = c->ptable ? kPageTokens : d.capacity, seqs = c->ptable ? c->n_pages : B;
  {
    cuuint64_t dims[2] = {(cuuint64_t)d.rank_k, B * kQRows};
    cuuint64_t strides[1] = {(cuuint64_t)d.rank_k * 2};
    cuuint32_t box[2] = {64, kQRows};
    if (!make_map(&st->q, c->qt16, 2, dims, strides, box)) return cudaErrorInvalidValue;
  }
  for (int side = 0; side < 2; ++side) {
    const int r = side ? d.rank_v : d.rank_k;
    cuuint64_t dims[3] = {(cuuint64_t)r, rows, seqs};
    cuuint64_t strides[2] = {(cuuint64_t)r * 2, rows * r * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)kTile, 1};
    if (!make_map(side ? &st->zv : &st->zk, side ? c->z_v : c->z_k, 3, dims, strides, box))
      return cudaErrorInvalidValue;
  }
  st->nslot_pair = slots_pair(&d);
  st->nslot_single = slots_single(&d);
  st->smem_pair = smem_for(d.rank_k, st->nslot_pair);
  st->smem_single = smem_for(d.rank_k, st->nslot_single);
  return cudaSuccess;
}

void tc_release(lr_cache* c) {
  if (c->desc.quant_bits == 4) {
    tc_i4_release(c);
    return;
  }
  delete reinterpret_cast<TcState*>(c->tc_state);
  c->tc_state = nullptr;
}

cudaError_t launch_decode_tc(const lr_cache* c, int n_splits, int split_tokens, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  if (d.quant_bits == 4) return launch_decode_tc_i4(c, n_splits, split_tokens, s);
  const TcState* st = reinterpret_cast<const TcState*>(c->tc_state);
  if (!st) return cudaErrorNotSupported;
  TcParams p;
  p.wait_ns = c->wait_ns;
  p.row_len = c->row_len;
  p.span = span_of(c->spans, SPAN_DECODE);
  p.map = row_map(c);
  p.r_k = d.rank_k;
  p.r_v = d.rank_v;
  p.ck = (d.rank_k + 127) / 128;
  p.cv = (d.rank_v + 127) / 128;
  p.kb_k = (d.rank_k + 63) / 64;
  p.tmem_cols = tmem_cols_for(d.rank_v);
  const bool pair = tc_ctas_per_sm(&d, c->hist_len, c->num_sms) == 2;
  p.Hq = d.n_q_heads;
  p.hist_len = c->hist_len;
  p.stable_len = std::min(c->stable_len, c->hist_len);
  p.split_tokens = split_tokens;
  p.n_splits = n_splits;
  p.nslot = pair ? st->nslot_pair : st->nslot_single;
  p.q_bytes = q_bytes_for(d.rank_k);
  p.part_o = c->part_o;
  p.part_ml = c->part_ml;
  p.err = c->dev_err;
  p.trace = c->trace;
  static std::atomic<uint32_t> optin_done{0};
  cudaError_t e = smem_optin(k_decode_tc, optin_done);
  if (e != cudaSuccess) return e;
  return launch_pdl(k_decode_tc, dim3(n_splits, d.batch), dim3(kThreads), pair ? st->smem_pair : st->smem_single, s,
                    st->q, st->zk, st->zv, p);
}
