// Tensor-core (tcgen05) split-sequence decode over int4 group-quantised latents.
//
// Method: TraceKV abstract (latent KV states stored with quantization, "optimized
// low-rank attention kernels").  Attention runs in rank space, as in the bf16 kernel:
//   S[t, j]  = z^_k,t . q~_j            GEMM1: M = 128 tokens, N = 32 heads, K = r_k
//   p[t, j]  = exp2(S[t, j] - m_j)      online softmax, lazy running max
//   O~[e, j] += sum_t z^_v,t[e] p[t, j]  GEMM2: M = 128 ranks per chunk, N = 32, K = 128 tokens
// where z^ = code * scale + zero is expanded in shared memory to fp16 (one rounding of
// the exact fused product-sum) and q~, p enter the MMAs as fp16 (11 significant bits,
// so neither needs the hi/lo split of the bf16 kernel).
//
// Data flow.  The cache stores int4 latents in 128-token blocks, group-major inside a
// block, so the codes and the {scale, zero} words of one side (K or V) of one tile are
// two contiguous runs (G x 2 KB and G x 512 B).  The producer (warp 0) moves each with
// one plain bulk copy into a ring of raw slots (per-SM copy throughput grows with the
// copy size; 2-10 KB copies from one stream fall well short of HBM bandwidth).  Eight
// dequantisation warps (thread = token row x half chunk) expand each 128-rank chunk
// (4 groups) of a raw slot into a 32 KB operand slot
// (128 tokens x 128 ranks, fp16, the 128-byte-swizzled K-major layout that GEMM1 reads
// as A and GEMM2 reads MN-major); lanes walk consecutive tokens, so their shared-memory
// reads and swizzled writes are free of bank conflicts.  Warp 1 owns TMEM and issues
// the MMAs from one thread.  Four softmax warps (thread = token row = TMEM lane) turn
// scores into probabilities and finish with the epilogue (thread = rank row).
//
// Pipeline.  Operand slots, raw slots and MMAs all follow the order
//   K(0), K(1), V(0), K(2), V(1), ..., K(n-1), V(n-2), V(n-1)
// so GEMM1 of tile s+1 runs while the softmax of tile s is still working: the scores
// and the probabilities are double-buffered (S in two TMEM column blocks, P in two
// shared-memory buffers).  When the running max of a head grows by more than 2^8 the
// softmax first waits for the value mix of the previous tile and rescales O~ in TMEM.
//
// Nibble order.  A code word holds elements m = 0..7 of an 8-rank run at bits 4m.  Two
// masks and one shift give the four fp16 pairs (m0,m4) (m1,m5) (m2,m6) (m3,m7) through
// the exponent-bias trick (0x6400 | n is 1024 + n; 0x5400 | 16n is 64 + n), so each run
// sits in shared memory in the order 0,4,1,5,2,6,3,7.  The query latents are stored in
// the same order (a score is an order-free sum over ranks), and the epilogue maps the
// rows of O~ back to rank order.
//
// Keys stored before the rotary embedding (kRope).  The score needs the rotated key,
// which has no rank-space form, so each tile's keys are rebuilt on the tensor cores:
//   K^_h[t, :] = z^_k,t B_k,h          GEMM0: M = 128 tokens, N = d = 128, K = r_k
// then rotated (rotate-half RoPE at the token's absolute position, cos / sin from the
// cache's fp64-derived table) and dotted with the raw query rows on CUDA cores by the
// softmax warps (thread = token row).  K^ for all four KV heads would need all of TMEM,
// so a CTA covers a pair of KV heads (grid x), query slots 16 h + jj for query head jj
// of pair head h; both CTAs of a pair dequantise the same tiles.  B_k enters as an fp16
// copy, [D rows][ranks] with each 8-rank run in the dequantised order, streamed per
// 64-rank sub-block (both heads' rows, one N = 256 MMA per 16 ranks) by TMA from a spare
// warp (warp 2) through a ring of up to four slots.  The rotation factors of a row are
// fetched one 16-pair chunk ahead (the next tile's first chunk during the last one), so
// their L2 latency stays off the chain rebuild -> rotate -> rebuild.  The value mix and
// the epilogue are those of the rank-space kernel with 32 slots.
//
// Every wait is bounded: on timeout the kernel records LR_ERR_TIMEOUT, drains its own
// copies and MMAs, frees TMEM and returns.
#include "tc_common.cuh"

#include <algorithm>

namespace {

using tc::drain_wait;
using tc::kLazy;
using tc::kSmemLimit;
using tc::kTile;
using tc::kTraceSlots;
using tc::warp_reduce_scatter32;

// 16 warps in four warpgroups: [producer, MMA, 2 idle] [4 softmax] [dequantisation x 8].
// A warp runs on sub-partition (warp % 4).  A single thread issuing N = 32 MMAs slows
// about fivefold when three ALU-bound warps share its sub-partition; with the producer,
// MMA and two idle warps in the first warpgroup, the MMA warp (1) shares sub-partition 1
// with one softmax warp and two dequantisation warps.  Measured against leaving those two
// dequantisation warps idle, the extra dequantisation throughput wins by ~3 %.  Launched
// at 128 registers per thread; the warpgroups then rebalance the block's 64K registers
// with setmaxnreg (the softmax keeps 32 scores and 32 running sums per row).
constexpr int kThreads = 512;
constexpr int kDqWarp0 = 8;                // first warp of the dequantisation warpgroups
constexpr int kDqThreads = 256;            // eight working dequantisation warps
constexpr int kDqWarps = 8;                // arrivals per operand slot / raw slot (one per warp)
constexpr int kSmWarps = 4;                // softmax warps (one arrival each)
constexpr int kLaunchRegs = 128;
constexpr int kRegsCtl = 56, kRegsSoftmax = 208, kRegsDq = 104;
constexpr int kRegsSoftmaxRope = 216;      // keys before RoPE: rotation and query dots too
static_assert(128 * kRegsCtl + 128 * kRegsSoftmax + 256 * kRegsDq <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
static_assert(128 * kRegsCtl + 128 * kRegsSoftmaxRope + 256 * kRegsDq <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kSubBytes = 128 * 128;       // 128 tokens x 64 ranks x 2 B
constexpr int kSlotBytes = 2 * kSubBytes;  // 128 tokens x 128 ranks
constexpr int kQRows = 32;                 // query heads, padded
constexpr int kQSubBytes = kQRows * 128;   // 32 rows x 64 ranks x 2 B
constexpr int kPBytes = 128 * 32 * 2;      // 128 tokens x 32 heads x 2 B
constexpr int kAuxBytes = 2048;
constexpr int kSCol = 0;                   // TMEM: S of tile s in columns [32 (s % 2), +32)
constexpr int kOCol = 64;                  // TMEM: O~ chunk c in columns [64 + 32c, +32)
constexpr int kMaxSlots = 4;
// keys before RoPE
constexpr int kRD = 128;                   // head dim of the rebuilt keys
constexpr int kGHMax = 2;                  // KV heads per CTA (K^ of both fills 256 columns)
constexpr int kMaxG = 32 / kGHMax;         // query slots per KV head
constexpr int kOColR = 256;                // TMEM: O~ chunk c in columns [256 + 32c, +32)
constexpr int kRopeG = 7;                  // query heads per KV head of the instantiated variant
constexpr int kNBMax = 4;                  // B_k ring slots (kv heads x 128 rows x 64 ranks, fp16)
constexpr int kMaxRaw = 6;                 // raw slot: one side of one tile, codes (G x 2 KB)
                                           // then {scale, zero} words (G x 512 B)

struct I4Params {
  const uint32_t* codes_k;
  const uint32_t* codes_v;
  const uint32_t* params_k;
  const uint32_t* params_v;
  long long cap;
  int r_k, r_v, G_k, G_v, ck, cv, kb_k, tmem_cols;
  int Hq, hist_len, stable_len, split_tokens, n_splits, nslot, nraw;
  uint32_t q_bytes, raw_bytes, raw_params;   // raw slot size; offset of its params
  float* part_o;
  float* part_ml;
  int* err;
  unsigned long long* trace;
  // keys before RoPE
  const float* qf;          // [B][Hq][d] scaled queries, fp32
  const float2* rope_cs;    // [capacity][d / 2] (cos, sin)
  int gh, gsz;              // KV heads per CTA, query heads per KV head
  uint32_t q_load_bytes;    // gh * gsz * d * 4
  int nb;                   // B_k ring slots of gh * 16 KB
};

// Barriers (arrival count; who arrives -> who waits).  Every ring is used in the unit order
// K(0), K(1), V(0), K(2), ..., and phase k of a barrier is waited with parity k & 1.
//   raw_full[nraw]    1 + tx   producer's two bulk copies -> dequantisation warps
//   raw_empty[nraw]   8        dequantisation warps -> producer
//   slot_full[nslot]  8        dequantisation warps (fenced stores) -> MMA issuer
//   slot_empty[nslot] 1        MMA commit -> dequantisation warps
//   q_full            1 + tx   producer (after the grid-dependency wait) -> MMA issuer, or
//                              the softmax warps for keys before RoPE
//   s_full[2]         1        MMA commit of GEMM1 -> softmax warps
//   s_empty[2]        4        softmax warps (scores read) -> MMA issuer
//   p_full[2]         4        softmax warps (fenced P stores) -> MMA issuer
//   p_empty[2]        1        MMA commit of GEMM2 -> softmax warps (P reuse, O~ rescale)
//   o_final           1        MMA commit after the last unit -> softmax warps (epilogue)
//   keys before RoPE, in place of s_full / s_empty:
//   k_full            1        MMA commit of GEMM0 -> softmax warps
//   k_empty           4        softmax warps (K^ read) -> MMA issuer (next GEMM0)
//   b_full[nb]        1 + tx   B_k producer (warp 2) -> MMA issuer
//   b_empty[nb]       1        MMA commit -> B_k producer
struct Aux {
  uint64_t slot_full[kMaxSlots];
  uint64_t slot_empty[kMaxSlots];
  uint64_t raw_full[kMaxRaw];
  uint64_t raw_empty[kMaxRaw];
  uint64_t s_full[2], s_empty[2], p_full[2], p_empty[2];
  uint64_t q_full, o_final;
  uint64_t k_full, k_empty, b_full[kNBMax], b_empty[kNBMax];
  uint32_t tmem_base;
  int abort_flag;
  float red[4][32];
  float m_s[32];
  float alpha_s[32];
};
static_assert(sizeof(Aux) <= kAuxBytes, "aux block");

struct I4State {
  CUtensorMap q;
  CUtensorMap bk;           // keys before RoPE: fp16 B_k [D][r_pad], rank runs permuted
  void* bk16 = nullptr;
  int r_pad = 0;
  int nslot, nraw, nb = 0;
  uint32_t raw_bytes, raw_params, q_bytes;
  size_t smem;
};

__device__ __forceinline__ bool wait_b(uint64_t* bar, uint32_t parity, Aux* aux, int* err) {
  return tc::wait_b(bar, parity, &aux->abort_flag, err);
}

// Eight int4 codes of one word -> four fp16 pairs (m0,m4) (m1,m5) (m2,m6) (m3,m7) of
// code * scale + zero; s2 = (scale, scale), z2 = (zero, zero).
__device__ __forceinline__ uint4 dequant8(uint32_t w, uint32_t s2, uint32_t z2) {
  const uint32_t a = (w & 0x000F000Fu) | 0x64006400u;   // 1024 + n
  const uint32_t b = (w & 0x00F000F0u) | 0x54005400u;   // 64 + n
  const uint32_t w8 = w >> 8;
  const uint32_t c = (w8 & 0x000F000Fu) | 0x64006400u;
  const uint32_t d = (w8 & 0x00F000F0u) | 0x54005400u;
  uint4 r;
  asm("{\n\t.reg .b32 t;\n\t"
      "sub.rn.f16x2 t, %1, %2;\n\t"
      "fma.rn.f16x2 %0, t, %3, %4;\n\t}"
      : "=r"(r.x)
      : "r"(a), "r"(0x64006400u), "r"(s2), "r"(z2));
  asm("{\n\t.reg .b32 t;\n\t"
      "sub.rn.f16x2 t, %1, %2;\n\t"
      "fma.rn.f16x2 %0, t, %3, %4;\n\t}"
      : "=r"(r.y)
      : "r"(b), "r"(0x54005400u), "r"(s2), "r"(z2));
  asm("{\n\t.reg .b32 t;\n\t"
      "sub.rn.f16x2 t, %1, %2;\n\t"
      "fma.rn.f16x2 %0, t, %3, %4;\n\t}"
      : "=r"(r.z)
      : "r"(c), "r"(0x64006400u), "r"(s2), "r"(z2));
  asm("{\n\t.reg .b32 t;\n\t"
      "sub.rn.f16x2 t, %1, %2;\n\t"
      "fma.rn.f16x2 %0, t, %3, %4;\n\t}"
      : "=r"(r.w)
      : "r"(d), "r"(0x54005400u), "r"(s2), "r"(z2));
  return r;
}

__device__ __forceinline__ void sts128(uint32_t addr, const uint4& v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Two fp32 lanes in one 64-bit register for the paired FMA: d = a * b + c per lane,
// each rounded once (IEEE fma).
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float lo2(uint64_t v) { return __uint_as_float((uint32_t)v); }
__device__ __forceinline__ float hi2(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// Shared memory: [aux 2 KB][q~ per 64-rank sub-block | fp32 query rows (kRope)]
//                [B_k ring nb x gh x 16 KB (kRope)][operand ring nslot x 32 KB]
//                [P double buffer 2 x 8 KB][raw ring nraw x raw_bytes]
// kG: query heads per KV head (compile time for the keys-before-RoPE dots, so that the
// kG accumulation chains interleave; 0 for the rank-space kernel).  A runtime count with a
// guard inside the unrolled loop serialised the chains (13 us per tile instead of 7).
template <bool kRope, int kG>
__global__ void __launch_bounds__(kThreads, 1)
    k_decode_tc_i4(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_b,
                   const I4Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (ptx::smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicExch(p.err, (int)LR_ERR_UNSUPPORTED);
    return;
  }
  Aux* aux = reinterpret_cast<Aux*>(smem_raw);
  uint8_t* q_s = smem_raw + kAuxBytes;
  uint8_t* bring = q_s + p.q_bytes;
  const uint32_t b_slot_bytes = kRope ? (uint32_t)(p.gh * kSubBytes) : 0u;
  uint8_t* ring = bring + (kRope ? p.nb * b_slot_bytes : 0);
  uint8_t* p_s = ring + p.nslot * kSlotBytes;
  uint8_t* raw = p_s + 2 * kPBytes;
  constexpr int kOC = kRope ? kOColR : kOCol;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = kRope ? (int)blockIdx.x : 0;
  const int split = kRope ? blockIdx.y : blockIdx.x, b = kRope ? blockIdx.z : blockIdx.y;
  const int tok_begin = split * p.split_tokens;
  const int tok_end = min(p.hist_len, tok_begin + p.split_tokens);
  const int ntiles = tok_end > tok_begin ? (tok_end - tok_begin + kTile - 1) / kTile : 0;
  const int nunits = 2 * ntiles;

  if (threadIdx.x == 0) {
    tc::trace_stamp(p.trace, 0);
    for (int s = 0; s < p.nslot; ++s) {
      ptx::mbar_init(&aux->slot_full[s], kDqWarps);
      ptx::mbar_init(&aux->slot_empty[s], 1);
    }
    for (int s = 0; s < p.nraw; ++s) {
      ptx::mbar_init(&aux->raw_full[s], 1);
      ptx::mbar_init(&aux->raw_empty[s], kDqWarps);
    }
    for (int k = 0; k < 2; ++k) {
      ptx::mbar_init(&aux->s_full[k], 1);
      ptx::mbar_init(&aux->s_empty[k], kSmWarps);
      ptx::mbar_init(&aux->p_full[k], kSmWarps);
      ptx::mbar_init(&aux->p_empty[k], 1);
    }
    ptx::mbar_init(&aux->q_full, 1);
    ptx::mbar_init(&aux->o_final, 1);
    if (kRope) {
      ptx::mbar_init(&aux->k_full, 1);
      ptx::mbar_init(&aux->k_empty, kSmWarps);
      for (int k = 0; k < p.nb; ++k) {
        ptx::mbar_init(&aux->b_full[k], 1);
        ptx::mbar_init(&aux->b_empty[k], 1);
      }
    }
    aux->abort_flag = 0;
    for (int j = 0; j < 32; ++j) aux->m_s[j] = -INFINITY;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0 && !kRope) ptx::prefetch_tmap(&tm_q);
  if (warp == 2 && lane == 0 && kRope) ptx::prefetch_tmap(&tm_b);
  if (warp == 1) {
    ptx::tmem_alloc(&aux->tmem_base, p.tmem_cols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = aux->tmem_base;
  // Only the producer reads memory that the preceding kernel writes (the query latents,
  // rows at or above stable_len); it waits for that kernel before those copies.  Every
  // other thread works on shared memory and TMEM behind the producer's barriers, and
  // the epilogue's writes follow the query latents' arrival.
  pdl_trigger();
  if (threadIdx.x == 32) tc::trace_stamp(p.trace, 1);

  // Roles by warpgroup; each sets its register budget first thing in its own branch,
  // so the compiler allocates that branch within the budget.
  if (warp < 4) {
    ptx::setmaxnreg_dec<kRegsCtl>();
    if (warp == 0) {
      // ------------------------------------------------------------- bulk-copy producer
      if (lane == 0 && ntiles > 0) {
        // the query rows: q~ (fp16, by TMA) or, for keys before RoPE, the pair's fp32 rows
        auto load_query = [&]() {
          if (kRope) {
            ptx::mbar_arrive_expect_tx(&aux->q_full, p.q_load_bytes);
            ptx::bulk_load(q_s, p.qf + ((size_t)b * p.Hq + (size_t)pair * p.gh * p.gsz) * kRD, p.q_load_bytes,
                           &aux->q_full);
          } else {
            ptx::mbar_arrive_expect_tx(&aux->q_full, p.q_bytes);
            for (int sb = 0; sb < p.kb_k; ++sb)
              ptx::tma_load_2d(q_s + sb * kQSubBytes, &tm_q, &aux->q_full, sb * 64, b * kQRows);
          }
        };
        bool waited = false, ok = true;
        int issued = 0;
        for (int u = 0; u < nunits && ok; ++u) {
          int tile;
          bool is_v;
          tc::unit_of(u, ntiles, &tile, &is_v);
          const int t0 = tok_begin + tile * kTile;
          const int n = min(kTile, tok_end - t0);
          const int rs = u % p.nraw, round = u / p.nraw;
          if (!waited && (round > 0 || t0 + n > p.stable_len)) {
            pdl_wait();
            load_query();
            waited = true;
          }
          if (round > 0 && !(ok = wait_b(&aux->raw_empty[rs], (round - 1) & 1, aux, p.err))) break;
          const int G = is_v ? p.G_v : p.G_k;
          const long long row0 = (long long)b * p.cap + t0;
          uint8_t* dst = raw + rs * p.raw_bytes;
          ptx::mbar_arrive_expect_tx(&aux->raw_full[rs], (uint32_t)G * 2560u);
          ptx::bulk_load(dst, (is_v ? p.codes_v : p.codes_k) + i4_code_index(row0, G, 0, 0), (uint32_t)G * 2048u,
                         &aux->raw_full[rs]);
          ptx::bulk_load(dst + p.raw_params, (is_v ? p.params_v : p.params_k) + i4_param_index(row0, G, 0),
                         (uint32_t)G * 512u, &aux->raw_full[rs]);
          issued = u + 1;
        }
        if (!waited) {
          pdl_wait();
          load_query();
        }
        if (!ok) {
          drain_wait(&aux->q_full, 0);
          for (int k = max(0, issued - p.nraw); k < issued; ++k)
            drain_wait(&aux->raw_full[k % p.nraw], (k / p.nraw) & 1);
        }
      }
    } else if (kRope && warp == 2) {
      // ------------------------------------------------------------- B_k producer (kRope)
      // (tile, 64-rank sub-block) in the MMA's order, one box of the pair's gh x 128 rows;
      // B_k is written before the cache is used, so no grid-dependency wait is needed.
      if (lane == 0 && ntiles > 0) {
        const int total = ntiles * p.kb_k;
        bool ok = true;
        int issued = 0;
        for (int k = 0; k < total; ++k) {
          const int slot = k % p.nb;
          if (k >= p.nb && !(ok = wait_b(&aux->b_empty[slot], ((k / p.nb) - 1) & 1, aux, p.err))) break;
          const int sb = k % p.kb_k;
          ptx::mbar_arrive_expect_tx(&aux->b_full[slot], b_slot_bytes);
          ptx::tma_load_2d(bring + slot * b_slot_bytes, &tm_b, &aux->b_full[slot], sb * 64, pair * p.gh * kRD);
          issued = k + 1;
        }
        if (!ok)
          for (int k = max(0, issued - p.nb); k < issued; ++k) drain_wait(&aux->b_full[k % p.nb], (k / p.nb) & 1);
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------- MMA issuer
      if (lane == 0 && ntiles > 0) {
        const uint32_t id = ptx::idesc_f16(0, 0, 0, 128, 32);    // GEMM1: fp16, K-major x K-major
        const uint32_t id2 = ptx::idesc_f16(0, 1, 1, 128, 32);   // GEMM2: fp16, MN-major x MN-major
        // Descriptors are built once; a step along K or to another slot adds its byte
        // offset >> 4 to the start-address field (shared-memory addresses stay below
        // 256 KB, so the 14-bit field never carries).
        const uint64_t kdesc0 = ptx::smem_desc(ptx::smem_u32(ring), 16, 1024, 2);       // Z_k, K-major SW128
        const uint64_t qdesc0 = ptx::smem_desc(ptx::smem_u32(q_s), 16, 1024, 2);        // q~, K-major SW128
        const uint64_t vdesc0 = ptx::smem_desc(ptx::smem_u32(ring), kSubBytes, 1024, 2); // Z_v, MN-major SW128
        const uint64_t pdesc0 = ptx::smem_desc(ptx::smem_u32(p_s), 128, 2048, 0);       // P, MN-major
        const uint32_t idk = ptx::idesc_f16(0, 0, 0, 128, kRope ? p.gh * kRD : 128);   // GEMM0 (kRope)
        const uint64_t bdesc0 = ptx::smem_desc(ptx::smem_u32(bring), 16, 1024, 2);      // B_k, K-major SW128
        bool ok = kRope ? true : wait_b(&aux->q_full, 0, aux, p.err);
        ptx::tc_fence_after();
        tc::trace_stamp(p.trace, 2);
        int pos = 0, bpos = 0;
        for (int u = 0; u < nunits && ok; ++u) {
          int tile;
          bool is_v;
          tc::unit_of(u, ntiles, &tile, &is_v);
          if (kRope && !is_v) {
            // GEMM0(tile): [K^_0 | K^_1] = Z_k [B_k,0 | B_k,1], columns [128 h, +128) per head
            if (tile >= 1 && !(ok = wait_b(&aux->k_empty, (tile - 1) & 1, aux, p.err))) break;
            ptx::tc_fence_after();
            for (int c = 0; c < p.ck && ok; ++c, ++pos) {
              const int slot = pos % p.nslot;
              if (!(ok = wait_b(&aux->slot_full[slot], (pos / p.nslot) & 1, aux, p.err))) break;
              ptx::tc_fence_after();
              const uint64_t a0 = kdesc0 + (uint64_t)((slot * kSlotBytes) >> 4);
              for (int sb = 0; sb < 2 && c * 128 + sb * 64 < p.r_k; ++sb, ++bpos) {
                const int bs = bpos % p.nb;
                if (!(ok = wait_b(&aux->b_full[bs], (bpos / p.nb) & 1, aux, p.err))) break;
                ptx::tc_fence_after();
                const uint64_t b0 = bdesc0 + (uint64_t)((bs * b_slot_bytes) >> 4);
                // sub-block sb of the A slot (16 KB) against the B slot; 32 bytes per step
                const int nk = min(4, (p.r_k - c * 128 - sb * 64) >> 4);
                for (int kk = 0; kk < nk; ++kk)
                  ptx::mma_f16(tmem, a0 + (uint64_t)(sb * (kSubBytes >> 4) + kk * 2), b0 + (uint64_t)(kk * 2), idk,
                               (c | sb | kk) ? 1u : 0u);
                ptx::mma_commit(&aux->b_empty[bs]);
              }
              if (!ok) break;
              ptx::mma_commit(&aux->slot_empty[slot]);
            }
            if (!ok) break;
            ptx::mma_commit(&aux->k_full);
            if (tile < 16) tc::trace_stamp(p.trace, 3 + 4 * tile);
          } else if (!is_v) {
            // GEMM1(tile): S[tile % 2] = Z_k q~^T
            const int sb2 = tile & 1;
            if (tile >= 2 && !(ok = wait_b(&aux->s_empty[sb2], ((tile - 2) >> 1) & 1, aux, p.err))) break;
            ptx::tc_fence_after();
            const uint32_t d_s = tmem + kSCol + 32 * sb2;
            for (int c = 0; c < p.ck && ok; ++c, ++pos) {
              const int slot = pos % p.nslot;
              if (!(ok = wait_b(&aux->slot_full[slot], (pos / p.nslot) & 1, aux, p.err))) break;
              ptx::tc_fence_after();
              const uint64_t a0 = kdesc0 + (uint64_t)((slot * kSlotBytes) >> 4);
              const uint64_t b0 = qdesc0 + (uint64_t)((c * 2 * kQSubBytes) >> 4);
              const int nk = min(8, (p.r_k - c * 128) >> 4);     // 16-rank K steps in this chunk
              // step kk: sub-block kk / 4 (16 KB on A, 4 KB on B), 32 bytes per step within it
              for (int kk = 0; kk < nk; ++kk) {
                const uint32_t ao = (uint32_t)((kk >> 2) * (kSubBytes >> 4) + (kk & 3) * 2);
                const uint32_t bo = (uint32_t)((kk >> 2) * (kQSubBytes >> 4) + (kk & 3) * 2);
                ptx::mma_f16(d_s, a0 + ao, b0 + bo, id, (c | kk) ? 1u : 0u);
              }
              ptx::mma_commit(&aux->slot_empty[slot]);
            }
            if (!ok) break;
            ptx::mma_commit(&aux->s_full[sb2]);
            if (tile < 16) tc::trace_stamp(p.trace, 3 + 4 * tile);
          } else {
            // GEMM2(tile): O~ += Z_v^T P[tile % 2]
            const int pb2 = tile & 1;
            if (!(ok = wait_b(&aux->p_full[pb2], (tile >> 1) & 1, aux, p.err))) break;
            ptx::tc_fence_after();
            const uint64_t b0 = pdesc0 + (uint64_t)((pb2 * kPBytes) >> 4);
            for (int c = 0; c < p.cv && ok; ++c, ++pos) {
              const int slot = pos % p.nslot;
              if (!(ok = wait_b(&aux->slot_full[slot], (pos / p.nslot) & 1, aux, p.err))) break;
              ptx::tc_fence_after();
              const uint64_t a0 = vdesc0 + (uint64_t)((slot * kSlotBytes) >> 4);
              const uint32_t d_o = tmem + kOC + c * 32;
              // K step kt = 16 tokens: 2 KB on A (16 swizzled rows), 256 B on P
#pragma unroll
              for (int kt = 0; kt < 8; ++kt)
                ptx::mma_f16(d_o, a0 + (uint64_t)(kt * 128), b0 + (uint64_t)(kt * 16), id2, (tile | kt) ? 1u : 0u);
              ptx::mma_commit(&aux->slot_empty[slot]);
            }
            if (!ok) break;
            ptx::mma_commit(&aux->p_empty[pb2]);
            if (tile < 16) tc::trace_stamp(p.trace, 6 + 4 * tile);
          }
        }
        ptx::mma_commit(&aux->o_final);
        if (!ok) drain_wait(&aux->o_final, 0);
      }
      __syncwarp();
    }
  } else if (warp < kDqWarp0) {
    ptx::setmaxnreg_inc<kRope ? kRegsSoftmaxRope : kRegsSoftmax>();
    if (ntiles > 0) {
      // ------------------------------------------------------------- softmax / epilogue
      const int qd = warp & 3;
      const int row = qd * 32 + lane;
      const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
      float l[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) l[j] = 0.f;
      bool ok = true;
      // keys before RoPE: the query rows are read here, from shared memory
      if (kRope) ok = ptx::named_bar_and(1, 128, wait_b(&aux->q_full, 0, aux, p.err));
      const float* q_f = reinterpret_cast<const float*>(q_s);
      // rotation factors: cs holds the chunk in use, csn the one after it
      float cs[32], csn[32];
      auto load_cs = [&](float(&dst)[32], int tile_i, int c0) {
        const int t = tok_begin + tile_i * kTile + row;
        const float2* src = p.rope_cs + (size_t)(t < tok_end ? t : tok_begin) * (kRD / 2) + c0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 v = __ldg(reinterpret_cast<const float4*>(src) + k);
          dst[4 * k] = v.x;
          dst[4 * k + 1] = v.y;
          dst[4 * k + 2] = v.z;
          dst[4 * k + 3] = v.w;
        }
      };
      if (kRope) load_cs(cs, 0, 0);
      for (int i = 0; i < ntiles && ok; ++i) {
        const int k2 = i & 1;
        const bool valid = tok_begin + i * kTile + row < tok_end;
        const uint32_t s_col = tmem + lane_off + kSCol + 32 * k2;
        float s[32];
        if (kRope) {
          ok = ptx::named_bar_and(1, 128, wait_b(&aux->k_full, i & 1, aux, p.err));
          if (!ok) break;
          ptx::tc_fence_after();
          if (i < 16 && threadIdx.x == 128) tc::trace_stamp(p.trace, 4 + 4 * i);
          // score of query slot 16 h + jj: q_jj . RoPE_t(K^_h[t]), pairs (c, c + 64)
#pragma unroll
          for (int j = 0; j < 32; ++j) s[j] = 0.f;
#pragma unroll 1
          for (int c0 = 0; c0 < kRD / 2; c0 += 16) {
            if (c0 + 16 < kRD / 2) load_cs(csn, i, c0 + 16);
            else if (i + 1 < ntiles) load_cs(csn, i + 1, 0);
#pragma unroll
            for (int h = 0; h < kGHMax; ++h) {
              if (h < p.gh) {
                uint32_t x1[16], x2[16];
                ptx::tmem_ld16(tmem + lane_off + h * kRD + c0, x1);
                ptx::tmem_ld16(tmem + lane_off + h * kRD + kRD / 2 + c0, x2);
                ptx::tmem_wait_ld();
                float r1[16], r2[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                  const float a = __uint_as_float(x1[k]), e = __uint_as_float(x2[k]);
                  r1[k] = a * cs[2 * k] - e * cs[2 * k + 1];
                  r2[k] = e * cs[2 * k] + a * cs[2 * k + 1];
                }
                // paired fp32 FMAs over adjacent elements (two partial sums per score,
                // folded at the end of the chunk)
                uint64_t acc[kG > 0 ? kG : 1];
#pragma unroll
                for (int jj = 0; jj < kG; ++jj) acc[jj] = pack2(s[h * kMaxG + jj], 0.f);
#pragma unroll
                for (int k = 0; k < 16; k += 4) {
                  const uint64_t ra = pack2(r1[k], r1[k + 1]), rb = pack2(r1[k + 2], r1[k + 3]);
                  const uint64_t rc = pack2(r2[k], r2[k + 1]), rd = pack2(r2[k + 2], r2[k + 3]);
#pragma unroll
                  for (int jj = 0; jj < kG; ++jj) {
                    const float* qr = q_f + (size_t)(h * kG + jj) * kRD + c0 + k;
                    const float4 qa = *reinterpret_cast<const float4*>(qr);
                    const float4 qb = *reinterpret_cast<const float4*>(qr + kRD / 2);
                    acc[jj] = ffma2(pack2(qa.x, qa.y), ra, acc[jj]);
                    acc[jj] = ffma2(pack2(qa.z, qa.w), rb, acc[jj]);
                    acc[jj] = ffma2(pack2(qb.x, qb.y), rc, acc[jj]);
                    acc[jj] = ffma2(pack2(qb.z, qb.w), rd, acc[jj]);
                  }
                }
#pragma unroll
                for (int jj = 0; jj < kG; ++jj) s[h * kMaxG + jj] = lo2(acc[jj]) + hi2(acc[jj]);
              }
            }
#pragma unroll
            for (int k = 0; k < 32; ++k) cs[k] = csn[k];
          }
          // K^ has been read: GEMM0 of the next tile may overwrite it
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&aux->k_empty);
          if (!valid) {
#pragma unroll
            for (int j = 0; j < 32; ++j) s[j] = -INFINITY;
          }
        } else {
          ok = ptx::named_bar_and(1, 128, wait_b(&aux->s_full[k2], (i >> 1) & 1, aux, p.err));
          if (!ok) break;
          ptx::tc_fence_after();
          if (i < 16 && threadIdx.x == 128) tc::trace_stamp(p.trace, 4 + 4 * i);
          uint32_t sv[32];
          ptx::tmem_ld32(s_col, sv);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) s[j] = valid ? __uint_as_float(sv[j]) : -INFINITY;
        }

        bool ex = false;
#pragma unroll
        for (int j = 0; j < 32; ++j) ex |= s[j] > aux->m_s[j] + kLazy;
        ex = ptx::named_bar_or(1, 128, ex);
        if (ex) {
          // the value mix of the previous tile must be complete before O~ is rescaled
          if (i >= 1) {
            ok = ptx::named_bar_and(1, 128, wait_b(&aux->p_empty[(i - 1) & 1], ((i - 1) >> 1) & 1, aux, p.err));
            if (!ok) break;
            ptx::tc_fence_after();
          }
          if (kRope) {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = s[j];
            aux->red[qd][lane] = warp_reduce_scatter32<true>(v, lane);
          } else {
            // the reduction consumes s; it is read again from TMEM
            aux->red[qd][lane] = warp_reduce_scatter32<true>(s, lane);
            uint32_t sv[32];
            ptx::tmem_ld32(s_col, sv);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) s[j] = valid ? __uint_as_float(sv[j]) : -INFINITY;
          }
          ptx::named_bar_sync(1, 128);
          if (qd == 0) {
            const float mt =
                fmaxf(fmaxf(aux->red[0][lane], aux->red[1][lane]), fmaxf(aux->red[2][lane], aux->red[3][lane]));
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
            for (int c = 0; c < p.cv; ++c) {
              uint32_t v2[32];
              ptx::tmem_ld32(tmem + lane_off + kOC + c * 32, v2);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j) v2[j] = __float_as_uint(__uint_as_float(v2[j]) * aux->alpha_s[j]);
              ptx::tmem_st32(tmem + lane_off + kOC + c * 32, v2);
            }
            ptx::tmem_wait_st();
          }
        }
        // P[i % 2] is free once the value mix of tile i - 2 has completed
        if (i >= 2) {
          ok = ptx::named_bar_and(1, 128, wait_b(&aux->p_empty[k2], ((i - 2) >> 1) & 1, aux, p.err));
          if (!ok) break;
        }
        // probabilities as fp16; l sums the rounded values the MMA uses
        const uint32_t prow = ptx::smem_u32(p_s + k2 * kPBytes + row * 16);
#pragma unroll
        for (int hg = 0; hg < 4; ++hg) {
          uint32_t hw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = hg * 8 + 2 * e;
            const __half2 h = __floats2half2_rn(exp2f(s[j] - aux->m_s[j]), exp2f(s[j + 1] - aux->m_s[j + 1]));
            const float2 f = __half22float2(h);
            l[j] += f.x;
            l[j + 1] += f.y;
            hw[e] = *reinterpret_cast<const uint32_t*>(&h);
          }
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(prow + hg * 2048), "r"(hw[0]), "r"(hw[1]),
                       "r"(hw[2]), "r"(hw[3])
                       : "memory");
        }
        // every lane makes its own P stores visible to the tensor core, then one arrival
        // per warp
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (!kRope) ptx::mbar_arrive(&aux->s_empty[k2]);
          ptx::mbar_arrive(&aux->p_full[k2]);
        }
        if (i < 16 && threadIdx.x == 128) tc::trace_stamp(p.trace, 5 + 4 * i);
      }
      if (ok) ok = ptx::named_bar_and(1, 128, wait_b(&aux->o_final, 0, aux, p.err));
      if (ok) {
        ptx::tc_fence_after();
        const size_t base_out = ((size_t)b * p.n_splits + split) * p.Hq;
        // TMEM row m of a chunk holds rank 8 (m / 8) + perm(m % 8), perm = 0,4,1,5,2,6,3,7
        const int m = qd * 32 + lane;
        const int e_in = (m & ~7) + ((m & 7) >> 1) + ((m & 1) << 2);
        // query head of slot j (-1: padding)
        auto head_of = [&](int j) -> int {
          if (!kRope) return j < p.Hq ? j : -1;
          const int h = j / kMaxG, jj = j % kMaxG;
          return (h < p.gh && jj < p.gsz) ? (pair * p.gh + h) * p.gsz + jj : -1;
        };
        for (int c = 0; c < p.cv; ++c) {
          uint32_t v2[32];
          ptx::tmem_ld32(tmem + lane_off + kOC + c * 32, v2);
          ptx::tmem_wait_ld();
          const int e = c * 128 + e_in;
          if (e < p.r_v) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int J = head_of(j);
              if (J >= 0) p.part_o[(base_out + J) * p.r_v + e] = __uint_as_float(v2[j]);
            }
          }
        }
        aux->red[qd][lane] = warp_reduce_scatter32<false>(l, lane);
        ptx::named_bar_sync(1, 128);
        const int J = head_of(lane);
        if (qd == 0 && J >= 0) {
          const float lt = (aux->red[0][lane] + aux->red[1][lane]) + (aux->red[2][lane] + aux->red[3][lane]);
          p.part_ml[(base_out + J) * 2] = aux->m_s[lane];
          p.part_ml[(base_out + J) * 2 + 1] = lt;
        }
        if (threadIdx.x == 128) tc::trace_stamp(p.trace, kTraceSlots - 1);
      }
    }
  } else {
    ptx::setmaxnreg_dec<kRegsDq>();
    // ------------------------------------------------------------- dequantisation
    if (ntiles > 0) {
      // warps 8..15 -> dq 0..255; unit v = (token v % 128, group v / 128 of the chunk) for
      // v = dq, dq + 256, ...; lanes walk consecutive tokens
      const int wi = warp - kDqWarp0;      // 0..7
      const bool dq_live = true;
      const int dq = wi * 32 + lane;
      const uint32_t ring_base = ptx::smem_u32(ring);
      bool ok = dq_live;
      int pos = 0;
      for (int u = 0; u < nunits && ok; ++u) {
        int tile;
        bool is_v;
        tc::unit_of(u, ntiles, &tile, &is_v);
        const int nvalid = tok_end - (tok_begin + tile * kTile);   // valid token rows of the tile
        const int G = is_v ? p.G_v : p.G_k;
        const int nch = is_v ? p.cv : p.ck;
        const int rs = u % p.nraw;
        // waits are made warp-uniform: the warp arrives once, after __syncwarp
        if (!(ok = __all_sync(0xffffffffu, wait_b(&aux->raw_full[rs], (u / p.nraw) & 1, aux, p.err)))) break;
        for (int c = 0; c < nch; ++c, ++pos) {
          const int slot = pos % p.nslot;
          if (pos >= p.nslot &&
              !(ok = __all_sync(0xffffffffu, wait_b(&aux->slot_empty[slot], ((pos / p.nslot) - 1) & 1, aux, p.err))))
            break;
          const int ng = min(4, G - 4 * c);
          const uint8_t* rb = raw + rs * p.raw_bytes + c * 8192;          // codes of groups 4c..
          const uint32_t* rp = reinterpret_cast<const uint32_t*>(raw + rs * p.raw_bytes + p.raw_params) + c * 512;
          const uint32_t dst = ring_base + slot * kSlotBytes;
          // up to three units per thread; all loads first, then the arithmetic and stores
          constexpr int kU = (4 * kTile + kDqThreads - 1) / kDqThreads;
          uint4 w[kU];
          uint32_t prm[kU];
#pragma unroll
          for (int k = 0; k < kU; ++k) {
            const int v = dq + k * kDqThreads, t = v & (kTile - 1), gl = v >> 7;
            w[k] = make_uint4(0u, 0u, 0u, 0u);
            prm[k] = 0u;
            if (v < ng * kTile && t < nvalid) {
              w[k] = reinterpret_cast<const uint4*>(rb)[gl * kTile + t];
              prm[k] = rp[gl * kTile + t];
            }
          }
#pragma unroll
          for (int k = 0; k < kU; ++k) {
            const int v = dq + k * kDqThreads, t = v & (kTile - 1), gl = v >> 7, sw = t & 7;
            if (v < ng * kTile) {
              const uint32_t s2 = __byte_perm(prm[k], 0u, 0x1010), z2 = __byte_perm(prm[k], 0u, 0x3232);
              // group gl = ranks 32 gl.. of the chunk: sub-block gl / 2, 16-byte columns 4 (gl % 2)..
              const uint32_t rowa = dst + (gl >> 1) * kSubBytes + t * 128;
              const int cb = (gl & 1) * 4;
              sts128(rowa + (((cb + 0) ^ sw) << 4), dequant8(w[k].x, s2, z2));
              sts128(rowa + (((cb + 1) ^ sw) << 4), dequant8(w[k].y, s2, z2));
              sts128(rowa + (((cb + 2) ^ sw) << 4), dequant8(w[k].z, s2, z2));
              sts128(rowa + (((cb + 3) ^ sw) << 4), dequant8(w[k].w, s2, z2));
            }
          }
          // each lane fences its own stores for the tensor core; one arrival per warp
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&aux->slot_full[slot]);
        }
        __syncwarp();
        if (ok && lane == 0) ptx::mbar_arrive(&aux->raw_empty[rs]);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, p.tmem_cols);
  }
}

// B_k as the fp16 B operand of GEMM0: out[n][pos] = B_k[rank(pos)][n] for the D output
// columns n, where position pos of each 8-rank run holds rank 0,4,1,5,2,6,3,7 (the order
// of the dequantised latents); ranks >= r_k are zero.  bf16 -> fp16 is exact for values
// of magnitude 2^-14 .. 65504.
__global__ void k_prep_bk16(const __nv_bfloat16* Bk, __half* out, int r_k, int r_pad, int D) {
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)D * r_pad) return;
  const int n = (int)(idx / r_pad), pos = (int)(idx % r_pad);
  const int i = (pos & ~7) | ((pos & 1) << 2) | ((pos >> 1) & 3);
  out[idx] = i < r_k ? __float2half_rn(__bfloat162float(Bk[(size_t)i * D + n])) : __float2half_rn(0.f);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------

int q_bytes_for(const lr_cache_desc* d) {
  if (d->rope_in_kernel) {
    const int gh = d->n_kv_heads % 2 == 0 ? 2 : 1;
    const int rows = gh * (d->n_q_heads / d->n_kv_heads);
    return ((rows * kRD * 4 + 1023) / 1024) * 1024;
  }
  return ((d->rank_k + 63) / 64) * kQSubBytes;
}

struct I4Layout {
  int nslot, nraw, nb;
  uint32_t raw_bytes, raw_params;
  size_t smem;
};

// Raw slots hold one side of one tile.  As many operand slots as leave room for two raw
// slots (up to four: the dequantisation can then run a full 128-rank chunk further ahead
// of the MMAs), then as many raw slots (up to 6) as fit in 227 KB.  Keys before RoPE add
// the B_k ring.
bool choose_layout(const lr_cache_desc* d, I4Layout* L) {
  const int G = std::max((d->rank_k + 31) / 32, (d->rank_v + 31) / 32);
  L->raw_params = (uint32_t)G * 2048u;
  L->raw_bytes = (uint32_t)G * 2560u;
  const size_t fixed = (size_t)kAuxBytes + q_bytes_for(d) + 2 * kPBytes;
  if (d->rope_in_kernel) {
    // two operand slots and two raw slots, then B_k slots up to one tile's worth (the next
    // tile's sub-blocks load while the current one is rotated), then raw slots
    const size_t bslot = (size_t)(d->n_kv_heads % 2 == 0 ? 2 : 1) * kSubBytes;
    const int kb = (d->rank_k + 63) / 64;
    const size_t base = fixed + 2 * (size_t)kSlotBytes + 2 * (size_t)L->raw_bytes;
    if (base + 2 * bslot > (size_t)kSmemLimit) return false;
    L->nb = std::min(kNBMax, std::max(2, std::min(kb, (int)(((size_t)kSmemLimit - base) / bslot))));
    L->nslot = 2;
    const size_t used = fixed + (size_t)L->nb * bslot + 2 * (size_t)kSlotBytes;
    L->nraw = std::min(kMaxRaw, (int)(((size_t)kSmemLimit - used) / L->raw_bytes));
    L->smem = used + (size_t)L->nraw * L->raw_bytes;
    return true;
  }
  L->nb = 0;
  for (int ns = kMaxSlots; ns >= 2; --ns) {
    if (fixed + (size_t)ns * kSlotBytes > (size_t)kSmemLimit) continue;
    const int nr =
        std::min(kMaxRaw, (int)(((size_t)kSmemLimit - fixed - (size_t)ns * kSlotBytes) / L->raw_bytes));
    if (nr >= 2) {
      L->nslot = ns;
      L->nraw = nr;
      L->smem = fixed + (size_t)ns * kSlotBytes + (size_t)nr * L->raw_bytes;
      return true;
    }
  }
  return false;
}

int kv_per_cta(const lr_cache_desc* d) {
  if (!d->rope_in_kernel) return d->n_kv_heads;
  return d->n_kv_heads % 2 == 0 ? 2 : 1;
}

}  // namespace

bool tc_i4_supported(const lr_cache_desc* d) {
  if (d->quant_bits != 4 || d->quant_group != 32) return false;
  if (d->dtype != LR_BF16) return false;
  if (d->n_q_heads > 32 || d->rank_v > 512) return false;
  // keys before RoPE: instantiated for the shape the parity tests cover (d = 128, seven
  // query heads per KV head, KV heads in pairs); other shapes take the CUDA-core path
  if (d->rope_in_kernel &&
      (d->head_dim != kRD || d->n_q_heads != kRopeG * d->n_kv_heads || d->n_kv_heads % kGHMax != 0))
    return false;
  I4Layout L;
  return choose_layout(d, &L);
}

int tc_i4_split_ctas(const lr_cache_desc* d) { return d->n_kv_heads / kv_per_cta(d); }

cudaError_t tc_i4_prepare(lr_cache* c, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  I4State* st = reinterpret_cast<I4State*>(c->tc_state);
  if (!st) {
    st = new (std::nothrow) I4State();
    if (!st) return cudaErrorMemoryAllocation;
    c->tc_state = st;
  }
  if (d.rope_in_kernel) {
    const int r_pad = ((d.rank_k + 127) / 128) * 128;
    if (!st->bk16) {
      cudaError_t e = cudaMalloc(&st->bk16, (size_t)c->D * r_pad * 2);
      if (e != cudaSuccess) return e;
      st->r_pad = r_pad;
    }
    const long long n = (long long)c->D * r_pad;
    k_prep_bk16<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(c->B_k),
                                                            reinterpret_cast<__half*>(st->bk16), d.rank_k, r_pad, c->D);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    cuuint64_t dims[2] = {(cuuint64_t)r_pad, (cuuint64_t)c->D};
    cuuint64_t strides[1] = {(cuuint64_t)r_pad * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)(kv_per_cta(&d) * kRD)};
    if (!tc::make_map(&st->bk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, st->bk16, 2, dims, strides, box))
      return cudaErrorInvalidValue;
    st->q = st->bk;   // unused by the kRope kernel
  } else {
    const size_t qbytes = (size_t)d.batch * kQRows * d.rank_k * 2;
    if (!c->qt16) {
      cudaError_t e = cudaMalloc(&c->qt16, qbytes);
      if (e != cudaSuccess) return e;
      e = cudaMemset(c->qt16, 0, qbytes);
      if (e != cudaSuccess) return e;
    }
    cuuint64_t dims[2] = {(cuuint64_t)d.rank_k, (cuuint64_t)d.batch * kQRows};
    cuuint64_t strides[1] = {(cuuint64_t)d.rank_k * 2};
    cuuint32_t box[2] = {64, kQRows};
    if (!tc::make_map(&st->q, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, c->qt16, 2, dims, strides, box))
      return cudaErrorInvalidValue;
    st->bk = st->q;   // unused by the rank-space kernel
  }
  I4Layout L;
  if (!choose_layout(&d, &L)) return cudaErrorNotSupported;
  st->nslot = L.nslot;
  st->nraw = L.nraw;
  st->nb = L.nb;
  st->raw_bytes = L.raw_bytes;
  st->raw_params = L.raw_params;
  st->q_bytes = (uint32_t)q_bytes_for(&d);
  st->smem = L.smem;
  return cudaSuccess;
}

void tc_i4_release(lr_cache* c) {
  I4State* st = reinterpret_cast<I4State*>(c->tc_state);
  if (st && st->bk16) cudaFree(st->bk16);
  delete st;
  c->tc_state = nullptr;
}

cudaError_t launch_decode_tc_i4(const lr_cache* c, int n_splits, int split_tokens, cudaStream_t s) {
  const lr_cache_desc& d = c->desc;
  const I4State* st = reinterpret_cast<const I4State*>(c->tc_state);
  if (!st) return cudaErrorNotSupported;
  const bool rope = d.rope_in_kernel != 0;
  I4Params p;
  p.codes_k = c->codes_k;
  p.codes_v = c->codes_v;
  p.params_k = c->params_k;
  p.params_v = c->params_v;
  p.cap = c->lat_cap;
  p.r_k = d.rank_k;
  p.r_v = d.rank_v;
  p.G_k = c->G_k;
  p.G_v = c->G_v;
  p.ck = (d.rank_k + 127) / 128;
  p.cv = (d.rank_v + 127) / 128;
  p.kb_k = (d.rank_k + 63) / 64;
  p.tmem_cols = rope ? 512 : ((kOCol + p.cv * 32) <= 128 ? 128 : 256);
  p.Hq = d.n_q_heads;
  p.hist_len = c->hist_len;
  p.stable_len = std::min(c->stable_len, c->hist_len);
  p.split_tokens = split_tokens;
  p.n_splits = n_splits;
  p.nslot = st->nslot;
  p.nraw = st->nraw;
  p.q_bytes = st->q_bytes;
  p.raw_bytes = st->raw_bytes;
  p.raw_params = st->raw_params;
  p.part_o = c->part_o;
  p.part_ml = c->part_ml;
  p.err = c->dev_err;
  // the timeline buffer holds S_max CTAs per sequence
  p.trace = n_splits * tc_i4_split_ctas(&d) <= c->S_max ? c->trace : nullptr;
  p.qf = c->qt;
  p.rope_cs = c->rope_cs;
  p.gh = kv_per_cta(&d);
  p.gsz = d.n_q_heads / d.n_kv_heads;
  p.q_load_bytes = (uint32_t)(p.gh * p.gsz * kRD * 4);
  p.nb = st->nb;
  // instantiation: 0 rank space; 1 keys before RoPE
  using Kern = void (*)(CUtensorMap, CUtensorMap, I4Params);
  static const Kern kerns[2] = {k_decode_tc_i4<false, 0>, k_decode_tc_i4<true, kRopeG>};
  if (rope && (p.gsz != kRopeG || p.gh != kGHMax)) return cudaErrorNotSupported;
  const int ki = rope ? 1 : 0;
  const Kern kern = kerns[ki];
  static std::atomic<uint32_t> optin_done[2] = {0, 0};
  cudaError_t e = smem_optin(kern, optin_done[ki]);
  if (e != cudaSuccess) return e;
  // The register rebalancing assumes the launch allocation the split was sized for.
  static std::atomic<int> regs[2] = {0, 0};
  if (regs[ki].load() == 0) {
    cudaFuncAttributes fa;
    regs[ki].store(cudaFuncGetAttributes(&fa, kern) == cudaSuccess ? fa.numRegs : -1);
  }
  if (regs[ki].load() != kLaunchRegs) return cudaErrorInvalidConfiguration;
  const dim3 grid = rope ? dim3(d.n_kv_heads / p.gh, n_splits, d.batch) : dim3(n_splits, d.batch);
  return launch_pdl(kern, grid, dim3(kThreads), st->smem, s, st->q, st->bk, p);
}
