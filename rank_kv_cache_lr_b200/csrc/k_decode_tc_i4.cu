// Tensor-core (tcgen05) split-sequence decode over int4 group-quantised latents.
//
// Method: TraceKV abstract (latent KV states stored with quantization, "optimized
// low-rank attention kernels").  Attention runs in rank space, as in the bf16 kernel:
//   S[t, j]  = z^_k,t . q~_j            GEMM1: M = 128 tokens, N = 32 heads, K = r_k
//   p[t, j]  = exp2(S[t, j] - m_j)      online softmax, lazy running max
//   O~[e, j] += sum_t z^_v,t[e] p[t, j]  GEMM2: M = 128 ranks per chunk, N = 32, K = 128 tokens
// where z^ = code * scale + zero is expanded to fp16 (one rounding of the exact fused
// product-sum) and q~, p enter the MMAs as fp16 (11 significant bits, so neither needs the
// hi/lo split of the bf16 kernel).
//
// Operands in tensor memory.  An M = 128 MMA with N = 32 that reads its A operand (128 x 16
// fp16 = 4 KB) from shared memory is bound by the shared-memory bandwidth (128 B per
// clock): the expanded latents would be written to and read back from shared memory once
// each, 256 KB per 128-token tile at r = 256.  Here the dequantisation warps write the
// expanded latents straight into tensor memory with tcgen05.st, and both GEMMs take their
// A operand from there (A in TMEM: lane = row, column c = K elements 2c, 2c + 1).  Shared
// memory carries only the packed codes (bulk copies), q~ and P.
//   GEMM1 A = z^_k tile: lane = token, K = ranks.  A dequantisation thread owns one token
//     row and expands its code words (keys are stored token-major).
//   GEMM2 A = z^_v chunk transposed: lane = rank, K = tokens.  Values are stored
//     rank-major (see lr_internal.cuh), so a thread owns one rank row and expands eight
//     tokens per word, each pair with its own fp16 {scale, zero}.
// A tcgen05.st reaches only the 32 lanes of the writing warp's sub-partition, so each side
// has four dequantisation warps, one per sub-partition (warp % 4 = lane quarter), each
// expanding all 64 columns of its 32 lanes.
//
// Data flow.  The producer (warp 0) moves the codes and the {scale, zero} words of one side
// (K or V) of one 128-token tile with two plain bulk copies into that side's ring of raw
// slots.  The four key warps expand each 128-rank chunk of a key slot into a 64-column
// operand slot of the key ring in TMEM, the four value warps do the same for the values
// into the value ring.  Warp 1 issues the key-side MMAs and warp 3 the value mix, each from
// one thread.  Four softmax warps (thread = token row = TMEM lane) turn scores into
// probabilities and finish with the epilogue (thread = rank row).
//
// Pipeline.  The producer issues the copies in the order
//   K(0), K(1), V(0), K(2), V(1), ..., K(n-1), V(n-2), V(n-1)
// so the keys of tile s+1 arrive before the values of tile s.  Each side's warps, rings and
// issuer then run on their own: the key side up to two tiles ahead of the softmax (the
// scores and the probabilities are double-buffered: S in two TMEM column blocks, P in two
// shared-memory buffers), the value side behind it, never holding up the keys of the next
// tile while a value chunk waits for its probabilities.  When the running max of a head
// grows by more than 2^8 the softmax first waits for the value mix of the previous tile and
// rescales O~ in TMEM.
//
// Nibble order.  A key code word holds elements m = 0..7 of an 8-rank run at bits 4m.  Two
// masks and one shift give the four fp16 pairs (m0,m4) (m1,m5) (m2,m6) (m3,m7) through
// the exponent-bias trick (0x6400 | n is 1024 + n; 0x5400 | 16n is 64 + n), so each run
// sits in TMEM in the order 0,4,1,5,2,6,3,7.  The query latents are stored in the same
// order (a score is an order-free sum over ranks).  A value word holds eight tokens, with
// tokens 2m and 2m + 1 in nibbles m and m + 4, so the same four pairs come out in token
// order, matching the probabilities.
//
// Keys stored before the rotary embedding (kRope).  The score needs the rotated key,
// which has no rank-space form, so each tile's keys are rebuilt on the tensor cores:
//   K^_h[t, :] = z^_k,t B_k,h          GEMM0: M = 128 tokens, N = d = 128, K = r_k
// (A = the same token-row operand as GEMM1) then rotated (rotate-half RoPE at the token's
// absolute position, cos / sin from the cache's fp64-derived table) and dotted with the
// raw query rows on CUDA cores by the softmax warps (thread = token row).  K^ for all four
// KV heads would need all of TMEM, so a CTA covers a pair of KV heads (grid x), query slots
// 16 h + jj for query head jj of pair head h; both CTAs of a pair dequantise the same
// tiles.  B_k enters as an fp16 copy, [D rows][ranks] with each 8-rank run in the
// dequantised order, streamed per 64-rank sub-block (both heads' rows, one N = 256 MMA per
// 16 ranks) by TMA from a spare warp (warp 2) through a ring of up to four slots.  The
// rotation factors of a row are fetched one 16-pair chunk ahead (the next tile's first
// chunk during the last one), so their L2 latency stays off the chain rebuild -> rotate
// -> rebuild.  The value mix and the epilogue are those of the rank-space kernel.
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

// Warpgroups: [producer, key MMAs, B_k producer / idle, value MMAs] [4 softmax] [key
// dequantisation] [value dequantisation], with 4 or 8 warps per dequantisation side (Cfg).  A
// warp runs on sub-partition (warp % 4), and a tcgen05.ld / st reaches TMEM lanes
// 32 (warp % 4) .. + 31.  The warpgroups rebalance the launch's registers with setmaxnreg
// (the softmax keeps 32 scores and 32 running sums per row).
constexpr int kDqWarp0 = 8;                // first warp of the dequantisation warpgroups
constexpr int kSmWarps = 4;                // softmax warps (one arrival each)
// Per variant: dequantisation warps per TMEM lane quarter and side (rank space: two, each
// expanding one 32-column half of every chunk, so that a sub-partition holds two warps of each
// side to hide each other's latency; keys before RoPE: one, expanding both halves), the block
// size, the launch allocation, and the per-warpgroup register budgets (multiples of 8):
// control, softmax / epilogue, dequantisation.  The budgets fill the launch allocation.
template <bool kRope> struct Cfg;
template <> struct Cfg<false> {
  static constexpr int dq_per_quarter = 2, threads = 256 + 256 * dq_per_quarter, launch_regs = 80;
  static constexpr int ctl = 48, softmax = 176, dq = 64;
};
template <> struct Cfg<true> {
  static constexpr int dq_per_quarter = 1, threads = 256 + 256 * dq_per_quarter, launch_regs = 128;
  static constexpr int ctl = 64, softmax = 240, dq = 104;
};
template <bool kRope> using Regs = Cfg<kRope>;
// Move this warpgroup from the launch allocation to `kTo` registers per thread: setmaxnreg.inc
// when raising, .dec when lowering (a .dec above the current count is an illegal instruction).
template <int kTo, int kFrom>
__device__ __forceinline__ void set_regs() {
  static_assert(kTo % 8 == 0 && kTo >= 24 && kTo <= 256, "setmaxnreg range");
  if constexpr (kTo > kFrom) ptx::setmaxnreg_inc<kTo>();
  else if constexpr (kTo < kFrom) ptx::setmaxnreg_dec<kTo>();
}
static_assert(128 * Cfg<false>::ctl + 128 * Cfg<false>::softmax + 256 * Cfg<false>::dq_per_quarter * Cfg<false>::dq <=
                  Cfg<false>::threads * Cfg<false>::launch_regs,
              "register split exceeds the launch allocation");
static_assert(128 * Cfg<true>::ctl + 128 * Cfg<true>::softmax + 256 * Cfg<true>::dq_per_quarter * Cfg<true>::dq <=
                  Cfg<true>::threads * Cfg<true>::launch_regs,
              "register split exceeds the launch allocation");
constexpr int kSubBytes = 128 * 128;       // B_k ring: 128 rows x 64 ranks x 2 B per KV head
constexpr int kQRows = 32;                 // query heads, padded
constexpr int kQSubBytes = kQRows * 128;   // 32 rows x 64 ranks x 2 B
constexpr int kPBytes = 128 * 32 * 2;      // 128 tokens x 32 heads x 2 B
constexpr int kAuxBytes = 2048;
// TMEM columns, rank space: S of tile s in [32 (s % 2), +32), O~ chunk c in [64 + 32 c, +32),
// operand slots of 64 columns from 192 (two for keys, three for values)
constexpr int kSCol = 0;
constexpr int kOCol = 64;
constexpr int kACol = 192;
// keys before RoPE: K^ of the pair in [0, 256), O~ in [256, 384), operand slots from 384
constexpr int kOColR = 256;
constexpr int kAColR = 384;
constexpr int kASlotCols = 64;             // one operand slot: 128 lanes x 128 fp16 K elements
constexpr int kMaxASlots = 5;
constexpr int kRD = 128;                   // head dim of the rebuilt keys
constexpr int kGHMax = 2;                  // KV heads per CTA (K^ of both fills 256 columns)
constexpr int kMaxG = 32 / kGHMax;         // query slots per KV head (the N of the score MMA)
constexpr int kQbHeadBytes = 2 * kMaxG * 128;   // fp16 query rows of one KV head: 2 sub-blocks x 16 x 128 B
constexpr int kNBMax = 4;                  // B_k ring slots (kv heads x 128 rows x 64 ranks, fp16)
constexpr int kMaxRaw = 8;                 // raw slot: one side of one tile, codes (G x 2 KB)
                                           // then {scale, zero} words (G x 512 B)

struct I4Params {
  unsigned long long wait_ns;   // bounded-wait limit (0: the default)
  const int32_t* row_len;       // per-row history lengths (device), or null
  unsigned long long* span;     // timeline span, or null
  const uint32_t* codes_k;
  const uint32_t* codes_v;
  const uint32_t* params_k;
  const uint32_t* params_v;
  RowMap map;                   // token -> latent row (block)
  int r_k, r_v, G_k, G_v, ck, cv, kb_k;
  int Hq, hist_len, stable_len, split_tokens, n_splits;
  int nks, nvs;                 // operand slots of the key ring [0, nks) and the value ring [nks, +nvs)
  int nrk, nrv;                 // raw slots of the key ring [0, nrk) and the value ring [nrk, +nrv)
  uint32_t q_bytes, raw_bytes, raw_params;   // raw slot size; offset of its params
  float* part_o;
  float* part_ml;
  int* err;
  unsigned long long* trace;
  // keys before RoPE
  const float* qf;          // [B][Hq][d] scaled queries, fp32
  const float2* rope_cs;    // (cos, sin), rope_cs_index layout
  int gh, gsz;              // KV heads per CTA, query heads per KV head
  uint32_t q_load_bytes;    // gh * gsz * d * 4
  uint32_t qf_bytes;        // the fp32 rows' block, rounded up to 1024 (the fp16 operand follows)
  int nb;                   // B_k ring slots of gh * 16 KB
};

// Barriers (arrival count; who arrives -> who waits).  Phase k of a barrier is waited with
// parity k & 1.
//   raw_full[]        1 + tx   producer's two bulk copies -> the side's dequantisation warps
//   raw_empty[]       4        the side's dequantisation warps -> producer
//   slot_full[]       4        the side's dequantisation warps (TMEM stores waited and fenced)
//                              -> the side's MMA issuer
//   slot_empty[]      1        MMA commit -> the side's dequantisation warps
//                              (raw slots [0, nrk) and operand slots [0, nks) hold keys, the
//                              rest values: each ring has one producer and one consumer that
//                              walk it in tile order, so no wait is on a phase more than one
//                              ahead of its barrier)
//   q_full            1 + tx   producer (after the grid-dependency wait) -> MMA issuer, or
//                              the softmax warps for keys before RoPE
//   s_full[2]         1        MMA commit of GEMM1 -> softmax warps
//   s_empty[2]        4        softmax warps (scores read) -> MMA issuer
//   p_full[2]         4        softmax warps (fenced P stores) -> MMA issuer
//   p_empty[2]        1        MMA commit of GEMM2 -> softmax warps (P reuse, O~ rescale)
//   o_final           1        value issuer's commit after its last unit -> softmax warps (epilogue)
//   k_fin             1        key issuer's commit after its last unit -> itself (drain before exit)
//   keys before RoPE, in place of s_empty:
//   k_full            1        MMA commit of GEMM0 -> softmax warps
//   krot_full         4        softmax warps (rotated fp16 keys stored, waited, fenced) -> MMA issuer
//   s_full[0]         1        MMA commit of the score MMAs -> softmax warps
//   k_empty           4        softmax warps (scores read) -> MMA issuer (next GEMM0)
//   qb_full           4        softmax warps (fp16 query operand stored, fenced) -> MMA issuer
//   b_full[nb]        1 + tx   B_k producer (warp 2) -> MMA issuer
//   b_empty[nb]       1        MMA commit -> B_k producer
struct Aux {
  uint64_t slot_full[kMaxASlots];
  uint64_t slot_empty[kMaxASlots];
  uint64_t raw_full[kMaxRaw];
  uint64_t raw_empty[kMaxRaw];
  uint64_t s_full[2], s_empty[2], p_full[2], p_empty[2];
  uint64_t q_full, o_final, k_fin;
  uint64_t k_full, k_empty, krot_full, qb_full, b_full[kNBMax], b_empty[kNBMax];
  uint32_t tmem_base;
  int abort_flag;
  unsigned long long wait_ns;   // this launch's wait limit
  float red[4][32];
  alignas(16) float m_s[32];
  float alpha_s[32];
};
static_assert(sizeof(Aux) <= kAuxBytes, "aux block");

struct I4State {
  CUtensorMap q;
  CUtensorMap bk;           // keys before RoPE: fp16 B_k [D][r_pad], rank runs permuted
  void* bk16 = nullptr;
  int r_pad = 0;
  int nraw, nb = 0;
  uint32_t raw_bytes, raw_params, q_bytes;
  size_t smem;
};

__device__ __forceinline__ bool wait_b(uint64_t* bar, uint32_t parity, Aux* aux, int* err) {
  return tc::wait_b(bar, parity, &aux->abort_flag, err, aux->wait_ns);
}
// The same, by a whole warp with one verdict for all its lanes.
__device__ __forceinline__ bool wait_w(uint64_t* bar, uint32_t parity, Aux* aux, int* err) {
  return __all_sync(0xffffffffu, wait_b(bar, parity, aux, err));
}

// One fp16 pair of int4 codes: (lo, hi) = n - bias, then * scale + zero (one rounding).
__device__ __forceinline__ uint32_t dq_pair(uint32_t biased, uint32_t bias, uint32_t s2, uint32_t z2) {
  uint32_t r;
  asm("{\n\t.reg .b32 t;\n\t"
      "sub.rn.f16x2 t, %1, %2;\n\t"
      "fma.rn.f16x2 %0, t, %3, %4;\n\t}"
      : "=r"(r)
      : "r"(biased), "r"(bias), "r"(s2), "r"(z2));
  return r;
}

// Eight int4 codes of one word -> four fp16 pairs (m0,m4) (m1,m5) (m2,m6) (m3,m7) of
// code * scale + zero, pair k with its own scale and zero pairs (s2.k, z2.k).
__device__ __forceinline__ uint4 dequant8(uint32_t w, const uint4& s2, const uint4& z2) {
  const uint32_t a = (w & 0x000F000Fu) | 0x64006400u;   // 1024 + n
  const uint32_t b = (w & 0x00F000F0u) | 0x54005400u;   // 64 + n
  const uint32_t w8 = w >> 8;
  const uint32_t c = (w8 & 0x000F000Fu) | 0x64006400u;
  const uint32_t d = (w8 & 0x00F000F0u) | 0x54005400u;
  uint4 r;
  r.x = dq_pair(a, 0x64006400u, s2.x, z2.x);
  r.y = dq_pair(b, 0x54005400u, s2.y, z2.y);
  r.z = dq_pair(c, 0x64006400u, s2.z, z2.z);
  r.w = dq_pair(d, 0x54005400u, s2.w, z2.w);
  return r;
}
__device__ __forceinline__ void put4(uint32_t (&v)[32], int at, const uint4& r) {
  v[at] = r.x;
  v[at + 1] = r.y;
  v[at + 2] = r.z;
  v[at + 3] = r.w;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Shared memory: [aux 2 KB][q~ per 64-rank sub-block | fp32 query rows, then the fp16
//                query operand of the score MMAs (kRope)]
//                [B_k ring nb x gh x 16 KB (kRope)][P double buffer 2 x 8 KB]
//                [raw ring nraw x raw_bytes]
template <bool kRope>
__global__ void __launch_bounds__(Cfg<kRope>::threads, 1)
    k_decode_tc_i4(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_b,
                   const I4Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (ptx::smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicExch(p.err, (int)LR_ERR_UNSUPPORTED);
    return;
  }
  span_begin(p.span);
  Aux* aux = reinterpret_cast<Aux*>(smem_raw);
  uint8_t* q_s = smem_raw + kAuxBytes;
  uint8_t* bring = q_s + p.q_bytes;
  const uint32_t b_slot_bytes = kRope ? (uint32_t)(p.gh * kSubBytes) : 0u;
  uint8_t* p_s = bring + (kRope ? p.nb * b_slot_bytes : 0);
  uint8_t* raw = p_s + 2 * kPBytes;
  constexpr int kOC = kRope ? kOColR : kOCol;
  constexpr int kAC = kRope ? kAColR : kACol;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = kRope ? (int)blockIdx.x : 0;
  const int split = kRope ? blockIdx.y : blockIdx.x, b = kRope ? blockIdx.z : blockIdx.y;
  const int tok_begin = split * p.split_tokens;
  const int tok_end = min(row_hist(p.row_len, b, p.hist_len), tok_begin + p.split_tokens);
  const int ntiles = tok_end > tok_begin ? (tok_end - tok_begin + kTile - 1) / kTile : 0;
  const int nunits = 2 * ntiles;
  // query head of score / output slot j (-1: padding)
  auto head_of = [&](int j) -> int {
    if (!kRope) return j < p.Hq ? j : -1;
    const int h = j / kMaxG, jj = j % kMaxG;
    return (h < p.gh && jj < p.gsz) ? (pair * p.gh + h) * p.gsz + jj : -1;
  };

  if (threadIdx.x == 0) {
    tc::trace_stamp(p.trace, 0);
    for (int s = 0; s < p.nks + p.nvs; ++s) {
      ptx::mbar_init(&aux->slot_full[s], 4 * Cfg<kRope>::dq_per_quarter);
      ptx::mbar_init(&aux->slot_empty[s], 1);
    }
    for (int s = 0; s < p.nrk + p.nrv; ++s) {
      ptx::mbar_init(&aux->raw_full[s], 1);
      ptx::mbar_init(&aux->raw_empty[s], 4 * Cfg<kRope>::dq_per_quarter);
    }
    for (int k = 0; k < 2; ++k) {
      ptx::mbar_init(&aux->s_full[k], 1);
      ptx::mbar_init(&aux->s_empty[k], kSmWarps);
      ptx::mbar_init(&aux->p_full[k], kSmWarps);
      ptx::mbar_init(&aux->p_empty[k], 1);
    }
    ptx::mbar_init(&aux->q_full, 1);
    ptx::mbar_init(&aux->o_final, 1);
    ptx::mbar_init(&aux->k_fin, 1);
    if (kRope) {
      ptx::mbar_init(&aux->k_full, 1);
      ptx::mbar_init(&aux->k_empty, kSmWarps);
      ptx::mbar_init(&aux->krot_full, kSmWarps);
      ptx::mbar_init(&aux->qb_full, kSmWarps);
      for (int k = 0; k < p.nb; ++k) {
        ptx::mbar_init(&aux->b_full[k], 1);
        ptx::mbar_init(&aux->b_empty[k], 1);
      }
    }
    aux->abort_flag = 0;
    aux->wait_ns = tc::wait_limit(p.wait_ns);
    for (int j = 0; j < 32; ++j) aux->m_s[j] = -INFINITY;
    ptx::fence_mbar_init();
  }
  if (warp == 0 && lane == 0 && !kRope) ptx::prefetch_tmap(&tm_q);
  if (warp == 2 && lane == 0 && kRope) ptx::prefetch_tmap(&tm_b);
  if (warp == 1) {
    ptx::tmem_alloc(&aux->tmem_base, 512);
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
    set_regs<Regs<kRope>::ctl, Cfg<kRope>::launch_regs>();
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
        int issued_k = 0, issued_v = 0;   // tiles whose copies were issued, per side
        // the latent row (block) of each unit is read one unit ahead, so that a paged cache's
        // table read overlaps the waits and copies of the unit before
        auto row_of_unit = [&](int u) -> long long {
          int tl;
          bool iv;
          tc::unit_of(u, ntiles, &tl, &iv);
          return p.map.row(b, tok_begin + tl * kTile);
        };
        long long row_next = nunits > 0 ? row_of_unit(0) : 0;
        for (int u = 0; u < nunits && ok; ++u) {
          int tile;
          bool is_v;
          tc::unit_of(u, ntiles, &tile, &is_v);
          const long long row0 = row_next;   // a whole block: one page
          if (u + 1 < nunits) row_next = row_of_unit(u + 1);
          const int t0 = tok_begin + tile * kTile;
          const int n = min(kTile, tok_end - t0);
          const int nr = is_v ? p.nrv : p.nrk;
          const int rs = (is_v ? p.nrk : 0) + tile % nr, round = tile / nr;
          if (!waited && (round > 0 || t0 + n > p.stable_len)) {
            pdl_wait();
            load_query();
            waited = true;
          }
          if (round > 0 && !(ok = wait_b(&aux->raw_empty[rs], (round - 1) & 1, aux, p.err))) break;
          const int G = is_v ? p.G_v : p.G_k;
          uint8_t* dst = raw + rs * p.raw_bytes;
          // one block of one side: G x 2 KB of codes and G x 512 B of params, at the same
          // offsets for the token-major keys and the rank-major values
          ptx::mbar_arrive_expect_tx(&aux->raw_full[rs], (uint32_t)G * 2560u);
          ptx::bulk_load(dst, (is_v ? p.codes_v : p.codes_k) + i4_code_index(row0, G, 0, 0), (uint32_t)G * 2048u,
                         &aux->raw_full[rs]);
          ptx::bulk_load(dst + p.raw_params, (is_v ? p.params_v : p.params_k) + i4_param_index(row0, G, 0),
                         (uint32_t)G * 512u, &aux->raw_full[rs]);
          (is_v ? issued_v : issued_k) = tile + 1;
        }
        if (!waited) {
          pdl_wait();
          load_query();
        }
        // Every copy this thread issued has landed before the CTA can exit: after an abort
        // (here or in another role, which may come after this loop) the consumers stop
        // waiting for them.  In a normal run these are the phases the consumers already
        // waited for, so the waits return at once.
        drain_wait(&aux->q_full, 0);
        for (int k = max(0, issued_k - p.nrk); k < issued_k; ++k) drain_wait(&aux->raw_full[k % p.nrk], (k / p.nrk) & 1);
        for (int k = max(0, issued_v - p.nrv); k < issued_v; ++k)
          drain_wait(&aux->raw_full[p.nrk + k % p.nrv], (k / p.nrv) & 1);
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
        (void)ok;   // drained whether or not the CTA aborted (see the producer above)
        for (int k = max(0, issued - p.nb); k < issued; ++k) drain_wait(&aux->b_full[k % p.nb], (k / p.nb) & 1);
      }
    } else if (warp == 1 || warp == 3) {
      // ------------------------------------------------------------- MMA issuers
      // Warp 1 issues the key side (GEMM1, or GEMM0 and the score MMAs), warp 3 the value
      // mix (GEMM2); each commits its own MMAs.  The whole warp runs its loop (operands
      // warp-uniform, K steps unrolled) and one elected lane issues: an MMA every ~18
      // cycles, the tensor core's pace at N = 32, where one lane alone needs ~50-80.
      const bool kside = warp == 1;
      if (ntiles > 0) {
        const uint32_t id = ptx::idesc_f16(0, 0, 0, 128, 32);    // GEMM1: fp16, A (TMEM) x K-major B
        const uint32_t id2 = ptx::idesc_f16(0, 0, 1, 128, 32);   // GEMM2: fp16, A (TMEM) x MN-major B
        // Descriptors are built once; a step along K or to another slot adds its byte
        // offset >> 4 to the start-address field (shared-memory addresses stay below
        // 256 KB, so the 14-bit field never carries).
        const uint64_t qdesc0 = ptx::smem_desc(ptx::smem_u32(q_s), 16, 1024, 2);        // q~, K-major SW128
        const uint64_t pdesc0 = ptx::smem_desc(ptx::smem_u32(p_s), 128, 2048, 0);       // P, MN-major
        const uint32_t idk = ptx::idesc_f16(0, 0, 0, 128, kRope ? p.gh * kRD : 128);   // GEMM0 (kRope)
        const uint64_t bdesc0 = ptx::smem_desc(ptx::smem_u32(bring), 16, 1024, 2);      // B_k, K-major SW128
        const uint32_t idq = ptx::idesc_f16(0, 0, 0, 128, kMaxG);                        // scores (kRope)
        const uint64_t qbdesc0 = ptx::smem_desc(ptx::smem_u32(q_s + p.qf_bytes), 16, 1024, 2);   // fp16 q, SW128
        bool ok = (kRope || !kside) ? true : wait_w(&aux->q_full, 0, aux, p.err);
        ptx::tc_fence_after();
        if (kside && lane == 0) tc::trace_stamp(p.trace, 2);
        // this issuer's operand-slot ring: the key ring is slots [0, nks), the value ring
        // [nks, nks + nvs)
        const int ring0 = kside ? 0 : p.nks, nring = kside ? p.nks : p.nvs;
        int pos = 0, bpos = 0;
        for (int u = 0; u < nunits && ok; ++u) {
          int tile;
          bool is_v;
          tc::unit_of(u, ntiles, &tile, &is_v);
          if (is_v == kside) continue;   // the other issuer's unit
          if (kRope && !is_v) {
            // GEMM0(tile): [K^_0 | K^_1] = Z_k [B_k,0 | B_k,1], columns [128 h, +128) per head
            if (tile >= 1 && !(ok = wait_w(&aux->k_empty, (tile - 1) & 1, aux, p.err))) break;
            ptx::tc_fence_after();
            for (int c = 0; c < p.ck && ok; ++c, ++pos) {
              const int slot = ring0 + pos % nring;
              if (!(ok = wait_w(&aux->slot_full[slot], (pos / nring) & 1, aux, p.err))) break;
              ptx::tc_fence_after();
              const uint32_t a0 = tmem + kAC + slot * kASlotCols;
              for (int sb = 0; sb < 2 && c * 128 + sb * 64 < p.r_k; ++sb, ++bpos) {
                const int bs = bpos % p.nb;
                if (!(ok = wait_w(&aux->b_full[bs], (bpos / p.nb) & 1, aux, p.err))) break;
                ptx::tc_fence_after();
                const uint64_t b0 = bdesc0 + (uint64_t)((bs * b_slot_bytes) >> 4);
                // K step kk of the sub-block: 8 TMEM columns on A, 32 bytes on B
                const int nk = min(4, (p.r_k - c * 128 - sb * 64) >> 4);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  if (kk < nk)
                    ptx::mma_f16_ta_elect(tmem, a0 + (uint32_t)(sb * 32 + kk * 8), b0 + (uint64_t)(kk * 2), idk,
                                     (c | sb | kk) ? 1u : 0u);
                ptx::mma_commit_elect(&aux->b_empty[bs]);
              }
              if (!ok) break;
              ptx::mma_commit_elect(&aux->slot_empty[slot]);
            }
            if (!ok) break;
            ptx::mma_commit_elect(&aux->k_full);
            if (tile < 16 && lane == 0) tc::trace_stamp(p.trace, 3 + 4 * tile);
            // scores of the pair's query heads against the rotated fp16 keys the softmax warps
            // wrote back over K^: per head, M = 128 tokens, N = 16 query slots, K = d
            if (tile == 0 && !(ok = wait_w(&aux->qb_full, 0, aux, p.err))) break;
            if (!(ok = wait_w(&aux->krot_full, tile & 1, aux, p.err))) break;
            ptx::tc_fence_after();
            for (int h = 0; h < p.gh; ++h)
#pragma unroll
              for (int kk = 0; kk < kRD / 16; ++kk)
                ptx::mma_f16_ta_elect(tmem + h * kRD + kRD / 2, tmem + h * kRD + kk * 8,
                           qbdesc0 + (uint64_t)((h * kQbHeadBytes + (kk >> 2) * (kQbHeadBytes / 2)) >> 4) +
                               (uint64_t)((kk & 3) * 2),
                           idq, kk ? 1u : 0u);
            ptx::mma_commit_elect(&aux->s_full[0]);
          } else if (!is_v) {
            // GEMM1(tile): S[tile % 2] = Z_k q~^T (consecutive MMAs into one accumulator issue
            // at the same rate as into alternating ones)
            const int sb2 = tile & 1;
            if (tile >= 2 && !(ok = wait_w(&aux->s_empty[sb2], ((tile - 2) >> 1) & 1, aux, p.err))) break;
            ptx::tc_fence_after();
            const uint32_t d_s = tmem + kSCol + 32 * sb2;
            for (int c = 0; c < p.ck && ok; ++c, ++pos) {
              const int slot = ring0 + pos % nring;
              if (!(ok = wait_w(&aux->slot_full[slot], (pos / nring) & 1, aux, p.err))) break;
              ptx::tc_fence_after();
              const uint32_t a0 = tmem + kAC + slot * kASlotCols;
              const uint64_t b0 = qdesc0 + (uint64_t)((c * 2 * kQSubBytes) >> 4);
              const int nk = min(8, (p.r_k - c * 128) >> 4);     // 16-rank K steps in this chunk
              // step kk: 8 TMEM columns on A; sub-block kk / 4 (4 KB), 32 bytes per step on B
#pragma unroll
              for (int kk = 0; kk < 8; ++kk) {
                const uint32_t bo = (uint32_t)((kk >> 2) * (kQSubBytes >> 4) + (kk & 3) * 2);
                if (kk < nk) ptx::mma_f16_ta_elect(d_s, a0 + (uint32_t)(kk * 8), b0 + bo, id, (c | kk) ? 1u : 0u);
              }
              ptx::mma_commit_elect(&aux->slot_empty[slot]);
            }
            if (!ok) break;
            ptx::mma_commit_elect(&aux->s_full[sb2]);
            if (tile < 16 && lane == 0) tc::trace_stamp(p.trace, 3 + 4 * tile);
          } else {
            // GEMM2(tile): O~ += Z_v^T P[tile % 2]
            const int pb2 = tile & 1;
            if (!(ok = wait_w(&aux->p_full[pb2], (tile >> 1) & 1, aux, p.err))) break;
            ptx::tc_fence_after();
            const uint64_t b0 = pdesc0 + (uint64_t)((pb2 * kPBytes) >> 4);
            for (int c = 0; c < p.cv && ok; ++c, ++pos) {
              const int slot = ring0 + pos % nring;
              if (!(ok = wait_w(&aux->slot_full[slot], (pos / nring) & 1, aux, p.err))) break;
              ptx::tc_fence_after();
              const uint32_t a0 = tmem + kAC + slot * kASlotCols;
              const uint32_t d_o = tmem + kOC + c * 32;
              // K step kt = 16 tokens: 8 TMEM columns on A, 256 B on P
#pragma unroll
              for (int kt = 0; kt < 8; ++kt)
                ptx::mma_f16_ta_elect(d_o, a0 + (uint32_t)(kt * 8), b0 + (uint64_t)(kt * 16), id2, (tile | kt) ? 1u : 0u);
              ptx::mma_commit_elect(&aux->slot_empty[slot]);
            }
            if (!ok) break;
            ptx::mma_commit_elect(&aux->p_empty[pb2]);
            if (tile < 16 && lane == 0) tc::trace_stamp(p.trace, 6 + 4 * tile);
          }
        }
        // the value issuer's last commit releases the epilogue; each issuer's MMAs have
        // completed before TMEM is freed, even if the epilogue aborted
        uint64_t* fin = kside ? &aux->k_fin : &aux->o_final;
        ptx::mma_commit_elect(fin);
        drain_wait(fin, 0);
      }
      __syncwarp();
    }
  } else if (warp < kDqWarp0) {
    set_regs<Regs<kRope>::softmax, Cfg<kRope>::launch_regs>();
    if (ntiles > 0) {
      // ------------------------------------------------------------- softmax / epilogue
      const int qd = warp & 3;
      const int row = qd * 32 + lane;
      const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
      float l[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) l[j] = 0.f;
      bool ok = true;
      if (kRope) {
        // keys before RoPE: the fp32 query rows become the fp16 B operand of the score MMAs,
        // [head][2 sub-blocks of 64 K][16 query slots][128 B] with the 128-byte swizzle;
        // K element 2m holds dimension m and 2m + 1 dimension m + 64 (the order in which the
        // rotated keys are stored), slots >= the group size are zero
        ok = ptx::named_bar_and(1, 128, wait_b(&aux->q_full, 0, aux, p.err));
        if (ok) {
          const float* q_f = reinterpret_cast<const float*>(q_s);
          uint8_t* qb = q_s + p.qf_bytes;
          for (int idx = threadIdx.x - 128; idx < p.gh * kMaxG * kRD; idx += 128) {
            const int hh = idx / (kMaxG * kRD), n = (idx / kRD) % kMaxG, k = idx % kRD;
            const int dim = (k & 1) ? (k >> 1) + kRD / 2 : (k >> 1);
            const float v = n < p.gsz ? q_f[(hh * p.gsz + n) * kRD + dim] : 0.f;
            const int sb = k >> 6, ch = (k & 63) >> 3;
            *reinterpret_cast<__half*>(qb + hh * kQbHeadBytes + sb * (kQbHeadBytes / 2) + n * 128 +
                                       ((ch ^ (n & 7)) << 4) + (k & 7) * 2) = __float2half_rn(v);
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&aux->qb_full);
        }
      }
      // rotation factors: cs holds the chunk in use, csn the one after it
      float cs[32], csn[32];
      auto load_cs = [&](float(&dst)[32], int tile_i, int c0) {
        // pairs c0 .. c0 + 15 of this row's token; lanes own consecutive tokens, so each
        // pair is one coalesced 256-byte read per warp
        const int t = tok_begin + tile_i * kTile + row;
        const float2* src = p.rope_cs + rope_cs_index(t < tok_end ? t : tok_begin, c0, kRD / 2);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float2 v = __ldg(src + k * 128);
          dst[2 * k] = v.x;
          dst[2 * k + 1] = v.y;
        }
      };
      // scores of tile buffer k2
      auto load_s = [&](int k2, bool valid, float(&s)[32]) {
        const uint32_t s_col = tmem + lane_off + kSCol + 32 * k2;
        uint32_t sv[16], sw[16];
        ptx::tmem_ld16(s_col, sv);
        ptx::tmem_ld16(s_col + 16, sw);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          s[j] = valid ? __uint_as_float(sv[j]) : -INFINITY;
          s[16 + j] = valid ? __uint_as_float(sw[j]) : -INFINITY;
        }
      };
      if (kRope) load_cs(cs, 0, 0);
      for (int i = 0; i < ntiles && ok; ++i) {
        const int k2 = i & 1;
        const bool valid = tok_begin + i * kTile + row < tok_end;
        float s[32];
        if (kRope) {
          ok = ptx::named_bar_and(1, 128, wait_b(&aux->k_full, i & 1, aux, p.err));
          if (!ok) break;
          ptx::tc_fence_after();
          if (i < 16 && threadIdx.x == 128) tc::trace_stamp(p.trace, 4 + 4 * i);
          // rotate-half RoPE of each row's keys at the token's position, written back over
          // K^ as fp16: pair (c, c + 64) of chunk c0 goes to column h * 128 + c (K elements
          // 2c, 2c + 1); a chunk's columns were read before they are written
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
                uint32_t w[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                  const float a = __uint_as_float(x1[k]), e = __uint_as_float(x2[k]);
                  const __half2 hv = __floats2half2_rn(a * cs[2 * k] - e * cs[2 * k + 1], e * cs[2 * k] + a * cs[2 * k + 1]);
                  w[k] = *reinterpret_cast<const uint32_t*>(&hv);
                }
                tmem_st16(tmem + lane_off + h * kRD + c0, w);
              }
            }
#pragma unroll
            for (int k = 0; k < 32; ++k) cs[k] = csn[k];
          }
          ptx::tmem_wait_st();
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&aux->krot_full);
          // the scores of the pair's query slots: head h's 16 slots in columns h * 128 + 64
          ok = ptx::named_bar_and(1, 128, wait_b(&aux->s_full[0], i & 1, aux, p.err));
          if (!ok) break;
          ptx::tc_fence_after();
#pragma unroll
          for (int h = 0; h < kGHMax; ++h) {
            uint32_t sv[16];
            if (h < p.gh) {
              ptx::tmem_ld16(tmem + lane_off + h * kRD + kRD / 2, sv);
              ptx::tmem_wait_ld();
            }
#pragma unroll
            for (int jj = 0; jj < kMaxG; ++jj) s[h * kMaxG + jj] = h < p.gh ? __uint_as_float(sv[jj]) : 0.f;
          }
          // the scores have been read: GEMM0 of the next tile may overwrite the region
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
          load_s(k2, valid, s);
        }

        bool ex = false;
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 mv = reinterpret_cast<const float4*>(aux->m_s)[j4];   // broadcast reads
          ex |= (s[4 * j4] > mv.x + kLazy) | (s[4 * j4 + 1] > mv.y + kLazy) | (s[4 * j4 + 2] > mv.z + kLazy) |
                (s[4 * j4 + 3] > mv.w + kLazy);
        }
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
            load_s(k2, valid, s);
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
          const float4 ma = reinterpret_cast<const float4*>(aux->m_s)[2 * hg];
          const float4 mb = reinterpret_cast<const float4*>(aux->m_s)[2 * hg + 1];
          const float mh[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = hg * 8 + 2 * e;
            const __half2 h = __floats2half2_rn(exp2f(s[j] - mh[2 * e]), exp2f(s[j + 1] - mh[2 * e + 1]));
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
        // TMEM row m of chunk c holds rank 128 c + m (values are expanded in rank order)
        const int m = qd * 32 + lane;
        for (int c = 0; c < p.cv; ++c) {
          uint32_t v2[32];
          ptx::tmem_ld32(tmem + lane_off + kOC + c * 32, v2);
          ptx::tmem_wait_ld();
          const int e = c * 128 + m;
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
    } else if (warp == 4) {
      // a split that starts beyond its row's length: zero weight in the merge
      const int J = head_of(lane);
      if (J >= 0) {
        const size_t base_out = ((size_t)b * p.n_splits + split) * p.Hq;
        p.part_ml[(base_out + J) * 2] = -INFINITY;
        p.part_ml[(base_out + J) * 2 + 1] = 0.f;
      }
    }
  } else {
    set_regs<Regs<kRope>::dq, Cfg<kRope>::launch_regs>();
    // ------------------------------------------------------------- dequantisation
    if (ntiles > 0) {
      // side = 0: keys (warps 8 .. 8 + 4 kDqPQ - 1), side = 1: values (the next 4 kDqPQ).
      // Warp quarter qd = warp % 4 owns TMEM lanes 32 qd .. + 31 of every operand slot of its
      // side and fills its 64 columns in two halves h of 32 columns (both halves, or with
      // two warps per quarter one half each).  Keys: token 32 qd + lane, ranks
      // 64 h .. + 63 of the chunk (groups 4c + 2h, + 1).  Values: rank 128 c + 32 qd + lane
      // (group 4c + qd), tokens 64 h .. + 63.
      const int qd = warp & 3;
      constexpr int kDqPQ = Cfg<kRope>::dq_per_quarter;
      const int dqj = warp - kDqWarp0;                   // [0, 8 kDqPQ): the side's warps, keys first
      const bool is_v = dqj >= 4 * kDqPQ;
      // with two warps per quarter, warp (dqj / 4) % 2 of the side expands half h of each chunk
      const int h_beg = kDqPQ == 2 ? (dqj >> 2) & 1 : 0, h_end = kDqPQ == 2 ? h_beg + 1 : 2;
      const uint32_t lane_off = (uint32_t)(qd * 32) << 16;
      const uint32_t raw_base = ptx::smem_u32(raw);
      const int G = is_v ? p.G_v : p.G_k;
      const int nch = is_v ? p.cv : p.ck;
      const int nr = is_v ? p.nrv : p.nrk, r0 = is_v ? p.nrk : 0;
      const int ring0 = is_v ? p.nks : 0, nring = is_v ? p.nvs : p.nks;
      const bool tracer = lane == 0 && qd == 0;
      bool ok = true;
      int pos = 0;
      for (int tile = 0; tile < ntiles && ok; ++tile) {
        const int rs = r0 + tile % nr;
        const uint32_t rb = raw_base + rs * p.raw_bytes;
        // waits are made warp-uniform: the warp arrives once, after __syncwarp
        if (!(ok = __all_sync(0xffffffffu, wait_b(&aux->raw_full[rs], (tile / nr) & 1, aux, p.err)))) break;
        for (int c = 0; c < nch; ++c, ++pos) {
          const int slot = ring0 + pos % nring;
          if (pos >= nring &&
              !(ok = __all_sync(0xffffffffu, wait_b(&aux->slot_empty[slot], ((pos / nring) - 1) & 1, aux, p.err))))
            break;
          ptx::tc_fence_after();
          bool stored = false;
#pragma unroll 1
          for (int h = h_beg; h < h_end; ++h) {
            uint32_t v[32];
            bool any = false;
            if (!is_v) {
              const int t = qd * 32 + lane;
              const int g0 = 4 * c + 2 * h;
              any = g0 < G;
#pragma unroll
              for (int gi = 0; gi < 2; ++gi) {
                const int g = g0 + gi;
                if (g < G) {
                  const uint4 w = lds128(rb + (uint32_t)(g * 2048 + t * 16));
                  const uint32_t prm = lds32(rb + p.raw_params + (uint32_t)((g * 128 + t) * 4));
                  const uint32_t s2 = __byte_perm(prm, 0u, 0x1010), z2 = __byte_perm(prm, 0u, 0x3232);
                  const uint4 ss = make_uint4(s2, s2, s2, s2), zz = make_uint4(z2, z2, z2, z2);
                  put4(v, 16 * gi + 0, dequant8(w.x, ss, zz));
                  put4(v, 16 * gi + 4, dequant8(w.y, ss, zz));
                  put4(v, 16 * gi + 8, dequant8(w.z, ss, zz));
                  put4(v, 16 * gi + 12, dequant8(w.w, ss, zz));
                } else {
#pragma unroll
                  for (int k = 0; k < 16; ++k) v[16 * gi + k] = 0u;
                }
              }
            } else {
              const int g = 4 * c + qd;
              any = g < G;
              if (any) {
                const int i = c * 128 + qd * 32 + lane;
                const uint32_t rowa = rb + (uint32_t)(i * 64);
                const uint32_t sc = rb + p.raw_params + (uint32_t)(g * 512 + h * 128);   // scales of tokens 64h..
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                  const int lc = 2 * h + half;                                   // 32-token column
                  const uint4 w = lds128(rowa + (uint32_t)(((lc ^ ((i >> 1) & 3))) * 16));
#pragma unroll
                  for (int k = 0; k < 4; ++k) {
                    // tokens 64 h + 32 half + 8 k .. + 7: scale and zero pairs (broadcast reads)
                    const uint32_t off = (uint32_t)((half * 32 + 8 * k) * 2);
                    const uint4 sp = lds128(sc + off), zp = lds128(sc + 256 + off);
                    const uint32_t wk = k == 0 ? w.x : (k == 1 ? w.y : (k == 2 ? w.z : w.w));
                    put4(v, 16 * half + 4 * k, dequant8(wk, sp, zp));
                  }
                }
              }
            }
            if (any) {
              ptx::tmem_st32(tmem + lane_off + (uint32_t)(kAC + slot * kASlotCols + 32 * h), v);
              stored = true;
            }
          }
          if (stored) ptx::tmem_wait_st();
          // each thread's TMEM stores are complete; order them before the arrival
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&aux->slot_full[slot]);
          if (!is_v && tile == 0 && c == 0 && tracer) tc::trace_stamp(p.trace, 67);
        }
        __syncwarp();
        if (ok && lane == 0) ptx::mbar_arrive(&aux->raw_empty[rs]);
        if (tracer && tile == (is_v ? 0 : 1)) tc::trace_stamp(p.trace, is_v ? 69 : 68);
        if (tracer && is_v && tile == ntiles - 1) tc::trace_stamp(p.trace, 70);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
  span_end(p.span);
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

// keys before RoPE: the pair's fp32 query rows (rounded up to 1 KB), then the fp16 operand
int qf_bytes_for(const lr_cache_desc* d) {
  const int gh = d->n_kv_heads % 2 == 0 ? 2 : 1;
  const int rows = gh * (d->n_q_heads / d->n_kv_heads);
  return ((rows * kRD * 4 + 1023) / 1024) * 1024;
}

int q_bytes_for(const lr_cache_desc* d) {
  if (d->rope_in_kernel) return qf_bytes_for(d) + kGHMax * kQbHeadBytes;
  return ((d->rank_k + 63) / 64) * kQSubBytes;
}

struct I4Layout {
  int nraw, nb;   // raw slots (split evenly between the key and the value ring); B_k slots
  uint32_t raw_bytes, raw_params;
  size_t smem;
};

// Raw slots hold one side of one tile; as many as fit in 227 KB (up to 8, at least one per
// side; the keys get the smaller half) after the query
// rows and P, and for keys before RoPE the B_k ring (up to one tile's worth of sub-blocks,
// so the next tile's load while the current one is rotated).  The operand slots are in TMEM.
bool choose_layout(const lr_cache_desc* d, I4Layout* L) {
  const int G = std::max((d->rank_k + 31) / 32, (d->rank_v + 31) / 32);
  L->raw_params = (uint32_t)G * 2048u;
  L->raw_bytes = (uint32_t)G * 2560u;
  size_t fixed = (size_t)kAuxBytes + q_bytes_for(d) + 2 * kPBytes;
  L->nb = 0;
  if (d->rope_in_kernel) {
    const size_t bslot = (size_t)(d->n_kv_heads % 2 == 0 ? 2 : 1) * kSubBytes;
    const int kb = (d->rank_k + 63) / 64;
    const size_t base = fixed + 2 * (size_t)L->raw_bytes;
    if (base + 2 * bslot > (size_t)kSmemLimit) return false;
    L->nb = std::min(kNBMax, std::max(2, std::min(kb, (int)(((size_t)kSmemLimit - base) / bslot))));
    fixed += (size_t)L->nb * bslot;
  }
  const int nr = std::min(kMaxRaw, (int)(((size_t)kSmemLimit - fixed) / L->raw_bytes));
  if (nr < 2) return false;
  L->nraw = nr;
  L->smem = fixed + (size_t)nr * L->raw_bytes;
  return true;
}

int kv_per_cta(const lr_cache_desc* d) {
  if (!d->rope_in_kernel) return d->n_kv_heads;
  return d->n_kv_heads % 2 == 0 ? 2 : 1;
}

}  // namespace

bool tc_i4_supported(const lr_cache_desc* d) {
  if (d->quant_bits != 4 || d->quant_group != 32) return false;
  if (d->dtype != LR_BF16) return false;
  if (d->rank_v > 512) return false;
  if (!d->rope_in_kernel && d->n_q_heads > 32) return false;   // all query heads in one N = 32 MMA
  // keys before RoPE: d = 128 (the rotation pairs and the score MMA's K) and at most 16
  // query heads per KV head (the score MMA's N); other shapes take the CUDA-core path
  if (d->rope_in_kernel && (d->head_dim != kRD || d->n_q_heads / d->n_kv_heads > kMaxG)) return false;
  // keys before RoPE keep O~ in 128 TMEM columns next to K^: r_v <= 512 fits
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
      cudaError_t e = lr_dev_malloc(&st->bk16, (size_t)c->D * r_pad * 2);
      if (e != cudaSuccess) return e;
      st->r_pad = r_pad;
    }
    const long long n = (long long)c->D * r_pad;
    cudaError_t e = launch_serial(k_prep_bk16, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, s,
                                  reinterpret_cast<const __nv_bfloat16*>(c->B_k), reinterpret_cast<__half*>(st->bk16),
                                  d.rank_k, r_pad, c->D);
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
      cudaError_t e = lr_dev_malloc(&c->qt16, qbytes);
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
  p.wait_ns = c->wait_ns;
  p.row_len = c->row_len;
  p.span = span_of(c->spans, SPAN_DECODE);
  p.codes_k = c->codes_k;
  p.codes_v = c->codes_v;
  p.params_k = c->params_k;
  p.params_v = c->params_v;
  p.map = row_map(c);
  p.r_k = d.rank_k;
  p.r_v = d.rank_v;
  p.G_k = c->G_k;
  p.G_v = c->G_v;
  p.ck = (d.rank_k + 127) / 128;
  p.cv = (d.rank_v + 127) / 128;
  p.kb_k = (d.rank_k + 63) / 64;
  p.Hq = d.n_q_heads;
  p.hist_len = c->hist_len;
  p.stable_len = std::min(c->stable_len, c->hist_len);
  p.split_tokens = split_tokens;
  p.n_splits = n_splits;
  // operand slots: keys before RoPE 1 + 1 (K^ fills half of TMEM); rank space 2 + 3 (the
  // values' ring holds a whole tile for r_v <= 384)
  p.nks = rope ? 1 : 2;
  p.nvs = rope ? 1 : 3;
  p.nrk = st->nraw / 2;
  p.nrv = st->nraw - p.nrk;
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
  p.qf_bytes = rope ? (uint32_t)qf_bytes_for(&d) : 0u;
  p.nb = st->nb;
  // instantiation: 0 rank space; 1 keys before RoPE
  using Kern = void (*)(CUtensorMap, CUtensorMap, I4Params);
  static const Kern kerns[2] = {k_decode_tc_i4<false>, k_decode_tc_i4<true>};
  if (rope && p.gsz > kMaxG) return cudaErrorNotSupported;
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
  if (regs[ki].load() != (rope ? Cfg<true>::launch_regs : Cfg<false>::launch_regs))
    return cudaErrorInvalidConfiguration;
  const dim3 grid = rope ? dim3(d.n_kv_heads / p.gh, n_splits, d.batch) : dim3(n_splits, d.batch);
  return launch_pdl(kern, grid, dim3(rope ? Cfg<true>::threads : Cfg<false>::threads), st->smem, s, st->q, st->bk, p);
}
