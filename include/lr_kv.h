/*
 * lr_kv.h — C ABI of the low-rank KV-cache decode library (NVIDIA B200, sm_100a).
 *
 * What the library computes (the pages describe the method; no code is given):
 *   TraceKV: Policy-Preserving Low-Rank KV Cache Compression for Reasoning
 *   Vision-Language Models, abstract — the KV cache stores low-dimensional
 *   latents of the key/value states (Z_k = K A_k, Z_v = V A_v), optionally
 *   combined with quantization, and "optimized low-rank attention kernels" run
 *   decode on them; keys and values are recovered through shared bases
 *   (K ~ Z_k B_k, V ~ Z_v B_v).  The ai4snews digest, Perspective section, fixes
 *   the latency workload: Qwen2.5-VL-7B decode at batch 16, 4K-32K context.
 *   iS-KV: Online Low-Rank KV Cache Compression via Block-Incremental SVD,
 *   abstract and method section — an exact recent window next to the low-rank
 *   history, older tokens folded into latents as they leave the window, and
 *   stored historical coordinates synchronised when the basis changes.
 *
 * Notation (per layer): B batch, Hq query heads, Hkv KV heads, d head_dim,
 * D = Hkv*d, r_k / r_v latent ranks, T tokens.  One latent group spans all KV
 * heads: the latent of a token is z_k = k_cat A_k with k_cat in R^D the
 * concatenation of its KV heads.  Query head j reads KV head j / (Hq/Hkv).
 *
 * Conventions for every call:
 *   - Tensor pointers are DEVICE pointers owned by the caller, contiguous,
 *     row-major, borrowed only for the call (stream-ordered).  The cache owns
 *     its own device buffers and copies A and B at creation.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on that stream; argument and capacity errors are
 *     returned before anything is launched.  LR_ERR_CUDA reports a launch or
 *     runtime error (cudaGetLastError after the launch).
 *   - Element type of q, out, k, v, A, B, stored latents and the window is the
 *     cache dtype (LR_F32 or LR_BF16).  Latent fills are always fp32; basis-sync
 *     rotations are always fp32.
 *   - A cache is not thread-safe; calls on one cache must be serialised.
 */
#ifndef LR_KV_H
#define LR_KV_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum lr_status {
  LR_OK = 0,
  LR_ERR_INVALID_ARG = 1,   /* bad pointer, shape or combination of options      */
  LR_ERR_UNSUPPORTED = 2,   /* valid but not implemented for this configuration  */
  LR_ERR_CAPACITY = 3,      /* the cache is full                                  */
  LR_ERR_CUDA = 4,          /* a CUDA runtime / launch error                      */
  LR_ERR_OOM = 5,           /* device allocation failed                           */
  LR_ERR_TIMEOUT = 6        /* a bounded device-side wait gave up (see lr_device_error) */
} lr_status;

typedef enum lr_dtype { LR_F32 = 0, LR_BF16 = 1 } lr_dtype;

/* Kernel path selection for lr_attn_decode. */
typedef enum lr_path {
  LR_PATH_AUTO = 0,   /* tensor-core path where supported, else SIMT           */
  LR_PATH_SIMT = 1,   /* fp32 CUDA-core path (every configuration)             */
  LR_PATH_TC = 2      /* tcgen05 path: bf16 / int4 latents with keys after RoPE;
                         int4 latents with keys before RoPE when head_dim = 128,
                         Hq = 7 Hkv and Hkv is even (keys rebuilt per tile)     */
} lr_path;

/* Cache description.  All counts are per layer; one cache holds one layer. */
typedef struct lr_cache_desc {
  int32_t batch;          /* B >= 1                                               */
  int32_t n_q_heads;      /* Hq <= 128, a multiple of n_kv_heads, Hq/Hkv <= 64      */
  int32_t n_kv_heads;     /* Hkv >= 1, Hkv * head_dim <= 4096                       */
  int32_t head_dim;       /* d, a multiple of 8, <= 256                            */
  int32_t rank_k;         /* r_k, multiple of 16, 16..512                          */
  int32_t rank_v;         /* r_v, multiple of 16, 16..512                          */
  int32_t capacity;       /* max tokens per sequence (history + window)            */
  int32_t window;         /* exact recent window W (0 = none)                      */
  int32_t quant_bits;     /* 0 = latents stored in dtype; 4 = int4 group quant     */
  int32_t quant_group;    /* group size along the rank axis; must be 32 when quant_bits = 4 */
  int32_t dtype;          /* lr_dtype                                              */
  int32_t rope_in_kernel; /* 1 = keys were compressed before RoPE: rotate (rotate-half)
                             each reconstructed key at its absolute position        */
  double rope_theta;      /* RoPE base, e.g. 1e6                                   */
  float softmax_scale;    /* 0 -> 1/sqrt(head_dim)                                 */
  int32_t latent_groups;  /* 0 or 1: one latent group spans all KV heads; g > 1 (dividing
                             n_kv_heads): g groups of n_kv_heads / g heads, each with its own
                             latents of rank_k / rank_v and its own bases, so g = n_kv_heads
                             is one latent per KV head.  g * rank_k and g * rank_v <= 512.  */
  int32_t page_tokens;    /* 0: each sequence's latents are one contiguous run of rows;
                             128: paged latents (a pool of n_pages pages of 128 token rows,
                             sequence b's token t in page table[b][t / 128], row t % 128;
                             lr_cache_set_block_table).  Paged caches need capacity % 128 == 0
                             and window == 0.                                       */
  int32_t n_pages;        /* paged: pages in the pool, >= 1 (0: batch * capacity / 128);
                             must be 0 when page_tokens is 0                         */
  int32_t reserved[2];    /* must be zero                                          */
} lr_cache_desc;

typedef struct lr_cache lr_cache;   /* opaque */

/* Device pointers and strides of the cache's storage, for inspection.
 * Int4 latents are stored in blocks of 128 tokens (int4_blocks = ceil(capacity / 128) per
 * sequence; block k of sequence b is block n = b*int4_blocks + k), each side's block being
 * one contiguous run of groups*2 KB of codes and one of groups*512 B of params.
 * Keys, token-major inside a block (group-major):
 *   codes_k  [B][int4_blocks][groups][128][4] uint32: element e of group g of token t is
 *            in word (n*groups + g)*512 + (t%128)*4 + e/8, bits 4(e%8)..+3;
 *   params_k [B][int4_blocks][groups][128] uint32: word (n*groups + g)*128 + t%128, a pair
 *            of fp16 {scale (low half), zero (high half)}.
 * Values, rank-major inside a block:
 *   codes_v  [B][int4_blocks][groups*32][16] uint32: rank i (= 32g + e) of token t (u = t%128)
 *            is in word (n*groups*32 + i)*16 + 4*((u/32) ^ ((i/2)%4)) + (u%32)/8,
 *            bits 4m..+3 with m = 4*(u%2) + (u/2)%4 (tokens 2k and 2k+1 in nibbles k, k+4);
 *   params_v [B][int4_blocks][groups][256] fp16 (same bytes as params_k): half
 *            (n*groups + g)*256 + u is the scale, half (n*groups + g)*256 + 128 + u the zero.
 * Unquantised latents: z [B][capacity][rank] in dtype.
 * Paged caches (n_pages > 0): the B sequences of the layouts above become one pool of
 * n_pages pages (z [n_pages][128][rank]; int4: block n = page n), and token t of sequence b
 * is token t % 128 of page table[b][t / 128] (lr_cache_set_block_table).
 * Window ring: [B][window+1][D] in dtype; token t lives in slot t % (window+1). */
typedef struct lr_cache_view {
  void* z_k; void* z_v;                 /* unquantised latents or NULL            */
  uint32_t* codes_k; uint32_t* codes_v; /* int4 codes or NULL                     */
  uint32_t* params_k; uint32_t* params_v; /* int4 {scale, zero} or NULL           */
  void* win_k; void* win_v;             /* window ring or NULL                    */
  void* A_k; void* B_k; void* A_v; void* B_v;   /* current bases (dtype)         */
  int32_t groups_k, groups_v;           /* ceil(rank/32) for int4 caches, else 0 */
  int32_t capacity, window_slots;
  int32_t int4_blocks;                  /* 128-token blocks per sequence (int4), else 0 */
  int32_t n_pages;                      /* pages of a paged cache's pool, else 0  */
} lr_cache_view;

/* Decode plan (host arithmetic only; exposed for tests and tooling). */
typedef struct lr_plan {
  int32_t path;          /* lr_path actually used                                 */
  int32_t n_splits;      /* sequence splits per batch row (history part)          */
  int32_t tile_tokens;   /* tokens per tile                                       */
  int32_t split_tokens;  /* tokens per split (multiple of tile_tokens)            */
  int32_t ctas;          /* main-kernel CTAs                                      */
} lr_plan;

/* ---- lifetime -------------------------------------------------------------
 * lr_cache_create — allocate a cache for `desc` and copy the bases.
 *   A_k [D][r_k], B_k [r_k][D], A_v [D][r_v], B_v [r_v][D], device, dtype.
 *   With g = latent_groups > 1 the bases are given per group: A_k [g][D/g][r_k],
 *   B_k [g][r_k][D/g] (group i covers KV heads i*Hkv/g .. and ranks i*r_k ..); the cache
 *   stores them as one block-diagonal basis of rank g*r_k (A [D][g r_k], B [g r_k][D], zero
 *   outside the blocks), and every latent row holds the g groups' latents one after another
 *   ([g*r_k]).  Latent fills (lr_kv_append_latent) and the view then use the rank g*r_k.
 *   A_* may be NULL when the caller only fills latents (lr_kv_append then
 *   returns LR_ERR_INVALID_ARG).  Returns LR_ERR_INVALID_ARG / LR_ERR_UNSUPPORTED
 *   for bad descriptions before touching the device, LR_ERR_OOM if allocation
 *   fails.  All cache memory is zero-initialised.  Blocks until the copies end. */
lr_status lr_cache_create(const lr_cache_desc* desc, const void* A_k, const void* B_k,
                          const void* A_v, const void* B_v, void* stream, lr_cache** out);

/* lr_cache_destroy — synchronise the device and free all cache memory. NULL is a no-op. */
lr_status lr_cache_destroy(lr_cache* cache);

/* ---- append (TraceKV abstract: latents of the KV states, with quantization;
 *      iS-KV abstract: exact recent window, older states folded into latents) --
 * lr_kv_append — append one token per sequence.
 *   k, v: [B][D] in dtype (keys as compressed: before RoPE when rope_in_kernel),
 *   16-byte aligned (else LR_ERR_INVALID_ARG).
 *   Without a window: z = k A_k and z_v = v A_v are computed in fp32 and stored
 *   (rounded to dtype, or int4-quantised) at slot len.  With a window: the token
 *   goes to ring slot len % (W+1); if the window already held W tokens, its
 *   oldest token is first folded into history slot hist_len (z = k_old A).
 *   LR_ERR_CAPACITY when len == capacity. */
lr_status lr_kv_append(lr_cache* cache, const void* k, const void* v, void* stream);

/* lr_kv_append_rows — append one token per sequence, each row at its own slot (a serving
 *   batch whose sequences are at different lengths; read with lr_attn_decode_varlen).
 *   k, v: [B][D] in dtype, 16-byte aligned (else LR_ERR_INVALID_ARG).  pos: [B] int32,
 *   device: row b's latents z = k_b A_k, z_v = v_b A_v are stored (as lr_kv_append stores
 *   them) at history slot pos[b]; a row whose pos lies outside [0, capacity) writes nothing,
 *   and the other slots are untouched.  max_len (host): the history length becomes
 *   max(history length, max_len), the caller's bound on every row's pos + 1; 0 <= max_len
 *   <= capacity (LR_ERR_INVALID_ARG below, LR_ERR_CAPACITY above).  Caches with a window
 *   return LR_ERR_UNSUPPORTED.  Graph-capturable: pos is read on the device. */
lr_status lr_kv_append_rows(lr_cache* cache, const void* k, const void* v, const int32_t* pos,
                            int32_t max_len, void* stream);

/* lr_kv_prefill — append n tokens per sequence from their exact keys and values (a prompt).
 *   k, v: [B][n][D] in dtype, 16-byte aligned (else LR_ERR_INVALID_ARG).  Each token's latents
 *   z = k A_k, z_v = v A_v are computed in fp32 and stored at slots len .. len + n - 1
 *   (rounded to dtype, or int4-quantised), as n calls of lr_kv_append would store them up to
 *   the summation order of the fp32 projection.  bf16 caches with D a multiple of 64 compute
 *   the projection as one tensor-core GEMM per 128-token tile; others append token by token
 *   on CUDA cores.  Caches with a window return LR_ERR_UNSUPPORTED; LR_ERR_CAPACITY when
 *   len + n > capacity. */
lr_status lr_kv_prefill(lr_cache* cache, const void* k, const void* v, int32_t n, void* stream);

/* lr_kv_append_latent — bulk fill of n history tokens from given latents.
 *   z_k [B][n][r_k], z_v [B][n][r_v] fp32, device.  Stored rounded to dtype or
 *   int4-quantised (group 32, fp16 scale/zero; reading stated in the oracle).
 *   Requires an empty window (history tokens precede window tokens).
 *   LR_ERR_CAPACITY if len + n > capacity. */
lr_status lr_kv_append_latent(lr_cache* cache, const float* z_k, const float* z_v,
                              int32_t n, void* stream);

/* ---- decode (TraceKV abstract: low-rank attention kernels) ------------------
 * lr_attn_decode — one decode step of attention over all len cached tokens.
 *   q [B][Hq][d] (dtype; already rotated at position len-1 when keys carry
 *   RoPE), out [B][Hq][d] (dtype), lse [B][Hq] fp32 natural-log log-sum-exp of
 *   the scaled logits, or NULL.  Computes, for every query head j of KV head h:
 *   softmax over t of s * q_j . k^_t,h, then the weighted sum of v^_t,h, where
 *   k^, v^ are the latents reconstructed through B (RoPE-rotated if requested)
 *   for history tokens and the exact tokens for the window.  len == 0 returns
 *   LR_ERR_INVALID_ARG. */
lr_status lr_attn_decode(lr_cache* cache, const void* q, void* out, float* lse, void* stream);

/* lr_attn_decode_varlen — lr_attn_decode for a batch whose rows hold different numbers of
 *   tokens (a serving batch of sequences at different lengths): row b attends to its first
 *   row_len[b] history tokens only.  row_len: [B] int32, device, each in
 *   1..history length (values outside are clamped to that range); the cache itself is
 *   filled up to its common length, and the tokens of a row beyond its row_len are not
 *   read.  The sequence splits are planned for the longest row; splits past a row's end
 *   carry zero weight.  Caches with an exact window return LR_ERR_UNSUPPORTED. */
lr_status lr_attn_decode_varlen(lr_cache* cache, const void* q, void* out, float* lse,
                                const int32_t* row_len, void* stream);

/* ---- context sharding (a split of each sequence's context over GPUs; the pages'
 *      workload, TraceKV digest Perspective: batch 16 at up to 32K tokens) -----------
 * Several caches (typically one per GPU) hold consecutive slices of the same sequences'
 * context, with the same bases and query.  Each computes a partial result over its slice;
 * the partials are exchanged (e.g. an all-gather over NCCL) and merged by the log-sum-exp
 * rule, then projected once through B_v.  Caches with a window or with keys before RoPE
 * return LR_ERR_UNSUPPORTED (their tokens' positions are not the slice's own).
 * lr_attn_decode_partial — the decode of this cache's tokens up to, not including, the
 *   output projection: part_o [B][Hq][r_v] fp32 = sum_t 2^(s_t - m) z_v,t, part_ml
 *   [B][Hq][2] fp32 = (m, l = sum_t 2^(s_t - m)) with s_t = log2(e) * softmax_scale *
 *   q . k_t (the rank-space form of one slice's softmax).  len >= 1 (else
 *   LR_ERR_INVALID_ARG).
 * lr_merge_partials — out [B][Hq][d] (dtype) and lse [B][Hq] (natural log, or NULL) of the
 *   whole context from n partials: part_o [n][B][Hq][r_v], part_ml [n][B][Hq][2] fp32,
 *   device, as lr_attn_decode_partial writes them (shard order does not matter).  Uses this
 *   cache's B_v; n <= the cache's partial capacity (LR_ERR_CAPACITY). */
lr_status lr_attn_decode_partial(lr_cache* cache, const void* q, float* part_o, float* part_ml,
                                 void* stream);
lr_status lr_merge_partials(lr_cache* cache, int32_t n, const float* part_o, const float* part_ml,
                            void* out, float* lse, void* stream);

/* lr_decode_step — one whole decode step: lr_kv_append(k, v) then lr_attn_decode(q,
 *   out, lse), with identical arguments, results and errors, but with the projection
 *   of the new token and the projection of the query run in one launch. */
lr_status lr_decode_step(lr_cache* cache, const void* k, const void* v, const void* q, void* out,
                         float* lse, void* stream);

/* ---- basis sync (iS-KV abstract: historical coordinates synchronised with the
 *      updated basis) ---------------------------------------------------------
 * lr_basis_sync — Z_hist <- Z_hist R for the history latents of every sequence,
 *   then install new bases.  R_k [r_k][r_k], R_v [r_v][r_v] fp32 device (per group,
 *   [g][r_k][r_k] and the bases in the per-group form of lr_cache_create), or NULL
 *   to leave that side's latents unchanged; B_k_new, B_v_new, A_k_new, A_v_new
 *   (dtype) or NULL to keep the current basis.  For orthogonal R, passing
 *   B' = R^T B keeps every reconstructed key/value unchanged.  The window is
 *   untouched.  Unquantised caches only (int4: LR_ERR_UNSUPPORTED). */
lr_status lr_basis_sync(lr_cache* cache, const float* R_k, const float* R_v,
                        const void* B_k_new, const void* B_v_new, const void* A_k_new,
                        const void* A_v_new, void* stream);

/* ---- basis update (iS-KV title and method section: a dynamically updated low-rank
 *      basis kept current by a block-incremental SVD) ----------------------------------
 * lr_basis_update — one block update of a truncated SVD, the textbook form of the step the
 *   pages name: with the current basis rows B [r][D] of `side` (0 keys, 1 values) and the
 *   Gram matrix S = Z^T Z of the history coordinates (Z = K_hist B^T), and a block of exact
 *   rows K [n][D]: Y = K B^T, the residual P = K - Y B with orthonormal rows Q^T spanning it
 *   (numerical rank: directions below 1e-6 of the block's largest row norm are dropped),
 *   G = [[S + Y^T Y, Y^T Rp^T], [Rp Y, Rp Rp^T]] with Rp^T = P Q, and its r leading
 *   eigenpairs (lam, V):  B' = V^T [B; Q^T],  R = V[:r, :],  S' = diag(lam).
 *   B' spans the leading right singular subspace of [Z B; K] (Eckart-Young).
 *   blk [n][D] dtype device, 16-byte aligned, 1 <= n <= 128 (else LR_ERR_INVALID_ARG).
 *   gram [r][r] fp32 device: S on entry, S' on return.  R_out [r][r] fp32 device: the
 *   history sync Z <- Z R, to be passed to lr_basis_sync with B' (and A').  B_new [r][D]
 *   and A_new = B'^T [D][r] in dtype, device, or NULL.  The current basis must have
 *   orthonormal rows (A = B^T).  Computed in fp64 on the GPU; the cache's latents are not
 *   touched.  One latent group only (else LR_ERR_UNSUPPORTED).  Eigenvector signs follow a
 *   fixed rule (the largest-magnitude entry of each column of V positive). */
lr_status lr_basis_update(lr_cache* cache, int32_t side, const void* blk, int32_t n, float* gram,
                          float* R_out, void* B_new, void* A_new, void* stream);

/* ---- decode without device allocation ----------------------------------------
 * (No counterpart on the pages; this entry point exists for callers that cannot
 * allocate device memory at decode time: serving engines that reserve almost all HBM
 * up front for their own pools, and latency-critical loops that cannot take the
 * implicit device synchronisation of cudaMalloc.)
 * lr_attn_decode_noalloc — the decode of lr_attn_decode, computed on the fp32
 *   CUDA-core path over caller-owned unquantised latents, without allocating: its
 *   working memory (query latents and per-split partial results) is one static device
 *   array of LR_NOALLOC_SCRATCH_BYTES that every GPU loading this library holds until
 *   process exit.
 *   desc: as for lr_cache_create, with window 0, quant_bits 0, rope_in_kernel 0, one
 *     latent group and page_tokens 0 (otherwise LR_ERR_UNSUPPORTED); len: tokens to attend, 1..capacity.
 *   z_k [B][capacity][r_k], z_v [B][capacity][r_v]: latents in the cache layout;
 *   B_k [r_k][D], B_v [r_v][D], q [B][Hq][d], out [B][Hq][d]: dtype, device;
 *   B_k and B_v 16-byte aligned (else LR_ERR_INVALID_ARG, before any launch);
 *   lse [B][Hq] fp32 or NULL.  The first kernel starts only after the work before the
 *   call on `stream` has completed, so that work may write the bases and the query.
 *   Uses fewer sequence splits when needed to fit the array, and returns
 *   LR_ERR_CAPACITY when even one split's working set exceeds it
 *   (4 * B * Hq * (r_k + r_v + 2) bytes > LR_NOALLOC_SCRATCH_BYTES).
 *   The first call on a device looks up the array's device address with that device
 *   current (cudaGetSymbolAddress); make that first call outside any stream capture.
 *   Every call overwrites the parts of the array it reads, so nothing carries over
 *   between calls; but all calls share the one array, so calls whose kernels can
 *   overlap on the GPU (unordered streams) race and corrupt each other's results. */
#define LR_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
lr_status lr_attn_decode_noalloc(const lr_cache_desc* desc, int32_t len, const void* z_k,
                                 const void* z_v, const void* B_k, const void* B_v,
                                 const void* q, void* out, float* lse, void* stream);

/* ---- bookkeeping ------------------------------------------------------------ */
/* Current total length, history length and window length (host-side counters). */
lr_status lr_cache_get_len(const lr_cache* cache, int32_t* len, int32_t* hist_len,
                           int32_t* win_len);
/* Drop tokens at positions >= len (no device work).  Caches with a window can drop only
 * the token of the last lr_kv_append / lr_decode_step (len = current length - 1; the
 * ring's spare slot still holds the token that append folded out of the window);
 * anything else returns LR_ERR_UNSUPPORTED. */
lr_status lr_cache_truncate(lr_cache* cache, int32_t len);
/* Device pointers of the storage (see lr_cache_view). */
lr_status lr_cache_view_get(const lr_cache* cache, lr_cache_view* out);
/* lr_cache_set_block_table — the page of every 128-token span of every sequence of a paged
 *   cache (page_tokens = 128).  Paging is a storage layout only (the method fixes what is
 *   computed per token, not where a token's latent row lives): every result equals that
 *   of a contiguous cache holding the same latents.
 *   table: host, [batch][capacity / 128] int32, each entry in [0, n_pages); the library
 *   checks every entry (LR_ERR_INVALID_ARG, nothing changed, if one is out of range or
 *   table is NULL) and copies the table to the device on `stream` (ordered after the work
 *   before the call there, so a decode queued earlier still reads the old table); the
 *   caller's array is no longer read once the call returns.  Not capturable in a CUDA
 *   graph (a copy from pageable memory).
 *   Sequences may share pages (a common prefix); an append into a shared page writes it
 *   for every sequence that maps it.  The rows of a page keep their contents when the
 *   table changes.  A new cache's table maps span j of sequence b to page
 *   (b * capacity / 128 + j) % n_pages.  LR_ERR_UNSUPPORTED for a cache that is not paged.
 *   With paging, lr_kv_prefill, lr_kv_append_latent, lr_decode_step and every decode call
 *   work as for contiguous caches; lr_basis_sync rotates every row of the pool (each page
 *   once, whatever maps it). */
lr_status lr_cache_set_block_table(lr_cache* cache, const int32_t* table, void* stream);
/* lr_cache_set_block_table_device — the same from a DEVICE array (int32, any alignment),
 *   copied device to device on `stream`, so that a serving loop can update the
 *   table inside a captured CUDA graph.  The library cannot check the entries without a host
 *   round trip: every kernel clamps a page index outside [0, n_pages) into the pool, so a bad
 *   entry gives wrong outputs for its sequence but never an access outside the cache's
 *   storage.  The caller's array must stay valid until the copy has run.
 *   LR_ERR_UNSUPPORTED for a cache that is not paged; LR_ERR_INVALID_ARG for NULL. */
lr_status lr_cache_set_block_table_device(lr_cache* cache, const int32_t* table, void* stream);
/* Force a decode path (LR_PATH_*) and/or a split count (0 = automatic). */
lr_status lr_cache_set_path(lr_cache* cache, int32_t path, int32_t n_splits);
/* The plan lr_attn_decode would use at the current length. */
lr_status lr_cache_plan(const lr_cache* cache, lr_plan* out);
/* Host-only planner: the plan for `desc` at length len on a GPU with num_sms SMs. */
lr_status lr_plan_decode(const lr_cache_desc* desc, int32_t len, int32_t num_sms,
                         int32_t path, int32_t n_splits, lr_plan* out);
/* Synchronise the cache's last stream and read its device error word
 * (0 = none; otherwise an LR_ERR_* code a kernel recorded, e.g. LR_ERR_TIMEOUT
 * from a bounded wait).  Clears the word. */
lr_status lr_device_error(lr_cache* cache, int32_t* code);
/* Record caller-owned CUDA events (cudaEvent_t passed as void*) immediately before and
 * after the main decode kernel (the split-sequence attention kernel) of every following
 * lr_attn_decode on this cache, on the call's stream, so that the kernel alone can be
 * timed; both NULL to stop.  The events must stay valid while set. */
lr_status lr_cache_set_kernel_events(lr_cache* cache, void* ev_start, void* ev_stop);
/* Timeline trace of the tensor-core decode kernel: when buf (device, capacity_words
 * 64-bit words >= LR_TRACE_SLOTS * batch * max splits + LR_TRACE_SPAN_WORDS) is set, every
 * CTA of each following decode writes %globaltimer stamps (ns) to
 * buf[((b * n_splits) + split) * LR_TRACE_SLOTS + slot]: 0 start, 1 set-up done,
 * 2 query latents in shared memory, 3+4i key tile i consumed, 4+4i its scores read,
 * 5+4i its probabilities written, 6+4i its value mix issued (tiles i < 16), 71 end.
 * The last LR_TRACE_SPAN_WORDS words hold kernel spans, as pairs (earliest CTA start,
 * latest CTA end) for: 0 the append / query projection kernel, 1 the split-sequence decode,
 * 2 the exact window, 3 the split merge; the caller sets each pair to (~0, 0) before a call
 * whose spans it wants.  (The max split count is the larger of 64 and two CTAs per SM
 * spread over the batch, capped at one split per 16 tokens of capacity.)
 * NULL stops tracing.  LR_ERR_CAPACITY if buf is too small. */
#define LR_TRACE_SLOTS 72
#define LR_TRACE_SPAN_WORDS 8
lr_status lr_cache_set_trace(lr_cache* cache, uint64_t* buf, int64_t capacity_words);
/* ---- failure testing (no counterpart on the pages) ----------------------------
 * lr_cache_set_wait_limit — limit, in nanoseconds, of every bounded wait inside this
 *   cache's tensor-core kernels (decode and basis sync); 0 restores the default (2 s).
 *   A wait that gives up makes its kernel record LR_ERR_TIMEOUT in the device error word
 *   (lr_device_error), finish its own copies and MMAs, free its tensor memory and return;
 *   that call's outputs are then undefined, the cache's contents are untouched.  For
 *   tests of that path: a limit of a few nanoseconds makes the first wait that is not
 *   already satisfied give up.  LR_ERR_INVALID_ARG for ns < 0. */
lr_status lr_cache_set_wait_limit(lr_cache* cache, int64_t ns);

/* lr_debug_inject_fault — make the library's next-but-`after` device allocation
 *   (kind LR_FAULT_ALLOC) or kernel launch (LR_FAULT_LAUNCH) fail without allocating or
 *   launching: `after` operations of that kind still succeed, the one after them fails,
 *   then the fault disarms itself; after = -1 disarms.  Process-wide.  The failing call
 *   returns LR_ERR_OOM (allocation) or LR_ERR_CUDA (launch); lr_cache_create frees what
 *   it had allocated.  A failed launch inside lr_decode_step can leave the appended token
 *   in the cache (its length then counts it).  LR_ERR_INVALID_ARG for another kind or
 *   after < -1. */
#define LR_FAULT_ALLOC 0
#define LR_FAULT_LAUNCH 1
lr_status lr_debug_inject_fault(int32_t kind, int64_t after);

/* sizeof(lr_cache_desc), sizeof(lr_cache_view), sizeof(lr_plan) as compiled (binding checks). */
void lr_abi_struct_sizes(int32_t* desc_size, int32_t* view_size, int32_t* plan_size);
/* Human-readable name of a status. */
const char* lr_status_string(lr_status status);
/* Number of kernel launches this library issued since load (all caches). */
int64_t lr_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* LR_KV_H */
