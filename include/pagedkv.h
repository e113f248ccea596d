/*
 * pagedkv.h -- C ABI of libpagedkv.so: paged KV-cache append and paged
 * single-query (decode) attention on NVIDIA B200 (sm_100a).
 *
 * The KV cache of one attention layer is a flat pool of fixed-size physical
 * blocks of `block_size` tokens; a sequence reaches its tokens through a block
 * table whose entry i names the physical block that holds its logical block i
 * ("Transformer anatomy", ch. 15 §15.5, PagedAttention: blocks of typically 16
 * tokens, per-sequence block table, append into the current block;
 * "LLM Primer VI", ch. 8 §8.1: a flat physical pool, the attention kernel takes
 * the block table as an extra input and fetches K and V indirectly by index).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Tensors are dense, row-major, and live in device memory of the current CUDA
 * device unless stated otherwise.  The caller owns every buffer; the library
 * keeps no pointer after a call returns.
 *
 *   k_cache, v_cache : [num_blocks][n_kv_heads][block_size][head_dim]
 *                      (within a block, one contiguous block_size x head_dim
 *                      tile per kv head)
 *   block_tables     : int32 [batch][max_blocks_per_seq]; entries past a
 *                      sequence's last block are never read
 *   context_lens     : int32 [batch]; tokens of each sequence, counting the
 *                      token appended in this step
 *   q, out           : [batch][n_q_heads][head_dim], same dtype as the caches
 *   slot_mapping     : int64 [num_tokens]; slot = block * block_size + offset
 *
 * Query head h reads kv head h / (n_q_heads / n_kv_heads) (grouped-query
 * attention with contiguous groups, "Transformer anatomy" ch. 15 §15.2 and
 * §15.7: h_kv < h_q).
 *
 * Supported: block_size == 16; head_dim in {64, 128}; n_q_heads a multiple of
 * n_kv_heads; dtype f32, f16 or bf16 (the same for q, caches and out); all
 * pointers 16-byte aligned; batch <= PKV_MAX_BATCH.
 *
 * Calls are asynchronous: they enqueue work on `stream` (a cudaStream_t; NULL
 * is the legacy default stream) and return.  Work enqueued on one stream runs
 * in order, so an append followed by a decode on the same stream sees the
 * appended token.
 *
 * Errors: arguments are checked on the host before anything is enqueued; a
 * failed check returns a status and enqueues nothing.  Values that only the
 * device sees (block ids, context lengths, slots) are range-checked by the
 * kernels: a bad value sets a bit in a per-device error word (read and cleared
 * by pkv_get_device_error), the offending access is skipped (a block whose
 * id is out of range contributes no token to any softmax; a row that is left
 * with no token is a zero row), and the kernel never traps.  No entry point
 * aborts the process.
 */
#ifndef PAGEDKV_H_
#define PAGEDKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PKV_MAX_BATCH 4096

typedef enum pkv_dtype {
  PKV_F32 = 0,
  PKV_F16 = 1,
  PKV_BF16 = 2
} pkv_dtype;

typedef enum pkv_status {
  PKV_OK = 0,
  PKV_ERR_INVALID_ARG = 1,   /* null pointer, negative size, misaligned pointer, n_q % n_kv != 0 */
  PKV_ERR_UNSUPPORTED = 2,   /* block_size, head_dim, dtype or batch outside the supported set */
  PKV_ERR_OUT_OF_RANGE = 3,  /* a kernel saw a bad block id, context length or slot */
  PKV_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  PKV_ERR_WORKSPACE = 5,     /* workspace too small */
  PKV_ERR_NO_BLOCKS = 6,     /* block manager: not enough free or evictable blocks (nothing changed) */
  PKV_ERR_HOST_MEMORY = 7    /* block manager: host allocation failed (the manager must be destroyed) */
} pkv_status;

/* Bits of the device error word (pkv_get_device_error). */
#define PKV_DEVERR_BLOCK_ID 0x1u   /* block table entry outside [0, num_blocks): nothing was read from
                                      it and its tokens were left out of the softmax */
#define PKV_DEVERR_CONTEXT 0x2u    /* context length < 0 or > max_blocks_per_seq * block_size: clamped */
#define PKV_DEVERR_SLOT 0x4u       /* slot >= num_blocks * block_size: the token was not written */
#define PKV_DEVERR_TIMEOUT 0x8u    /* a bounded in-kernel wait (2 s by default) gave up: that launch's
                                      output is undefined (the kernel drained its own copies and ended) */
#define PKV_DEVERR_SCHEDULE 0x10u  /* the decode workspace was not zero-filled before its first use: that
                                      launch's result is wrong (the workspace is zeroed again) */

/*
 * paged_kv_append -- write the K/V of new tokens into their cache slots.
 *
 * For each token i with s = slot_mapping[i] >= 0 and every kv head h:
 *   k_cache[s / block_size][h][s % block_size][:] = k[i][h][:]
 *   v_cache[s / block_size][h][s % block_size][:] = v[i][h][:]
 * ("Transformer anatomy" ch. 15 §15.5: a new token goes into the current
 * block; §15.1: its K and V are concatenated onto the cache).  A negative slot
 * marks a padding token and is skipped.  A slot >= num_blocks * block_size is
 * skipped and sets PKV_DEVERR_SLOT.  The copy is bit-exact.  Two tokens with
 * the same slot race (one of them wins).
 *
 *   k, v          : device, [num_tokens][n_kv_heads][head_dim], dtype
 *   slot_mapping  : device, int64 [num_tokens]
 *   k_cache, v_cache : device, layout above; written in place
 *   stream        : cudaStream_t
 */
pkv_status paged_kv_append(const void* k, const void* v, const int64_t* slot_mapping,
                           int32_t num_tokens, void* k_cache, void* v_cache,
                           int32_t num_blocks, int32_t block_size, int32_t n_kv_heads,
                           int32_t head_dim, pkv_dtype dtype, void* stream);

/*
 * paged_attention_workspace_size -- device scratch bytes that
 * paged_attention_decode needs on the current device for this shape (the
 * partial softmax states of split contexts and their merge metadata).  The
 * result depends on the device's SM count, not on context lengths.
 */
pkv_status paged_attention_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                          int32_t head_dim, pkv_dtype dtype, size_t* bytes);

typedef struct pkv_decode_options pkv_decode_options;

/* The same for paged_attention_decode_ex with `options` (NULL = defaults):
 * balancing chunks need (1 + balance_chunks) times the records. */
pkv_status paged_attention_workspace_size_ex(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                             int32_t head_dim, pkv_dtype dtype,
                                             const pkv_decode_options* options, size_t* bytes);

/*
 * paged_attention_decode -- single-query attention through the block table.
 *
 * For every sequence b and query head h, with kv = h / (n_q_heads / n_kv_heads),
 * n = context_lens[b], and K_j, V_j the rows of logical token j found at
 * block_tables[b][j / block_size], slot j % block_size, kv head kv:
 *   s_j = scale * <q[b][h], K_j>,  out[b][h] = sum_j softmax(s)_j V_j
 * ("KV Cache and PagedAttention" (gyaansetu): dot Q with all K, weights,
 * weighted sum of V; "PagedAttention: KV cache memory management" (yfxerp)
 * §3.2: the per-page loop, read as one softmax over the whole context).
 * n == 0 gives a zero row.  Scores, softmax and accumulation are fp32; the
 * result is rounded to the dtype (round to nearest even).
 *
 * Long contexts are split across work units (split-KV) and merged with a
 * log-sum-exp reduction.  The result is bit-for-bit independent of where the
 * blocks sit in the pool and of whether blocks are shared between sequences;
 * it depends, within rounding, on the split chosen for the device.
 *
 *   workspace     : device scratch of at least paged_attention_workspace_size()
 *                   bytes, 256-byte aligned, owned by the caller and not
 *                   shared by two calls in flight at once.  Used with
 *                   balancing chunks (paged_attention_decode_ex), it must be
 *                   zero-filled before its first use; every call leaves it
 *                   ready for the next (one that was not cleared gives a
 *                   wrong result for that call and sets PKV_DEVERR_SCHEDULE).
 *                   NULL makes the library take a stream-ordered allocation
 *                   for this call (cudaMallocAsync / cudaFreeAsync on
 *                   `stream`)
 *   workspace_bytes : size of `workspace`
 */
pkv_status paged_attention_decode(const void* q, const void* k_cache, const void* v_cache,
                                  const int32_t* block_tables, int32_t max_blocks_per_seq,
                                  const int32_t* context_lens, int32_t batch, int32_t num_blocks,
                                  float scale, int32_t n_q_heads, int32_t n_kv_heads,
                                  int32_t head_dim, int32_t block_size, void* out, pkv_dtype dtype,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * paged_kv_append_and_decode -- one decode step in one launch: the result of
 * paged_kv_append(k, v, slot_mapping, num_tokens, k_cache, v_cache, ...)
 * followed by paged_attention_decode(q, k_cache, v_cache, ...) on the same
 * stream, bit for bit, in the cache and in `out` ("Transformer anatomy"
 * ch. 15 §15.1: the new token's K and V join the cache, then its query
 * attends over all of it; §15.5: the new token goes into its slot of the
 * current block).
 *
 * Every CTA of the decode kernel first writes its share of the new rows into
 * their slots (a negative slot is skipped; one >= num_blocks * block_size is
 * skipped and sets PKV_DEVERR_SLOT); a grid-wide barrier then orders those
 * writes before the first K/V tile is read.  This saves the separate append
 * launch and the gap between the two kernels.  Arguments are those of the
 * two calls (k, v: [num_tokens][n_kv_heads][head_dim] of `dtype`); the
 * workspace rules are paged_attention_decode's.  batch == 0 runs the append
 * alone.
 */
pkv_status paged_kv_append_and_decode(const void* q, const void* k, const void* v,
                                      const int64_t* slot_mapping, int32_t num_tokens, void* k_cache,
                                      void* v_cache, const int32_t* block_tables,
                                      int32_t max_blocks_per_seq, const int32_t* context_lens,
                                      int32_t batch, int32_t num_blocks, float scale, int32_t n_q_heads,
                                      int32_t n_kv_heads, int32_t head_dim, int32_t block_size, void* out,
                                      pkv_dtype dtype, void* workspace, size_t workspace_bytes,
                                      void* stream);

/*
 * paged_attention_decode_cascade -- paged_attention_decode for batches whose
 * sequences share prefix blocks (prefix caching: sequences that start with the
 * same block-aligned tokens point their tables at the same physical blocks,
 * "Transformer anatomy" ch. 15 §15.6; refcounted block sharing for parallel
 * sampling and prefix caching, "LLM Primer VI" ch. 8 §8.1 and §8.3).
 *
 * Group i owns a shared prefix of prefix_lens[i] tokens (a multiple of
 * block_size) held by blocks prefix_block_tables[i][0 .. prefix_lens[i]/16).
 * Sequence b with g = seq_group[b] >= 0 has the context "prefix of group g"
 * followed by its private suffix of context_lens[b] tokens, held by
 * block_tables[b][..]; seq_group[b] = -1 means no shared prefix (context_lens
 * and block_tables then cover the whole context).  The result equals
 * paged_attention_decode over the concatenated tables, within rounding.
 *
 * The prefix is read once per (group, kv head) and evaluated as one dense
 * attention over all member rows on tensor cores; the suffixes go through the
 * decode kernel, which continues from each row's prefix state.  16-bit dtypes
 * only (PKV_F32 returns PKV_ERR_UNSUPPORTED).  A group id >= n_groups or a bad
 * prefix length sets PKV_DEVERR_CONTEXT.
 *
 *   prefix_block_tables : device, int32 [n_groups][max_prefix_blocks]
 *   prefix_lens, seq_group : device, int32 [n_groups], [batch]
 *   workspace : at least paged_attention_cascade_workspace_size() bytes (or
 *               NULL for a stream-ordered allocation), 256-byte aligned
 */
pkv_status paged_attention_cascade_workspace_size(int32_t batch, int32_t n_q_heads, int32_t n_kv_heads,
                                                  int32_t head_dim, pkv_dtype dtype, size_t* bytes);

pkv_status paged_attention_decode_cascade(const void* q, const void* k_cache, const void* v_cache,
                                          int32_t n_groups, const int32_t* prefix_block_tables,
                                          int32_t max_prefix_blocks, const int32_t* prefix_lens,
                                          const int32_t* seq_group, const int32_t* block_tables,
                                          int32_t max_blocks_per_seq, const int32_t* context_lens,
                                          int32_t batch, int32_t num_blocks, float scale,
                                          int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                          int32_t block_size, void* out, pkv_dtype dtype,
                                          void* workspace, size_t workspace_bytes, void* stream);

/* Tuning and test hooks for paged_attention_decode_cascade_ex. Zero-initialise. */
typedef struct pkv_cascade_options {
  int32_t prefix_splits; /* 0: default; 1..4: CTAs (one thread-block cluster) per 128-row prefix
                            tile, each taking an equal share of the prefix, merged in the
                            cluster's rank 0 through distributed shared memory (tensor-memory
                            prefix kernel only) */
  int32_t prefix_kernel; /* 0: default (tensor-memory kernel for head_dim 128, else the mma.sync
                            kernel); 1: tensor-memory kernel (PKV_ERR_UNSUPPORTED where it does
                            not apply); 2: mma.sync kernel */
  int32_t reserved[6];   /* must be zero */
} pkv_cascade_options;

/* paged_attention_decode_cascade with options (NULL options = the default). */
pkv_status paged_attention_decode_cascade_ex(const void* q, const void* k_cache, const void* v_cache,
                                             int32_t n_groups, const int32_t* prefix_block_tables,
                                             int32_t max_prefix_blocks, const int32_t* prefix_lens,
                                             const int32_t* seq_group, const int32_t* block_tables,
                                             int32_t max_blocks_per_seq, const int32_t* context_lens,
                                             int32_t batch, int32_t num_blocks, float scale,
                                             int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                             int32_t block_size, void* out, pkv_dtype dtype,
                                             void* workspace, size_t workspace_bytes, void* stream,
                                             const pkv_cascade_options* options);

/* Tuning and test hooks for paged_attention_decode_ex. Zero-initialise. */
struct pkv_decode_options {
  int32_t num_units;   /* 0: default split (one work unit per consumer warp on every SM);
                          n > 0: use at most n work units (n = 1 computes every row in one
                          unit, with no split and no merge) */
  int32_t force_simt;  /* 1: CUDA-core path even where the tensor-core path applies */
  int32_t balance_chunks;  /* 0: none (default: every unit runs exactly its own tile range);
                              1..4: balancing chunks cut from the end of each unit's range and
                              claimed at run time by the first warps to run out of work.  The
                              result stays deterministic.  Needs the larger workspace of
                              paged_attention_workspace_size_ex, zero-filled before first use.
                              Measured on B200 it costs more than the imbalance it removes */
  int32_t static_permille; /* 0: default (800); 500..999: share of its range a unit keeps */
  int32_t wait_limit_us;   /* 0: default (2 s); n > 0: every bounded wait of this launch gives up
                              after n microseconds (with PKV_DEVERR_TIMEOUT) */
  int32_t test_withhold_unit; /* test hook for the failure path. 0: off; u + 1: the producer never
                                 issues the copies of work unit u (u < the unit count), so that
                                 its consumer's bounded wait runs out: the launch returns with
                                 PKV_DEVERR_TIMEOUT set and writes no defined result, and the
                                 next call is unaffected.  Nothing faults or hangs */
  int32_t reserved[2]; /* must be zero */
};

/* paged_attention_decode with options (NULL options = paged_attention_decode). */
pkv_status paged_attention_decode_ex(const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* context_lens, int32_t batch,
                                     int32_t num_blocks, float scale, int32_t n_q_heads,
                                     int32_t n_kv_heads, int32_t head_dim, int32_t block_size,
                                     void* out, pkv_dtype dtype, void* workspace,
                                     size_t workspace_bytes, void* stream,
                                     const pkv_decode_options* options);

/*
 * paged_attention_decode_noalloc -- paged_attention_decode for callers that
 * cannot allocate device memory.  (The pages have no counterpart: this entry
 * point is an addition of this library.)
 *
 * Some callers cannot call cudaMalloc or any allocator: a plugin whose host
 * framework owns all device memory and hands it no allocator, a serving loop
 * that must never allocate on its hot path (an allocation can synchronise the
 * device and stall every stream), or a process that has already given all
 * free memory to its KV-cache pool.  This entry point takes the same inputs
 * and outputs as paged_attention_decode, minus the workspace, and allocates
 * nothing: the scratch for split contexts lives in one file-scope device array
 * of PKV_STATIC_WORKSPACE_BYTES (24 MiB), which every GPU that loads the
 * library holds until the process exits.
 *
 * - Sizes whose scratch (paged_attention_workspace_size) exceeds the array
 *   are rejected with PKV_ERR_WORKSPACE before anything is enqueued.  On a
 *   148-SM B200 every supported shape fits.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current and caches it; make that
 *   first call before any stream capture.
 * - Every call on a device shares the one array and it keeps the last call's
 *   contents.  The array starts zero-filled and every call leaves its
 *   scheduling counter at zero again.  Calls whose work overlaps on the GPU
 *   (on different streams, or from several host threads without ordering)
 *   race on the array and give wrong results: order them.
 * Results are bit-identical to paged_attention_decode with its default split.
 */
#define PKV_STATIC_WORKSPACE_BYTES (24u * 1024u * 1024u)

pkv_status paged_attention_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                          const int32_t* block_tables, int32_t max_blocks_per_seq,
                                          const int32_t* context_lens, int32_t batch, int32_t num_blocks,
                                          float scale, int32_t n_q_heads, int32_t n_kv_heads,
                                          int32_t head_dim, int32_t block_size, void* out,
                                          pkv_dtype dtype, void* stream);

/*
 * paged_kv_copy_blocks -- copy whole physical blocks inside the pool, both
 * caches: for p in [0, n_pairs),
 *   k_cache[dst[p]] = k_cache[src[p]],  v_cache[dst[p]] = v_cache[src[p]]
 * (every kv head, token and dim of the block).  This is the copy of
 * copy-on-write: a block shared by several block tables ("LLM Primer VI"
 * ch. 8 §8.1, refcounted sharing for parallel sampling) that one of them is
 * about to append to is first duplicated into a fresh block.  pkv_bm_append
 * emits the pairs; run this copy before paged_kv_append writes the new token.
 * The copy is bit-exact.  A dst block must not appear twice nor be a src of
 * the same call (the pairs would race).  A src or dst outside [0, num_blocks)
 * skips that pair and sets PKV_DEVERR_BLOCK_ID.
 *
 *   src_blocks, dst_blocks : device, int32 [n_pairs]
 *   k_cache, v_cache       : device, [num_blocks][n_kv_heads][block_size][head_dim], dtype
 *   stream                 : cudaStream_t
 */
pkv_status paged_kv_copy_blocks(void* k_cache, void* v_cache, const int32_t* src_blocks,
                                const int32_t* dst_blocks, int32_t n_pairs, int32_t num_blocks,
                                int32_t block_size, int32_t n_kv_heads, int32_t head_dim,
                                pkv_dtype dtype, void* stream);

/* ------------------------------------------------------------------------
 * Host block manager (pkv_bm_*): the allocator that produces the block tables
 * and slot mappings the kernels above consume.  Pure host code; no call
 * touches the GPU.  Not thread-safe: one manager per scheduler thread.
 *
 * Model ("Transformer anatomy" ch. 15 §15.5): a pool of num_blocks physical
 * blocks of block_size tokens; every sequence owns a block table; a new token
 * goes into the sequence's last block, and a new block is taken from the free
 * pool when that block is full; freeing a sequence returns its blocks.
 * Blocks are refcounted so that several tables can point at one block
 * ("LLM Primer VI" ch. 8 §8.1): pkv_bm_fork shares all blocks of a sequence,
 * and an append into a shared, partly filled last block first moves the
 * appending sequence onto a private copy (copy-on-write).
 *
 * Prefix caching ("Transformer anatomy" ch. 15 §15.6; "LLM Primer VI" ch. 8
 * §8.3): when enabled, each full prompt block is keyed by a hash that the
 * caller supplies (pkv_bm_hash_blocks computes the chained hash used by the
 * tests: block i's key covers all tokens up to the end of block i).  A new
 * sequence whose leading block keys are cached shares those blocks and
 * reports how many prompt tokens need no prefill.  A cached block whose
 * refcount drops to 0 stays cached and evictable; eviction takes the least
 * recently released one.  Partly filled blocks are never cached.
 *
 * Determinism: a new block is the lowest-numbered free block; if none is
 * free, the least recently released cached block is evicted (its key is
 * dropped).  pkv_bm_free releases a sequence's blocks from its last block to
 * its first, so a prefix outlives its own suffix in the LRU order.
 *
 * Every call validates first and changes nothing when it returns an error.
 * ------------------------------------------------------------------------ */
typedef struct pkv_block_manager pkv_block_manager;

typedef struct pkv_bm_stats_t {
  int32_t num_blocks;
  int32_t free_blocks;         /* refcount 0 and not cached */
  int32_t cached_idle_blocks;  /* refcount 0, cached, evictable (LRU list) */
  int32_t used_blocks;         /* refcount > 0 */
  int32_t cached_blocks;       /* blocks holding a prefix-cache key, used or idle */
  int32_t sequences;
  int64_t tokens;              /* sum of sequence lengths */
  int64_t allocated_slots;     /* sum over sequences of table length * block_size */
} pkv_bm_stats_t;

/* Create a manager over blocks [0, num_blocks).  enable_prefix_cache != 0
 * turns the hash-keyed prefix cache on.  *out is owned by the caller and
 * released with pkv_bm_destroy. */
pkv_status pkv_bm_create(int32_t num_blocks, int32_t block_size, int32_t enable_prefix_cache,
                         pkv_block_manager** out);
void pkv_bm_destroy(pkv_block_manager* bm);

/* Chained block keys of a prompt: for every full block i of `tokens`
 * (n_tokens / block_size of them), hashes[i] = FNV-1a 64 over the 8
 * little-endian bytes of the previous key (seed for i = 0) followed by the
 * block's tokens as little-endian int32.  hashes: host, n_tokens / block_size
 * entries. */
pkv_status pkv_bm_hash_blocks(const int32_t* tokens, int64_t n_tokens, int32_t block_size, uint64_t seed,
                              uint64_t* hashes);

/* Add a sequence holding n_prompt_tokens tokens (ceil(n / block_size)
 * blocks).  block_hashes (host, n_prompt_tokens / block_size keys, or NULL)
 * are the keys of its full blocks.  The leading run of keys found in the
 * cache shares the cached blocks; the other blocks are new, and new full
 * blocks are registered under their keys.  *n_cached_tokens (may be NULL)
 * receives the shared prompt tokens, a multiple of block_size, whose K/V are
 * already in the cache.  PKV_ERR_INVALID_ARG if seq_id exists. */
pkv_status pkv_bm_add_sequence(pkv_block_manager* bm, int64_t seq_id, int64_t n_prompt_tokens,
                               const uint64_t* block_hashes, int64_t* n_cached_tokens);

/* New sequence `child` with the same tokens as `parent`, sharing every
 * block of it (refcount + 1 each). */
pkv_status pkv_bm_fork(pkv_block_manager* bm, int64_t parent, int64_t child);

/* Reserve the slot of one new token for each of n distinct sequences, in
 * order.  slot_mapping (host, int64 [n]) receives block * block_size +
 * offset, ready for paged_kv_append.  cow_src / cow_dst (host, int32, room
 * for n each) receive the copy-on-write pairs, *n_cow their count; copy them
 * with paged_kv_copy_blocks before writing the new tokens.  Context lengths
 * grow by one.  PKV_ERR_NO_BLOCKS if the pool cannot supply the new and
 * copied blocks of the whole call. */
pkv_status pkv_bm_append(pkv_block_manager* bm, const int64_t* seq_ids, int32_t n, int64_t* slot_mapping,
                         int32_t* cow_src, int32_t* cow_dst, int32_t* n_cow);

/* Drop a sequence and release its blocks (last block first). */
pkv_status pkv_bm_free(pkv_block_manager* bm, int64_t seq_id);

/* Export the block tables and context lengths of n sequences, row i for
 * seq_ids[i]: block_tables (host, int32 [n][width], unused entries -1) and
 * context_lens (host, int32 [n]).  PKV_ERR_INVALID_ARG if a table is longer
 * than width or a sequence is unknown. */
pkv_status pkv_bm_get_tables(const pkv_block_manager* bm, const int64_t* seq_ids, int32_t n, int32_t width,
                             int32_t* block_tables, int32_t* context_lens);

/* Pool occupancy counters. */
pkv_status pkv_bm_stats(const pkv_block_manager* bm, pkv_bm_stats_t* out);

/* Refcount of one block. */
pkv_status pkv_bm_refcount(const pkv_block_manager* bm, int32_t block, int32_t* refcount);

/*
 * paged_attention_decode_mq -- several queries per sequence: the last q_len
 * tokens of every context are new (already written with paged_kv_append, for
 * instance a draft to verify: "LLM Primer VI" ch. 8, speculative decoding, or
 * a prefill chunk) and each attends to the context up to its own position:
 *   query i of sequence b sees tokens j < context_lens[b] - q_len + i + 1.
 * Otherwise as paged_attention_decode.
 *
 *   q, out   : device, [batch][q_len][n_q_heads][head_dim], f16 or bf16
 *   q_len    : 1 .. 16
 *   context_lens[b] : >= q_len (0 gives zero rows; 0 < n < q_len is clamped
 *              to 0 and sets PKV_DEVERR_CONTEXT)
 *   workspace: paged_attention_mq_workspace_size() bytes, or NULL
 * Each (sequence, group of kv-head-sharing query heads) runs as one set of
 * up to 16 (query, head) rows on the tensor cores.
 */
pkv_status paged_attention_mq_workspace_size(int32_t batch, int32_t q_len, int32_t n_q_heads, int32_t n_kv_heads,
                                             int32_t head_dim, pkv_dtype dtype, size_t* bytes);
pkv_status paged_attention_decode_mq(const void* q, const void* k_cache, const void* v_cache,
                                     const int32_t* block_tables, int32_t max_blocks_per_seq,
                                     const int32_t* context_lens, int32_t batch, int32_t q_len, int32_t num_blocks,
                                     float scale, int32_t n_q_heads, int32_t n_kv_heads, int32_t head_dim,
                                     int32_t block_size, void* out, pkv_dtype dtype, void* workspace,
                                     size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * INT8 paged KV cache (quantised KV, "Transformer anatomy" ch. 15 §15.7:
 * 8-bit K and V halve the cache bytes for a small loss of accuracy).
 *
 * Format (block_size 16, head dim d = 64 or 128): one byte array
 * kv_cache[num_blocks][n_kv_heads][R], R = 32 * d + 128 (4224 at d = 128),
 * holding one record per (block, kv head):
 *   bytes [0, 16 d)        K codes: row j (block offset j) of d bytes; its
 *                          16-byte chunk c is stored at chunk position
 *                          c ^ (j % min(8, d / 16));
 *   bytes [16 d, 32 d)     V codes, transposed: row e (dim e) of 16 bytes;
 *                          the token at block offset j is at byte
 *                          4 * ((j % 8) / 2) + 2 * (j / 8) + (j % 2);
 *   bytes [32 d, 32 d + 64)        16 fp32 K scales, by block offset;
 *   bytes [32 d + 64, 32 d + 128)  16 fp32 V scales.
 * A (token, kv head) row x of K or V is stored as codes
 *   c_e = rint(x_e / s), s = max_e |x_e| / 127 (binary32 division, round half
 *   to even; all codes 0 when the row is 0), and read as s * c_e.
 * The record is laid out so that a decode moves it with one contiguous copy
 * and reads it from shared memory without bank conflicts.
 * ------------------------------------------------------------------------ */

/*
 * paged_kv_append_int8 -- quantise and write the K/V of new tokens into
 * their slots of the INT8 cache (slot semantics as paged_kv_append; codes and
 * scales are bit-exact with the definition above).
 *
 *   k, v     : device, [num_tokens][n_kv_heads][head_dim], `dtype` (f32, f16, bf16)
 *   kv_cache : device, 16-byte aligned, layout above; written in place
 */
pkv_status paged_kv_append_int8(const void* k, const void* v, pkv_dtype dtype, const int64_t* slot_mapping,
                                int32_t num_tokens, uint8_t* kv_cache, int32_t num_blocks, int32_t block_size,
                                int32_t n_kv_heads, int32_t head_dim, void* stream);

/*
 * paged_attention_decode_int8 -- paged_attention_decode over the INT8 cache:
 * the same attention with K_j = s_j * (K codes) and V_j likewise.  q and out
 * are f16 or bf16 (`dtype`), head_dim 128.  Q K^T runs on the integer tensor
 * cores with every Q row put on a 14-bit grid (scale max|q| / 8191, two signed
 * 8-bit halves); P V runs in f16.  Workspace as paged_attention_decode (same
 * size function).  Tolerance against the fp64 oracle on the same codes: as
 * the 16-bit decode.
 */
pkv_status paged_attention_decode_int8(const void* q, const uint8_t* kv_cache, const int32_t* block_tables,
                                       int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t batch,
                                       int32_t num_blocks, float scale, int32_t n_q_heads, int32_t n_kv_heads,
                                       int32_t head_dim, int32_t block_size, void* out, pkv_dtype dtype,
                                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * pkv_get_device_error -- synchronise `stream`, then read and clear the
 * current device's error word.  *flags receives the PKV_DEVERR_* bits seen
 * since the last call.  Returns PKV_ERR_OUT_OF_RANGE if any bit was set,
 * PKV_ERR_CUDA if synchronisation failed, else PKV_OK.
 */
pkv_status pkv_get_device_error(void* stream, uint32_t* flags);

/* Static, NUL-terminated description of a status code. */
const char* pkv_status_string(pkv_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDKV_H_ */
