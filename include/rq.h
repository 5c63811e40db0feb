/*
 * rq.h -- C ABI of the B200 (sm_100a) ResidualQuant decode-attention library.
 *
 * Method: "ResidualQuant: KV Cache Quantization for Looped Transformers with
 * 2-Bit Residuals" (arXiv 2610.10381; abstract, and the ai4snews summary,
 * paragraphs 1-4).  A looped Transformer produces its own K/V per (layer,
 * loop); the cache keeps the final loop of each loop group as an INT4
 * "anchor" and every other loop as a BF16 least-squares coefficient plus an
 * INT2 residual of the rotated difference, so that
 *     K_l ~= s_l * a_hat + R^T r_hat          (two cache reads per loop)
 * Decode attention returns softmax(q K^T * scale) V over that cache.
 *
 * Conventions shared by every call:
 *   - All device pointers are CUDA global-memory pointers of the current
 *     device, which must be the device the cache was created on (else
 *     RQ_ERR_INVALID).  "stream" is a cudaStream_t passed as void* (NULL =
 *     the legacy default stream).  Work is enqueued asynchronously; no call
 *     synchronises the host except rq_cache_create/destroy and
 *     rq_cache_export (which copies to host memory).
 *   - BF16 arrays hold IEEE bfloat16 bit patterns (uint16).
 *   - Calls return an rq_status (0 = RQ_OK, negative = error) and never
 *     throw; a failing call leaves the cache state unchanged.
 *   - Calls that touch one cache must not run concurrently with each other
 *     (the cache owns one split-combine workspace); enqueue them on one
 *     stream, or order the streams.
 *   - Ownership: the caller owns q, k, v, out and (optionally) the cache's
 *     device arena; the library owns the host-side handle and, when it
 *     allocated the arena itself, the arena.  Once created, the arena is
 *     written only by this library's calls (the decode kernel relies on it:
 *     see rq_decode_attn).
 */
#ifndef RQ_H
#define RQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RQ_OK = 0,
    RQ_ERR_INVALID = -1,      /* bad argument (null pointer, index out of range, ...) */
    RQ_ERR_UNSUPPORTED = -2,  /* configuration outside what the kernels implement */
    RQ_ERR_NOMEM = -3,        /* caller arena too small, or device allocation failed */
    RQ_ERR_CAPACITY = -4,     /* append would exceed max_tokens / max_tail_tokens */
    RQ_ERR_STATE = -5,        /* call out of order (e.g. anchor append before its loops) */
    RQ_ERR_CUDA = -6,         /* a CUDA runtime call failed (sticky errors included) */
    RQ_ERR_TIMEOUT = -7       /* a device-side bounded wait gave up (see rq_check) */
} rq_status;

typedef enum {
    RQ_FMT_RESIDUAL = 0,      /* INT anchor + INT residuals (the compressed cache) */
    RQ_FMT_BF16 = 1           /* every loop stored uncompressed in BF16 (comparison) */
} rq_format;

/*
 * Cache shape and format.
 *   num_layers       layers sharing the cache object
 *   num_loops        recurrent loops per layer (Ouro-1.4B: 4; Huginn: 32)
 *   loops_per_group  loops per anchor group; the anchor is the LAST loop of
 *                    each group (Ouro 4/4; Huginn-style 32 loops in 8 groups
 *                    of 4, per the ai4snews summary, paragraph 1).
 *                    num_loops % loops_per_group == 0.
 *   batch            sequences B (at most 256); appends add the same number
 *                    of tokens to every sequence, while committed lengths may
 *                    differ per sequence (rq_cache_truncate_seq)
 *   max_tokens       committed-token capacity per (layer, group), at most
 *                    262144 (256 split partials of up to 1024 tokens)
 *   max_tail_tokens  in-flight tokens a non-anchor loop may hold before the
 *                    group's anchor commits them
 *   num_kv_heads     H_kv
 *   num_q_heads      H_q; H_q % H_kv == 0 and H_q/H_kv in {1,2,4,8};
 *                    query head h reads kv head h / (H_q/H_kv)
 *   head_dim         d; must be 128
 *   group_size       g in {16, 32}: quantization groups along head_dim, each
 *                    with an FP8-E4M3 scale and an FP8-E4M3 minimum
 *   anchor_bits      {4, 2};  resid_bits {2, 4}
 *   rotate           1: residuals rotated by R = H_d diag(sigma)/sqrt(d)
 *                    (Sylvester Hadamard; sigma_j = -1 iff the top bit of
 *                    splitmix64(seed + j) is set); 0: R = I
 *   format           rq_format
 *   seed             rotation seed (shared by K and V and all loops)
 *   scale_mode       coefficient of a residual loop (the abstract's scaling
 *                    ablation): 0 least squares <x, ref>/<ref, ref> (the
 *                    method), 1 norm ratio |x|/|ref|, 2 none (s = 1); 0 when
 *                    ref = 0 (modes 0, 1).  Stored in BF16 either way.
 *   anchor_mode      reference of a residual loop (the abstract's reference
 *                    ablation): 0 the group's last loop, shared by all other
 *                    loops (the method: two cache reads per loop); 1 chained:
 *                    the group's FIRST loop is quantized at anchor_bits and
 *                    loop l >= 1 is a residual against the reconstruction of
 *                    loop l - 1, so rebuilding loop l reads l + 1 records.
 *                    The group is still committed when its last loop is
 *                    appended.
 *   rotation_per_layer  0: one rotation per cache; 1: layer i uses the seed
 *                    seed + i * 2^32 (rotations fixed per layer)
 *   block_tokens     0: each sequence's records are contiguous (capacity
 *                    max_tokens); 128 or 256: paged -- records live in
 *                    blocks of this many tokens drawn from a pool of
 *                    num_blocks physical blocks per (layer, group), through a
 *                    per-sequence block table shared by all layers and groups
 *                    (the library allocates blocks as sequences grow and
 *                    returns them when sequences shrink; see
 *                    rq_cache_fork_seq).  RQ_FMT_RESIDUAL only.
 *   num_blocks       paged: physical blocks per pool (each holds block_tokens
 *                    tokens of every kv head); 0 otherwise
 * Fields after `seed` are zero for the method with contiguous records.
 */
typedef struct rq_config {
    int32_t num_layers;
    int32_t num_loops;
    int32_t loops_per_group;
    int32_t batch;
    int32_t max_tokens;
    int32_t max_tail_tokens;
    int32_t num_kv_heads;
    int32_t num_q_heads;
    int32_t head_dim;
    int32_t group_size;
    int32_t anchor_bits;
    int32_t resid_bits;
    int32_t rotate;
    int32_t format;
    uint64_t seed;
    int32_t scale_mode;
    int32_t anchor_mode;
    int32_t rotation_per_layer;
    int32_t block_tokens;
    int32_t num_blocks;
} rq_config;

typedef struct rq_cache rq_cache;

/* Human-readable name of a status code (static string). */
const char *rq_status_string(int status);

/* Validates cfg.  RQ_OK, RQ_ERR_INVALID or RQ_ERR_UNSUPPORTED. */
int rq_config_check(const rq_config *cfg);

/* Device bytes rq_cache_create needs for cfg (records, BF16 tails, split
 * workspace, alignment padding); 0 if cfg is invalid. */
size_t rq_cache_required_bytes(const rq_config *cfg);

/* Committed storage per token: bytes of all records one token occupies over
 * all layers, loops, heads, K and V (codes + FP8 scale/min + BF16
 * coefficients; BF16 format: 2 bytes per element).  This is the figure behind
 * the pages' effective-bitwidth accounting (ai4snews summary, paragraph 2):
 * for 4 loops, INT4 anchor, INT2 residuals, g = 32 it is 19.34% of BF16
 * (the 80.7% reduction).  0 if cfg is invalid. */
size_t rq_cache_token_bytes(const rq_config *cfg);

/* Creates a cache.  dev_mem: caller-owned device arena of at least
 * rq_cache_required_bytes(cfg) bytes, 256-byte aligned, or NULL to let the
 * library cudaMalloc it.  The arena is zeroed (synchronously).  On success
 * *out receives the handle.  Errors: INVALID, UNSUPPORTED, NOMEM, CUDA. */
int rq_cache_create(const rq_config *cfg, void *dev_mem, size_t bytes, rq_cache **out);

/* Frees the handle and, if the library allocated it, the arena
 * (synchronises the device first).  NULL is accepted. */
int rq_cache_destroy(rq_cache *cache);

/*
 * Append n_tokens tokens of one (layer, loop) for every sequence.
 *   k_bf16, v_bf16: device, [batch][n_tokens][num_kv_heads][head_dim] BF16.
 * RQ_FMT_RESIDUAL:
 *   - a non-anchor loop copies its K/V into that loop's BF16 tail (the
 *     in-flight tokens, read by decode as they are);
 *   - the anchor loop (last loop of its group) requires every other loop of
 *     the group to hold exactly n_tokens tail tokens (else RQ_ERR_STATE);
 *     it quantizes the anchor to INT<anchor_bits> (groups of g, FP8 scale
 *     and min), and for each other loop computes the least-squares
 *     coefficient s = <x_l, a_hat>/<a_hat, a_hat> (BF16), the residual
 *     x_l - s_hat a_hat, rotates it by R and quantizes it to
 *     INT<resid_bits> the same way (ai4snews summary, paragraph 1); then it
 *     commits the tokens and empties the group's tails.  The encoding
 *     decisions are taken in fp64.
 * RQ_FMT_BF16: the tokens are stored in that loop's BF16 cache directly.
 * Errors: INVALID, CAPACITY, STATE, CUDA.  The input buffers may be reused
 * once the enqueued work has run.
 */
int rq_append(rq_cache *cache, int layer, int loop, const void *k_bf16, const void *v_bf16,
              int n_tokens, void *stream);

/*
 * Single-token decode attention for one (layer, loop) over the compressed
 * cache (format RQ_FMT_RESIDUAL).
 *   q_bf16: device, [batch][num_q_heads][head_dim] BF16.
 *   out:    device, [batch][num_q_heads][head_dim] fp32.
 *   softmax_scale: logits are scale * <q, k>; <= 0 selects 1/sqrt(head_dim).
 * Keys/values seen: the committed tokens of the loop's group (anchor loop:
 * the dequantized anchor; other loops: s_hat a_hat + R^T r_hat), followed by
 * the loop's BF16 tail tokens.  With no key at all the output is zero.
 * Overlap: the kernel is launched so that it may start while the previous
 * work on `stream` is still running (programmatic dependent launch).  Before
 * that work has completed it reads only committed records that no append
 * enqueued earlier can still be writing; q, the tail, out and everything else
 * are touched only after it.  The observable results are those of plain
 * stream order.
 * Errors: INVALID, STATE (wrong format), CUDA.
 */
int rq_decode_attn(rq_cache *cache, int layer, int loop, const void *q_bf16, float *out,
                   float softmax_scale, void *stream);

/*
 * rq_append(cache, layer, loop, k, v, n_tokens) followed by
 * rq_decode_attn(cache, layer, loop, q, out, softmax_scale) on the same
 * stream, with the same results, state changes and errors.  For a non-anchor
 * loop of an RQ_FMT_RESIDUAL cache holding committed tokens, it is one kernel
 * launch: the decode kernel writes the new tokens into the loop's BF16 tail
 * itself before merging the tail (the per-step order of the ai4snews
 * summary's decode: the new token's earlier loops are kept uncompressed and
 * attended to).  Otherwise it enqueues the two calls.  The paper has no
 * counterpart to the fusion; it saves a launch per non-anchor loop.
 *   k_bf16, v_bf16: as for rq_append; q_bf16, out: as for rq_decode_attn.
 * Errors: INVALID, CAPACITY, STATE, CUDA; on error nothing is appended.
 */
int rq_append_decode_attn(rq_cache *cache, int layer, int loop, const void *k_bf16, const void *v_bf16,
                          int n_tokens, const void *q_bf16, float *out, float softmax_scale, void *stream);

/* The same attention over an RQ_FMT_BF16 cache: the uncompressed comparison
 * kernel (the role BF16 FlashAttention plays in the ai4snews summary,
 * paragraph 4).  Errors: INVALID, STATE (wrong format), CUDA. */
int rq_decode_attn_bf16(rq_cache *cache, int layer, int loop, const void *q_bf16, float *out,
                        float softmax_scale, void *stream);

/*
 * Multi-token causal attention for one (layer, loop) over the compressed
 * cache (format RQ_FMT_RESIDUAL): the attention of a chunked prefill, or of
 * several drafted tokens, after their K/V were appended (rq_append with
 * n_tokens = n on every loop so far).  The ai4snews summary's decode study
 * (paragraph 4) times decode only; this call is the step before it, reading
 * the same records the decode reads.
 *   q_bf16: device, [batch][n_tokens][num_q_heads][head_dim] BF16: the n most
 *           recent tokens of every sequence, oldest first.
 *   out:    device, [batch][n_tokens][num_q_heads][head_dim] fp32.
 *   softmax_scale: as for rq_decode_attn.
 * Keys/values: the sequence of the loop's group's committed tokens (as
 * rq_decode_attn reconstructs them) followed by the loop's BF16 tail tokens;
 * query token i (0-based) of sequence b sees its first
 * len_b + n_tail - n_tokens + 1 + i tokens (len_b: b's committed tokens), so
 * the n new tokens are the last ones -- committed at an anchor loop, in the
 * tail at the other loops -- and each sees itself and the ones before it.
 * The split partials live in a device buffer the cache allocates on the
 * first call (and grows when a later call needs more:
 * batch * n_tokens * num_q_heads * splits * 132 floats), and the arrival
 * counters of the splits (batch * num_kv_heads *
 * ceil(n_tokens * num_q_heads / num_kv_heads / 64)
 * ints, zeroed when allocated and left at zero by every call) in a second
 * one; both are freed by rq_cache_destroy.  Those allocations synchronise the
 * device, so make the first call of a size before any stream capture.  Calls
 * on one cache share the buffers: calls whose work overlaps (other streams)
 * must be ordered by the caller.
 * Errors: INVALID (null pointer, n_tokens < 1, index out of range), STATE
 * (wrong format, or a sequence holds fewer than n_tokens tokens),
 * UNSUPPORTED (n_tokens > 65535, an INT2 anchor with INT4 residuals -- the
 * multi-token kernel is built for INT4/INT2, INT2/INT2 and INT4/INT4 -- or
 * the chained, previous-loop reference),
 * NOMEM, CUDA.  UNSUPPORTED is returned before any allocation.
 */
int rq_prefill_attn(rq_cache *cache, int layer, int loop, const void *q_bf16, int n_tokens, float *out,
                    float softmax_scale, void *stream);

/*
 * rq_decode_attn without any allocation: identical arguments, results and
 * errors, except that the split-combine partials go to a fixed array the
 * library holds in device memory (8 MiB per GPU that loads the library, kept
 * until process exit) instead of the cache's workspace.  The paper has no
 * counterpart to this call; it is a deployment convenience.
 *   For callers that must not allocate device memory after start-up: a plugin
 *   inside a host framework that owns all device memory and offers no
 *   allocator, a serving loop whose memory is planned once, or work issued
 *   during stream capture, where allocation calls are refused.
 *   Limits: batch * num_q_heads * S * 132 floats must fit in 2^21 - 2^16
 *   floats (the last 2^16 words of the array hold the combine counters), S
 *   being the split count the call chooses (at most ceil(T/64)), and
 *   batch * num_q_heads must not exceed 65536; beyond either the call returns
 *   RQ_ERR_CAPACITY and enqueues nothing.
 *   The first call on a device looks up the array's device address (and
 *   zeroes its counters, synchronously); make it before any stream capture.
 *   The current device must be the cache's (else RQ_ERR_INVALID).  All calls
 *   on a device share the array: calls whose GPU work overlaps race on it and
 *   must be ordered by the caller.
 *   Format must be RQ_FMT_RESIDUAL (else RQ_ERR_STATE).
 */
int rq_decode_attn_noalloc(rq_cache *cache, int layer, int loop, const void *q_bf16, float *out,
                           float softmax_scale, void *stream);

/* Committed length of (layer, group): the longest sequence's.  group =
 * loop / loops_per_group for the residual format; for the BF16 format pass
 * the loop index. */
int rq_cache_length(const rq_cache *cache, int layer, int group, int *len);

/* Committed length of sequence `seq` of (layer, group). */
int rq_cache_length_seq(const rq_cache *cache, int layer, int group, int seq, int *len);

/* In-flight (tail) tokens of (layer, loop); 0 for anchor loops and for the
 * BF16 format. */
int rq_cache_tail_length(const rq_cache *cache, int layer, int loop, int *n);

/* Roll the committed length of (layer, group) back to new_len (<= current),
 * e.g. to discard rejected tokens: every sequence keeps min(its length,
 * new_len).  The group's tails must be empty (else RQ_ERR_STATE).
 * Host-side only: no device work. */
int rq_cache_truncate(rq_cache *cache, int layer, int group, int new_len);

/* The same for one sequence: its committed length becomes new_len (<= its
 * current length).  Sequences of one cache may so hold different numbers of
 * committed tokens (a ragged batch); decode attends, for each sequence, to
 * its own committed tokens (plus the loop's tail tokens), and later appends
 * write each sequence's tokens after its own last one.  Errors: INVALID,
 * STATE (non-empty tails).  Host-side only. */
int rq_cache_truncate_seq(rq_cache *cache, int layer, int group, int seq, int new_len);

/*
 * Copy the committed records of (layer, loop) to host memory in the logical
 * record format (for tests and inspection; synchronises `stream`):
 * (len = rq_cache_length; rows past a shorter sequence's length hold no token of it)
 * The loop's own record is the anchor record for the group's last loop
 * (anchor_mode 0) or its first loop (anchor_mode 1), a residual record for
 * the others; the host buffers must be sized for that kind:
 *   anchor record: host_codes [2][B][H_kv][len][d*anchor_bits/8]  (K then V)
 *                  host_meta  [2][B][H_kv][len][2*d/g]  ([scale, min] per group)
 *                  host_coef  unused (may be NULL)
 *   residual:      host_codes [2][B][H_kv][len][d*resid_bits/8]
 *                  host_meta  [2][B][H_kv][len][2*d/g]
 *                  host_coef  [2][B][H_kv][len] BF16
 * Code packing: element i at byte i*b/8, bit (i*b)%8, LSB first.
 * Errors: INVALID, STATE (BF16 format), CUDA.
 */
int rq_cache_export(const rq_cache *cache, int layer, int loop, void *host_codes, void *host_meta,
                    void *host_coef, void *stream);

/* Algorithmic bytes one decode call of (layer, loop) moves at the current
 * lengths: codes + FP8 meta + BF16 coefficients of the records read (anchor
 * and, for non-anchor loops, the loop's residual), BF16 tail tokens, BF16 q
 * and fp32 out.  Split-combine traffic is not counted.  0 on bad input. */
size_t rq_decode_bytes(const rq_cache *cache, int layer, int loop);

/*
 * Paged caches (block_tokens > 0): records live in blocks of block_tokens
 * tokens (every kv head of one sequence) drawn from a pool of num_blocks per
 * (layer, group), addressed through a per-sequence block table shared by all
 * layers and groups -- the layout of a serving engine's paged KV cache (the
 * ai4snews summary, paragraph 4, integrates the method with vLLM).  The
 * library owns the pool: rq_append takes blocks from the free list as a
 * sequence grows past its last block (RQ_ERR_CAPACITY when none is left;
 * nothing is appended then), and rq_cache_truncate / rq_cache_truncate_seq
 * return the blocks no (layer, group) of the sequence needs any more.
 * Blocks carry reference counts: a forked sequence shares its source's
 * blocks until either sequence writes into a shared one, which is then
 * copied first (copy-on-write, enqueued on the appending call's stream).
 * Decode, rq_prefill_attn, export and the other calls work on paged caches
 * as on contiguous ones.
 */

/* Makes sequence dst (every committed length 0, no tail tokens in the cache)
 * a copy of sequence src that shares src's blocks: its committed lengths
 * become src's, and later appends to either copy the shared block they
 * write into.  Enqueues a few small copies on `stream`.  Errors: INVALID,
 * UNSUPPORTED (contiguous cache), STATE (dst not empty, or tails not empty),
 * CUDA. */
int rq_cache_fork_seq(rq_cache *cache, int src, int dst, void *stream);

/* Permutes the free list with a seeded Fisher-Yates shuffle (splitmix64
 * draws), so that later allocations scatter over the pool (tests and
 * fragmentation studies).  Host only.  Errors: INVALID, UNSUPPORTED. */
int rq_cache_shuffle_free_blocks(rq_cache *cache, uint64_t seed);

/* Number of free blocks in the pool.  Errors: INVALID, UNSUPPORTED. */
int rq_cache_free_blocks(const rq_cache *cache, int *n);

/* The physical blocks of sequence seq, in token order: *n receives their
 * count, host_blocks (may be NULL) the first min(*n, max_blocks) ids.
 * Errors: INVALID, UNSUPPORTED. */
int rq_cache_seq_blocks(const rq_cache *cache, int seq, int32_t *host_blocks, int max_blocks, int *n);

/* Reports asynchronous failures: RQ_ERR_TIMEOUT if a kernel's bounded wait
 * gave up (the error word and the split-combine counters -- the cache's,
 * rq_prefill_attn's and rq_decode_attn_noalloc's on this device -- are then
 * cleared, so later calls start clean), RQ_ERR_CUDA if the context holds a
 * sticky error, RQ_ERR_STATE if rq_prefill_attn's split-arrival counters are
 * not all zero after its calls completed (they are cleared), else RQ_OK.
 * Synchronises the device. */
int rq_check(rq_cache *cache);

#ifdef __cplusplus
}
#endif

#endif /* RQ_H */
