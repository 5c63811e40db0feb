// rq_internal.h -- layout of the cache arena and the launch interface shared
// by the host API (api.cpp) and the CUDA kernels.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/rq.h"

namespace rq {

constexpr int kHeadDim = 128;
constexpr int kTokTile = 64;        // padding granule of every token stream
constexpr int kMaxSplits = 256;     // split-KV partitions per (b, kv head)
constexpr int kMaxChunk = 1024;     // tokens per CTA (bounds the per-CTA shared-memory buffers)
constexpr int kMaxBatch = 256;      // sequences per cache (their lengths travel in the launch arguments)
constexpr int kMaxDevices = 64;     // devices a process may drive (per-device function attributes)
constexpr size_t kAlign = 256;

// Runs `set` (a cudaFuncSetAttribute call) once per device: function
// attributes are per-device state.  `done` is the caller's static flag array.
template <typename F>
cudaError_t once_per_device(bool (&done)[kMaxDevices], F set) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (done[dev]) return cudaSuccess;
    e = set();
    if (e == cudaSuccess) done[dev] = true;
    return e;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Byte sizes of one record (one token-head, K or V).
struct RecordSizes {
    int a_codes;   // anchor codes: d * anchor_bits / 8
    int r_codes;   // residual codes: d * resid_bits / 8
    int meta;      // (d / g) * 2: [scale e4m3, min e4m3] per group
};

// Token-to-row mapping of the record arrays of one (layer, group).  Each
// array is [blocks][H_kv][bt][record]: a block holds bt consecutive tokens of
// one sequence, for every kv head.  Contiguous caches have one block per
// sequence (block b, bt = the padded capacity Tp); paged caches draw blocks of
// bt = block_tokens tokens from a pool through a per-sequence block table.
struct Pages {
    const int *table;   // [B][mb] physical block of each block of tokens; null: contiguous
    int mb;             // table entries per sequence
    int bt;             // tokens per block
    int shift;          // log2(bt) (paged)
};

// Row (record index) of token t of (sequence b, kv head h).
__host__ __device__ inline size_t rec_row(const Pages &p, int H, int b, int h, int t) {
    if (!p.table) return ((size_t)b * H + h) * p.bt + (size_t)t;
    return (((size_t)p.table[(size_t)b * p.mb + (t >> p.shift)] * H + h) << p.shift) + (size_t)(t & (p.bt - 1));
}

// Where every array of the arena lives.  All token streams are laid out
// [blocks][H_kv][bt][record] (see Pages): the records of one (block, head)
// are one contiguous, 16-byte-aligned run.
struct Layout {
    rq_config cfg;
    RecordSizes rec;
    int groups;          // anchor groups per layer = num_loops / loops_per_group
    int Lg;              // loops per group
    int Tp;              // padded token capacity of a sequence (max_tokens rounded up to kTokTile)
    bool paged;          // records in a pool of blocks (block_tokens > 0)
    int BT;              // tokens per block (contiguous: Tp)
    int NBLK;            // blocks per array (contiguous: B)
    int MB;              // block-table entries per sequence (contiguous: 1)
    int tail_cap;        // max_tail_tokens
    int splits_max;      // partial slots per (b, q head)
    // residual format: per (layer, group)
    size_t anchor_codes_bytes;   // one kv side: B*H*Tp*a_codes
    size_t anchor_meta_bytes;    // one kv side: B*H*Tp*meta
    size_t anchor_block;         // both kv sides, aligned
    size_t resid_codes_bytes, resid_meta_bytes, resid_coef_bytes;
    size_t resid_block;          // one non-anchor loop, both kv sides
    size_t tail_bytes;           // one kv side of one loop: B*tail_cap*H*d*2
    size_t tail_block;           // one non-anchor loop, both kv sides
    size_t group_block;          // anchor + (Lg-1) residual + (Lg-1) tail blocks
    // BF16 format: per (layer, loop)
    size_t bf16_side;            // B*H*Tp*d*2
    size_t bf16_block;           // both kv sides
    // workspace
    size_t off_records;          // start of the record area (0)
    size_t records_bytes;
    size_t off_partials;         // float [B][Hq][splits_max][kPartialStride]
    size_t off_counters;         // int [B][H_kv]
    size_t off_err;              // int error word (+ pad)
    size_t off_vmax;             // int [layers][groups][Lg][B][H_kv]: largest V scale byte per stream
    size_t off_table;            // int [B][MB]: block table (paged)
    size_t total;
};

constexpr int kPartialStride = kHeadDim + 4;   // o[128], m, l, pad, pad

bool make_layout(const rq_config &cfg, Layout *out);

// --------------------------------------------------------------- kernels
// Per-sequence token counts (committed length, or the position a write starts at).
struct SeqLens {
    int v[kMaxBatch];
};

struct AppendArgs {
    // inputs: anchor-loop K/V (kv = 0 K, 1 V), [B][n][H][d] bf16
    const uint16_t *x_anchor[2];
    // tails of the non-anchor loops of the group: tail(kv, j) = tail0 +
    // j*tail_loop_stride + kv*tail_kv_stride (bytes); layout [B][cap][H][d]
    const uint8_t *tail0;
    size_t tail_loop_stride, tail_kv_stride;
    // anchor records: codes/meta of side kv at anchor0 + kv*anchor_kv_stride
    uint8_t *a_codes0, *a_meta0;
    size_t anchor_kv_stride;
    // residual records of loop j: r_*0 + j*resid_loop_stride + kv*resid_kv_stride
    uint8_t *r_codes0, *r_meta0, *r_coef0;
    size_t resid_loop_stride, resid_kv_stride;
    // largest FP8 scale byte of each V stream of the group, [Lg][B][H]
    // (record j < nres: residual of loop j; j = nres: the anchor), raised
    // with atomicMax as records are written
    int *vmax;
    SeqLens pos0;                              // first token position written, per sequence
    Pages pg;                                  // token -> record row
    int B, H, n, tail_cap, nres;               // nres = Lg - 1
    int g, ba, br, rotate;
    int scale_mode;                            // 0 least squares, 1 norm ratio, 2 none
    int chained;                               // 1: loop 0 is the anchor, loop l a residual against loop l - 1
    uint32_t sigma[4];
};

struct TailArgs {
    const uint16_t *src[2];   // [B][n][H][d]
    uint16_t *dst[2];         // [B][cap][H][d]
    int B, H, n, pos0, cap;
};

struct Bf16StoreArgs {
    const uint16_t *src[2];   // [B][n][H][d]
    uint16_t *dst[2];         // [B][H][Tp][d]
    SeqLens pos0;             // first token position written, per sequence
    int B, H, n, Tp;
};

constexpr int kMaxChain = 3;   // residual records one decode may chain (the chained reference, groups of 4)

struct DecodeArgs {
    // anchor streams (kv 0 = K, 1 = V)
    const uint8_t *a_codes[2], *a_meta[2];
    // residual streams of the records the loop's reconstruction reads, in
    // chain order (one for the shared reference; none for the anchor's own loop)
    const uint8_t *r_codes[kMaxChain][2], *r_meta[kMaxChain][2];
    const uint16_t *r_coef[kMaxChain][2];
    int nr;                   // residual records read
    // BF16 format streams
    const uint16_t *bf[2];
    const uint16_t *q;        // [B][Hq][d] bf16
    float *partials;          // [B][Hq][splits_max][kPartialStride]
    int *counters;            // [B * Hq] arrival counters of the fused split combine (zero between calls)
    int *err;                 // device error word (bounded waits that gave up)
    float *out;               // [B][Hq][d] fp32
    const uint16_t *tail_k, *tail_v;   // [B][tail_cap][H][d] BF16 in-flight tokens, or null
    // largest FP8 scale byte of the anchor V and (residual loops) the loop's
    // residual V stream of every (sequence, kv head), [B][H]: upper bounds of
    // the V scales, from which the weights' fixed point is chosen
    const int *vmax_a, *vmax_r[kMaxChain];
    // committed records below token `stable` are not written by any work
    // that may still run when this kernel starts (see the programmatic
    // launch in api.cpp); records from `stable` on are read only after the
    // kernel's grid-dependency wait
    int stable;
    int n_tail, tail_cap;
    // fused append: n_new tokens [B][n_new][H][d] written to tail rows
    // tail_pos.. (included in n_tail) by split 0 of each unit before the combine
    const uint16_t *new_k, *new_v;
    uint16_t *tail_k_w, *tail_v_w;
    int n_new, tail_pos;
    SeqLens seqT;             // committed tokens of each sequence (T = their maximum)
    Pages pg;                 // token -> record row (compressed format)
    int B, H, Hq, G, T, Tp, S, chunk, splits_max;   // Tp: row stride of the BF16 format
    int g;
    float scale_log2;         // softmax_scale * log2(e)
    int rotate;
    uint32_t sigma[4];
};

// Tokens [*t0, *t0 + *n) of split `split` of S: the ceil(T/64) tiles are
// dealt out evenly (tile counts differ by at most one; chunk >= the largest).
__host__ __device__ inline void split_range(int split, int S, int T, int *t0, int *n) {
    const int nt = (T + kTokTile - 1) / kTokTile;
    const int lo = (int)((long long)split * nt / S), hi = (int)((long long)(split + 1) * nt / S);
    *t0 = lo * kTokTile;
    *n = (hi * kTokTile < T ? hi * kTokTile : T) - *t0;
}

struct CombineArgs {
    const float *partials;
    const uint16_t *q;
    const uint16_t *tail_k, *tail_v;   // [B][cap][H][d] or null
    float *out;               // [B][Hq][d]
    int B, H, Hq, G, S, splits_max, n_tail, tail_cap;
    float scale_log2;
};

// Block-table writes and whole-block copies of a paged cache (copy-on-write
// of blocks shared by forked sequences), up to kMaxBlockOps of each per launch.
constexpr int kMaxBlockOps = 32;
constexpr int kMaxArrays = 4 + 6 * 15;   // record arrays of a loop group of up to 16 loops
struct BlockOpsArgs {
    int *table;
    uint8_t *records;          // start of the record area
    size_t group_block;        // bytes of one (layer, group) block
    int n_groups;              // layers x groups
    int n_arrays;
    size_t arr_off[kMaxArrays];   // record arrays inside a group block
    int arr_rec[kMaxArrays];      // their bytes per record
    size_t rows_per_block;        // H_kv x tokens per block
    int n_sets, n_copies;
    int set_idx[kMaxBlockOps], set_val[kMaxBlockOps];
    int copy_src[kMaxBlockOps], copy_dst[kMaxBlockOps];
};
cudaError_t launch_block_ops(const BlockOpsArgs &a, cudaStream_t st);

cudaError_t launch_append(const AppendArgs &a, cudaStream_t st);
cudaError_t launch_tail_copy(const TailArgs &a, cudaStream_t st);
cudaError_t launch_bf16_store(const Bf16StoreArgs &a, cudaStream_t st);
// a.nr residual records: 0, 1, or (INT4 anchor / INT2 residuals only) 2-3
bool decode_rq_supported(int ba, int br, int nr);
cudaError_t launch_decode_rq(const DecodeArgs &a, int ba, int br, cudaStream_t st);
cudaError_t launch_decode_bf16(const DecodeArgs &a, cudaStream_t st);
cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st);
// resident CTAs per SM of the decode kernels for a given chunk (tokens per CTA)
int decode_rq_occupancy(int G, int ba, int br, int nr, int g, int chunk);
int decode_bf16_occupancy(int G, int chunk);

// rq_decode_attn with the split partials and the combine counters in
// caller-supplied device scratch instead of the cache's workspace: `partials`
// holds partial_floats floats, `counters` max_units ints that are zero
// between calls.
int decode_with_scratch(rq_cache *c, int layer, int loop, const void *q, float *out, float scale, void *stream,
                        float *partials, size_t partial_floats, int *counters, size_t max_units);

// The device the cache's arena lives on.
int cache_device(const rq_cache *c);

// Zeroes the allocation-free entry point's combine counters on the current
// device if that device's scratch address has been resolved (after a
// bounded wait gave up; see rq_check).  Enqueued on the legacy stream.
void noalloc_reset_counters();

}  // namespace rq
