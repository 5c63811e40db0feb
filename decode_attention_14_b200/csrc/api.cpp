// api.cpp -- the C ABI declared in include/rq.h: argument validation, the
// cache's host-side state (committed lengths, tail counts), arena layout and
// kernel launches.  Every arithmetic step of the method runs in the CUDA
// kernels; this file only moves pointers and sizes around.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>

#include "prefill.h"
#include "rq_internal.h"

using namespace rq;

struct rq_cache {
    Layout lay;
    uint8_t *base = nullptr;
    bool owned = false;
    int device = 0;
    int sms = 148;
    std::vector<int> len;     // residual: [layer][group]; bf16: [layer][loop]; the longest sequence
    std::vector<int> seq;     // the same, per sequence: [layer][group or loop][batch]
    std::vector<int> ntail;   // [layer][loop]
    // per length slot: the first token position the most recent record write
    // (an anchor append) started at, over the sequences; records below it are
    // not touched by any append still in flight
    std::vector<int> wstart;
    // a block-table change is (or may be) in flight: the next decode reads the
    // table only after its grid-dependency wait
    bool table_dirty = false;
    std::vector<uint32_t> sigma;   // [layer][4]: sign bits of the layer's rotation
    // resident CTAs per SM for chunk = 64 * (i + 1), by residual records read (0 .. kMaxChain)
    int occ[kMaxChain + 1][kMaxChunk / kTokTile];
    // split partials of rq_prefill_attn, allocated on first use and grown on demand
    float *prefill_ws = nullptr;
    size_t prefill_ws_floats = 0;
    // arrival counters of rq_prefill_attn's row blocks (zeroed once; every
    // launch leaves them at zero)
    int *prefill_cnt = nullptr;
    size_t prefill_cnt_n = 0;
    // paged records: host copy of the block table [B][MB] (-1: no block),
    // reference counts of the physical blocks (forked sequences share
    // blocks), and the free list (blocks are taken from its back)
    std::vector<int> table;
    std::vector<int> ref;
    std::vector<int> free_blocks;
};

namespace {

// splitmix64 (Steele, Lea & Flood, OOPSLA 2014): golden-gamma increment and
// the 30/27/31 xor-shift-multiply finaliser.
uint64_t splitmix64(uint64_t x) {
    uint64_t z = x + 0x9E3779B97F4A7C15ULL;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

// The last loop of its group: its append commits the group's tokens (the
// other loops keep theirs in BF16 tails until then).
bool is_commit_loop(const Layout &L, int loop) { return (loop % L.Lg) == L.Lg - 1; }

// The record a loop's own K/V is stored in: -1 the anchor record, else the
// index of its residual record.  Last-loop reference: the commit loop is the
// anchor and loop j < Lg - 1 is residual j.  Chained reference: loop 0 is
// the anchor and loop j >= 1 is residual j - 1 (its reconstruction reads
// the anchor and residuals 0 .. j - 1).
int record_slot(const Layout &L, int loop) {
    const int j = loop % L.Lg;
    if (L.cfg.anchor_mode == 1) return j == 0 ? -1 : j - 1;
    return j == L.Lg - 1 ? -1 : j;
}

uint8_t *group_base(const rq_cache *c, int layer, int group) {
    const Layout &L = c->lay;
    return c->base + L.off_records + ((size_t)layer * L.groups + group) * L.group_block;
}

uint8_t *anchor_codes(const rq_cache *c, int layer, int group, int kv) {
    const Layout &L = c->lay;
    return group_base(c, layer, group) + kv * (L.anchor_codes_bytes + L.anchor_meta_bytes);
}
uint8_t *anchor_meta(const rq_cache *c, int layer, int group, int kv) {
    return anchor_codes(c, layer, group, kv) + c->lay.anchor_codes_bytes;
}
size_t resid_side(const Layout &L) { return L.resid_codes_bytes + L.resid_meta_bytes + L.resid_coef_bytes; }
uint8_t *resid_codes(const rq_cache *c, int layer, int group, int j, int kv) {
    const Layout &L = c->lay;
    return group_base(c, layer, group) + L.anchor_block + (size_t)j * L.resid_block + kv * resid_side(L);
}
uint8_t *resid_meta(const rq_cache *c, int layer, int group, int j, int kv) {
    return resid_codes(c, layer, group, j, kv) + c->lay.resid_codes_bytes;
}
uint8_t *resid_coef(const rq_cache *c, int layer, int group, int j, int kv) {
    return resid_meta(c, layer, group, j, kv) + c->lay.resid_meta_bytes;
}
uint8_t *tail_ptr(const rq_cache *c, int layer, int group, int j, int kv) {
    const Layout &L = c->lay;
    return group_base(c, layer, group) + L.anchor_block + (size_t)(L.Lg - 1) * L.resid_block +
           (size_t)j * L.tail_block + kv * L.tail_bytes;
}
uint16_t *bf16_ptr(const rq_cache *c, int layer, int loop, int kv) {
    const Layout &L = c->lay;
    return (uint16_t *)(c->base + L.off_records + ((size_t)layer * L.cfg.num_loops + loop) * L.bf16_block +
                        kv * L.bf16_side);
}

// largest V scale byte of record r (r < Lg - 1: residual of loop r; r = Lg - 1:
// the anchor) of every (sequence, kv head) of (layer, group): int [B][H]
int *vmax_ptr(const rq_cache *c, int layer, int group, int r) {
    const Layout &L = c->lay;
    const size_t bh = (size_t)L.cfg.batch * L.cfg.num_kv_heads;
    return (int *)(c->base + L.off_vmax) + (((size_t)layer * L.groups + group) * L.Lg + r) * bh;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? RQ_OK : RQ_ERR_CUDA; }

// Token -> record row mapping of the compressed format.
Pages pages_of(const rq_cache *c) {
    const Layout &L = c->lay;
    Pages p;
    p.table = L.paged ? (const int *)(c->base + L.off_table) : nullptr;
    p.mb = L.MB;
    p.bt = L.BT;
    p.shift = 0;
    while (L.paged && (1 << p.shift) < L.BT) p.shift++;
    return p;
}

// The record arrays inside one (layer, group) block of the arena, as
// (offset, bytes per record) pairs (the BF16 tails excluded).
int record_arrays(const Layout &L, size_t *off, int *rec) {
    int n = 0;
    for (int kv = 0; kv < 2; kv++) {
        const size_t a0 = kv * (L.anchor_codes_bytes + L.anchor_meta_bytes);
        off[n] = a0;
        rec[n++] = L.rec.a_codes;
        off[n] = a0 + L.anchor_codes_bytes;
        rec[n++] = L.rec.meta;
    }
    const size_t side = L.resid_codes_bytes + L.resid_meta_bytes + L.resid_coef_bytes;
    for (int j = 0; j < L.Lg - 1; j++)
        for (int kv = 0; kv < 2; kv++) {
            const size_t r0 = L.anchor_block + (size_t)j * L.resid_block + kv * side;
            off[n] = r0;
            rec[n++] = L.rec.r_codes;
            off[n] = r0 + L.resid_codes_bytes;
            rec[n++] = L.rec.meta;
            off[n] = r0 + L.resid_codes_bytes + L.resid_meta_bytes;
            rec[n++] = 2;
        }
    return n;
}

// Device work of block operations collected on the host: block-table
// entries to set and whole blocks to copy (copy-on-write of shared blocks).
struct PendingOps {
    std::vector<std::pair<int, int>> sets;     // (table index, block)
    std::vector<std::pair<int, int>> copies;   // (source block, destination block)
};

int flush_ops(rq_cache *c, const PendingOps &ops, cudaStream_t st) {
    const Layout &L = c->lay;
    BlockOpsArgs a;
    std::memset(&a, 0, sizeof(a));
    a.table = (int *)(c->base + L.off_table);
    a.records = c->base + L.off_records;
    a.group_block = L.group_block;
    a.n_groups = L.cfg.num_layers * L.groups;
    a.n_arrays = record_arrays(L, a.arr_off, a.arr_rec);
    a.rows_per_block = (size_t)L.cfg.num_kv_heads * L.BT;
    size_t i = 0, k = 0;
    while (i < ops.sets.size() || k < ops.copies.size()) {
        a.n_sets = a.n_copies = 0;
        for (; i < ops.sets.size() && a.n_sets < kMaxBlockOps; i++) {
            a.set_idx[a.n_sets] = ops.sets[i].first;
            a.set_val[a.n_sets++] = ops.sets[i].second;
        }
        for (; k < ops.copies.size() && a.n_copies < kMaxBlockOps; k++) {
            a.copy_src[a.n_copies] = ops.copies[k].first;
            a.copy_dst[a.n_copies++] = ops.copies[k].second;
        }
        c->table_dirty = true;
        if (launch_block_ops(a, st) != cudaSuccess) return RQ_ERR_CUDA;
    }
    return RQ_OK;
}

// Blocks a sequence needs: those holding any committed token of any
// (layer, group).
int blocks_needed(const rq_cache *c, int b) {
    const Layout &L = c->lay;
    int mx = 0;
    for (size_t slot = 0; slot < c->len.size(); slot++) mx = std::max(mx, c->seq[slot * L.cfg.batch + b]);
    return (mx + L.BT - 1) / L.BT;
}

// Returns blocks k >= keep of sequence b to the pool (host only: the device
// table keeps stale entries, never read past a sequence's length).
void release_blocks(rq_cache *c, int b, int keep) {
    const Layout &L = c->lay;
    for (int k = keep; k < L.MB; k++) {
        int &e = c->table[(size_t)b * L.MB + k];
        if (e < 0) continue;
        if (--c->ref[e] == 0) c->free_blocks.push_back(e);
        e = -1;
    }
}

// Before tokens [pos0_b, pos0_b + n) of every sequence are written: every
// block they fall in is allocated, and a block shared with another sequence
// is first copied (copy-on-write).  Enqueues the table and copy work on st.
// All or nothing: on CAPACITY (pool exhausted) the host state is restored.
int prepare_blocks(rq_cache *c, const SeqLens &pos0, int n, cudaStream_t st) {
    const Layout &L = c->lay;
    const std::vector<int> table0 = c->table, ref0 = c->ref, free0 = c->free_blocks;
    PendingOps ops;
    for (int b = 0; b < L.cfg.batch; b++) {
        const int k0 = pos0.v[b] / L.BT, k1 = (pos0.v[b] + n - 1) / L.BT;
        for (int k = k0; k <= k1; k++) {
            int &e = c->table[(size_t)b * L.MB + k];
            if (e >= 0 && c->ref[e] == 1) continue;
            if (c->free_blocks.empty()) {
                c->table = table0;
                c->ref = ref0;
                c->free_blocks = free0;
                return RQ_ERR_CAPACITY;
            }
            const int nb = c->free_blocks.back();
            c->free_blocks.pop_back();
            c->ref[nb] = 1;
            if (e >= 0) {   // shared: copy, then drop this sequence's reference
                ops.copies.push_back({e, nb});
                c->ref[e]--;
            }
            e = nb;
            ops.sets.push_back({b * L.MB + k, nb});
        }
    }
    const int s = flush_ops(c, ops, st);
    if (s != RQ_OK) {
        c->table = table0;
        c->ref = ref0;
        c->free_blocks = free0;
    }
    return s;
}

// per-sequence lengths of length slot `slot` (= layer * groups + group, or
// layer * loops + loop for the BF16 format)
int *seq_lens(rq_cache *c, size_t slot) { return c->seq.data() + slot * c->lay.cfg.batch; }
const int *seq_lens(const rq_cache *c, size_t slot) { return c->seq.data() + slot * c->lay.cfg.batch; }
void fill_lens(const int *v, int B, SeqLens *out) {
    for (int b = 0; b < B; b++) out->v[b] = v[b];
}
void grow(rq_cache *c, size_t slot, int n) {
    int *v = seq_lens(c, slot);
    for (int b = 0; b < c->lay.cfg.batch; b++) v[b] += n;
    c->len[slot] += n;
}

float resolve_scale(float s) { return s > 0.f ? s : 1.0f / std::sqrt((float)kHeadDim); }

// Kernels run on the current device and address the cache's arena, so the
// two must be the same device.
bool on_cache_device(const rq_cache *c) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return dev == c->device;
}

// Split-KV partition of T tokens over `units` independent (sequence, kv head
// [, q-head pair]) problems.  The ceil(T/64) tiles are dealt out evenly over
// S splits (split_range); chunk is the largest split, at most kMaxChunk.
// Among the admissible split counts the one with the least wave-quantised
// work (waves x tokens of the largest CTA, plus a fixed per-CTA cost) is
// taken, waves counted from the kernel's measured occupancy.
#ifndef RQ_SPLIT_OVERHEAD_TILES
#define RQ_SPLIT_OVERHEAD_TILES 2
#endif
void choose_splits(const rq_cache *c, int T, int units, int which, int *S, int *chunk) {
    if (T <= 0) {
        *S = 0;
        *chunk = kTokTile;
        return;
    }
    const int s_lo = (T + kMaxChunk - 1) / kMaxChunk;
    const int s_hi = std::min(c->lay.splits_max, (T + kTokTile - 1) / kTokTile);
    long best_cost = -1;
    int best_s = s_lo, best_ch = kMaxChunk;
    const int nt = (T + kTokTile - 1) / kTokTile;
    for (int s = s_lo; s <= std::max(s_lo, s_hi); s++) {
        const int ch = (nt + s - 1) / s * kTokTile;
        const int ss = s;
        const int slots = std::max(1, c->occ[which][ch / kTokTile - 1] * c->sms);
        const long waves = ((long)ss * units + slots - 1) / slots;
        const long cost = waves * (ch + RQ_SPLIT_OVERHEAD_TILES * kTokTile);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best_s = ss;
            best_ch = ch;
        }
    }
#ifdef RQ_SPLIT_FORCE_S
    if (RQ_SPLIT_FORCE_S >= s_lo && RQ_SPLIT_FORCE_S <= std::max(s_lo, s_hi)) {
        best_s = RQ_SPLIT_FORCE_S;
        best_ch = (nt + best_s - 1) / best_s * kTokTile;
    }
#endif
    *S = best_s;
    *chunk = best_ch;
}

}  // namespace

namespace rq {

bool make_layout(const rq_config &cfg, Layout *out) {
    Layout L;
    std::memset(&L, 0, sizeof(L));
    L.cfg = cfg;
    const size_t B = cfg.batch, H = cfg.num_kv_heads, Hq = cfg.num_q_heads;
    if (cfg.format == RQ_FMT_RESIDUAL) {
        L.rec.a_codes = kHeadDim * cfg.anchor_bits / 8;
        L.rec.r_codes = kHeadDim * cfg.resid_bits / 8;
        L.rec.meta = (kHeadDim / cfg.group_size) * 2;
    }
    L.Lg = cfg.loops_per_group;
    L.groups = cfg.num_loops / cfg.loops_per_group;
    L.Tp = (int)align_up((size_t)cfg.max_tokens, kTokTile);
    L.tail_cap = cfg.max_tail_tokens;
    L.splits_max = std::min(kMaxSplits, L.Tp / kTokTile);
    L.paged = cfg.block_tokens > 0;
    L.BT = L.paged ? cfg.block_tokens : L.Tp;
    L.NBLK = L.paged ? cfg.num_blocks : cfg.batch;
    L.MB = L.paged ? (cfg.max_tokens + cfg.block_tokens - 1) / cfg.block_tokens : 1;
    // rows of every record array: blocks x heads x tokens per block
    const size_t bht = (size_t)L.NBLK * H * (size_t)L.BT;
    if (cfg.format == RQ_FMT_RESIDUAL) {
        L.anchor_codes_bytes = align_up(bht * L.rec.a_codes, kAlign);
        L.anchor_meta_bytes = align_up(bht * L.rec.meta, kAlign);
        L.anchor_block = 2 * (L.anchor_codes_bytes + L.anchor_meta_bytes);
        L.resid_codes_bytes = align_up(bht * L.rec.r_codes, kAlign);
        L.resid_meta_bytes = align_up(bht * L.rec.meta, kAlign);
        L.resid_coef_bytes = align_up(bht * 2, kAlign);
        L.resid_block = 2 * (L.resid_codes_bytes + L.resid_meta_bytes + L.resid_coef_bytes);
        L.tail_bytes = align_up(B * (size_t)L.tail_cap * H * kHeadDim * 2, kAlign);
        L.tail_block = 2 * L.tail_bytes;
        L.group_block = L.anchor_block + (size_t)(L.Lg - 1) * (L.resid_block + L.tail_block);
        L.records_bytes = (size_t)cfg.num_layers * L.groups * L.group_block;
    } else {
        L.bf16_side = align_up(bht * kHeadDim * 2, kAlign);
        L.bf16_block = 2 * L.bf16_side;
        L.records_bytes = (size_t)cfg.num_layers * cfg.num_loops * L.bf16_block;
    }
    L.off_records = 0;
    L.off_partials = align_up(L.records_bytes, kAlign);
    size_t partial_bytes = align_up(B * Hq * (size_t)L.splits_max * kPartialStride * sizeof(float), kAlign);
    L.off_counters = L.off_partials + partial_bytes;
    L.off_err = L.off_counters + align_up(B * Hq * sizeof(int), kAlign);
    L.off_vmax = L.off_err + kAlign;
    const size_t vmax_bytes = cfg.format == RQ_FMT_RESIDUAL
                                  ? align_up((size_t)cfg.num_layers * L.groups * L.Lg * B * H * sizeof(int), kAlign)
                                  : 0;
    L.off_table = L.off_vmax + vmax_bytes;
    const size_t table_bytes = L.paged ? align_up(B * (size_t)L.MB * sizeof(int), kAlign) : 0;
    L.total = L.off_table + table_bytes;
    *out = L;
    return true;
}

}  // namespace rq

extern "C" {

const char *rq_status_string(int status) {
    switch (status) {
    case RQ_OK: return "ok";
    case RQ_ERR_INVALID: return "invalid argument";
    case RQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case RQ_ERR_NOMEM: return "out of memory / arena too small";
    case RQ_ERR_CAPACITY: return "capacity exceeded";
    case RQ_ERR_STATE: return "call out of order / wrong cache format";
    case RQ_ERR_CUDA: return "CUDA error";
    case RQ_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
    }
}

int rq_config_check(const rq_config *c) {
    if (!c) return RQ_ERR_INVALID;
    if (c->num_layers < 1 || c->num_loops < 1 || c->loops_per_group < 1 || c->batch < 1 ||
        c->max_tokens < 1 || c->max_tail_tokens < 0 || c->num_kv_heads < 1 || c->num_q_heads < 1)
        return RQ_ERR_INVALID;
    if (c->num_loops % c->loops_per_group != 0) return RQ_ERR_INVALID;
    if (c->num_q_heads % c->num_kv_heads != 0) return RQ_ERR_INVALID;
    if (c->format != RQ_FMT_RESIDUAL && c->format != RQ_FMT_BF16) return RQ_ERR_INVALID;
    if (c->rotate != 0 && c->rotate != 1) return RQ_ERR_INVALID;
    if (c->scale_mode < 0 || c->scale_mode > 2 || c->anchor_mode < 0 || c->anchor_mode > 1 ||
        c->rotation_per_layer < 0 || c->rotation_per_layer > 1 || c->block_tokens < 0 || c->num_blocks < 0)
        return RQ_ERR_INVALID;
    if (c->block_tokens != 0) {
        if (c->block_tokens != 128 && c->block_tokens != 256) return RQ_ERR_UNSUPPORTED;
        if (c->format != RQ_FMT_RESIDUAL) return RQ_ERR_UNSUPPORTED;
        if (c->loops_per_group > 16) return RQ_ERR_UNSUPPORTED;   // copy-on-write covers groups of up to 16 loops
        if (c->num_blocks < 1) return RQ_ERR_INVALID;
    } else if (c->num_blocks != 0) {
        return RQ_ERR_INVALID;
    }
    if (c->format == RQ_FMT_BF16 && (c->scale_mode != 0 || c->anchor_mode != 0)) return RQ_ERR_INVALID;
    int G = c->num_q_heads / c->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return RQ_ERR_UNSUPPORTED;
    if (c->head_dim != kHeadDim) return RQ_ERR_UNSUPPORTED;
    if (c->format == RQ_FMT_RESIDUAL) {
        if (c->group_size != 16 && c->group_size != 32) return RQ_ERR_UNSUPPORTED;
        if (c->anchor_bits != 2 && c->anchor_bits != 4) return RQ_ERR_UNSUPPORTED;
        if (c->resid_bits != 2 && c->resid_bits != 4) return RQ_ERR_UNSUPPORTED;
        if (c->loops_per_group > 1 && c->max_tail_tokens < 1) return RQ_ERR_INVALID;
    }
    // size sanity: every per-stream offset must fit the kernels' 64-bit math
    // and the token index the kernels' 32-bit math
    if (c->max_tokens > kMaxSplits * kMaxChunk || c->max_tail_tokens > (1 << 20)) return RQ_ERR_UNSUPPORTED;
    if (c->batch > kMaxBatch) return RQ_ERR_UNSUPPORTED;
    return RQ_OK;
}

size_t rq_cache_required_bytes(const rq_config *cfg) {
    if (rq_config_check(cfg) != RQ_OK) return 0;
    Layout L;
    make_layout(*cfg, &L);
    return L.total;
}

size_t rq_cache_token_bytes(const rq_config *c) {
    if (rq_config_check(c) != RQ_OK) return 0;
    const size_t heads = (size_t)c->num_kv_heads, layers = (size_t)c->num_layers;
    if (c->format == RQ_FMT_BF16)
        return layers * c->num_loops * heads * 2 * kHeadDim * 2;
    const size_t meta = (kHeadDim / c->group_size) * 2;
    const size_t a = kHeadDim * c->anchor_bits / 8 + meta;
    const size_t r = kHeadDim * c->resid_bits / 8 + meta + 2;
    const size_t groups = c->num_loops / c->loops_per_group;
    return layers * heads * 2 * groups * (a + (size_t)(c->loops_per_group - 1) * r);
}

int rq_cache_create(const rq_config *cfg, void *dev_mem, size_t bytes, rq_cache **out) {
    if (!out) return RQ_ERR_INVALID;
    *out = nullptr;
    int st = rq_config_check(cfg);
    if (st != RQ_OK) return st;
    rq_cache *c = new (std::nothrow) rq_cache();
    if (!c) return RQ_ERR_NOMEM;
    make_layout(*cfg, &c->lay);
    if (cudaGetDevice(&c->device) != cudaSuccess) {
        delete c;
        return RQ_ERR_CUDA;
    }
    cudaDeviceGetAttribute(&c->sms, cudaDevAttrMultiProcessorCount, c->device);
    if (dev_mem) {
        if (bytes < c->lay.total || ((uintptr_t)dev_mem % kAlign) != 0) {
            delete c;
            return RQ_ERR_NOMEM;
        }
        c->base = (uint8_t *)dev_mem;
        c->owned = false;
    } else {
        void *p = nullptr;
        if (cudaMalloc(&p, c->lay.total) != cudaSuccess) {
            cudaGetLastError();
            delete c;
            return RQ_ERR_NOMEM;
        }
        c->base = (uint8_t *)p;
        c->owned = true;
    }
    if (cudaMemset(c->base, 0, c->lay.total) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
        if (c->owned) cudaFree(c->base);
        delete c;
        return RQ_ERR_CUDA;
    }
    const Layout &L = c->lay;
    c->len.assign((size_t)cfg->num_layers * (cfg->format == RQ_FMT_RESIDUAL ? L.groups : cfg->num_loops), 0);
    c->seq.assign(c->len.size() * (size_t)cfg->batch, 0);
    c->ntail.assign((size_t)cfg->num_layers * cfg->num_loops, 0);
    c->wstart.assign(c->len.size(), 0x7FFFFFFF);
    if (L.paged) {
        c->table.assign((size_t)cfg->batch * L.MB, -1);
        c->ref.assign(L.NBLK, 0);
        c->free_blocks.resize(L.NBLK);
        for (int i = 0; i < L.NBLK; i++) c->free_blocks[i] = L.NBLK - 1 - i;   // block 0 first
    }
    {
        const int G = cfg->num_q_heads / cfg->num_kv_heads;
        for (int i = 0; i < kMaxChunk / kTokTile; i++) {
            const int ch = kTokTile * (i + 1);
            for (int nr = 0; nr <= kMaxChain; nr++) {
                if (cfg->format == RQ_FMT_BF16)
                    c->occ[nr][i] = decode_bf16_occupancy(G, ch);
                else if (nr <= 1 || (cfg->anchor_mode == 1 && nr < cfg->loops_per_group &&
                                     decode_rq_supported(cfg->anchor_bits, cfg->resid_bits, nr)))
                    c->occ[nr][i] = decode_rq_occupancy(G, cfg->anchor_bits, cfg->resid_bits, nr, cfg->group_size, ch);
                else
                    c->occ[nr][i] = 1;
            }
        }
        cudaGetLastError();
    }
    c->sigma.assign((size_t)cfg->num_layers * 4, 0u);
    if (cfg->rotate)
        for (int layer = 0; layer < cfg->num_layers; layer++) {
            const uint64_t seed = cfg->seed + (cfg->rotation_per_layer ? (uint64_t)layer << 32 : 0);
            for (int j = 0; j < kHeadDim; j++)
                if (splitmix64(seed + (uint64_t)j) >> 63) c->sigma[(size_t)layer * 4 + j / 32] |= 1u << (j % 32);
        }
    *out = c;
    return RQ_OK;
}

int rq_cache_destroy(rq_cache *c) {
    if (!c) return RQ_OK;
    int st = RQ_OK;
    if (c->owned || c->prefill_ws || c->prefill_cnt) {
        if (cudaDeviceSynchronize() != cudaSuccess) st = RQ_ERR_CUDA;
    }
    if (c->owned) cudaFree(c->base);
    if (c->prefill_ws) cudaFree(c->prefill_ws);
    if (c->prefill_cnt) cudaFree(c->prefill_cnt);
    delete c;
    return st;
}

int rq_append(rq_cache *c, int layer, int loop, const void *k, const void *v, int n, void *stream) {
    if (!c || !k || !v || n < 1) return RQ_ERR_INVALID;
    if (!on_cache_device(c)) return RQ_ERR_INVALID;
    const Layout &L = c->lay;
    const rq_config &cfg = L.cfg;
    if (layer < 0 || layer >= cfg.num_layers || loop < 0 || loop >= cfg.num_loops) return RQ_ERR_INVALID;
    cudaStream_t st = (cudaStream_t)stream;
    if (cfg.format == RQ_FMT_BF16) {
        const size_t slot = (size_t)layer * cfg.num_loops + loop;
        if (c->len[slot] + n > cfg.max_tokens) return RQ_ERR_CAPACITY;
        Bf16StoreArgs a;
        a.src[0] = (const uint16_t *)k;
        a.src[1] = (const uint16_t *)v;
        a.dst[0] = bf16_ptr(c, layer, loop, 0);
        a.dst[1] = bf16_ptr(c, layer, loop, 1);
        a.B = cfg.batch;
        a.H = cfg.num_kv_heads;
        a.n = n;
        fill_lens(seq_lens(c, slot), cfg.batch, &a.pos0);
        a.Tp = L.Tp;
        int s = cuda_status(launch_bf16_store(a, st));
        if (s == RQ_OK) grow(c, slot, n);
        return s;
    }
    const int group = loop / L.Lg, j = loop % L.Lg;
    const size_t slot = (size_t)layer * L.groups + group;
    if (!is_commit_loop(L, loop)) {
        int &nt = c->ntail[(size_t)layer * cfg.num_loops + loop];
        if (nt + n > L.tail_cap) return RQ_ERR_CAPACITY;
        TailArgs a;
        a.src[0] = (const uint16_t *)k;
        a.src[1] = (const uint16_t *)v;
        a.dst[0] = (uint16_t *)tail_ptr(c, layer, group, j, 0);
        a.dst[1] = (uint16_t *)tail_ptr(c, layer, group, j, 1);
        a.B = cfg.batch;
        a.H = cfg.num_kv_heads;
        a.n = n;
        a.pos0 = nt;
        a.cap = L.tail_cap;
        int s = cuda_status(launch_tail_copy(a, st));
        if (s == RQ_OK) nt += n;
        return s;
    }
    // anchor loop: every other loop of the group must hold exactly these n tokens
    for (int jj = 0; jj < L.Lg - 1; jj++)
        if (c->ntail[(size_t)layer * cfg.num_loops + group * L.Lg + jj] != n) return RQ_ERR_STATE;
    if (c->len[slot] + n > cfg.max_tokens) return RQ_ERR_CAPACITY;
    AppendArgs a;
    std::memset(&a, 0, sizeof(a));
    a.x_anchor[0] = (const uint16_t *)k;
    a.x_anchor[1] = (const uint16_t *)v;
    a.nres = L.Lg - 1;
    if (a.nres > 0) {
        a.tail0 = tail_ptr(c, layer, group, 0, 0);
        a.tail_loop_stride = L.tail_block;
        a.tail_kv_stride = L.tail_bytes;
        a.r_codes0 = resid_codes(c, layer, group, 0, 0);
        a.r_meta0 = resid_meta(c, layer, group, 0, 0);
        a.r_coef0 = resid_coef(c, layer, group, 0, 0);
        a.resid_loop_stride = L.resid_block;
        a.resid_kv_stride = resid_side(L);
    }
    a.a_codes0 = anchor_codes(c, layer, group, 0);
    a.a_meta0 = anchor_meta(c, layer, group, 0);
    a.anchor_kv_stride = L.anchor_codes_bytes + L.anchor_meta_bytes;
    a.vmax = vmax_ptr(c, layer, group, 0);
    a.B = cfg.batch;
    a.H = cfg.num_kv_heads;
    a.n = n;
    fill_lens(seq_lens(c, slot), cfg.batch, &a.pos0);
    a.pg = pages_of(c);
    a.tail_cap = L.tail_cap;
    a.g = cfg.group_size;
    a.ba = cfg.anchor_bits;
    a.br = cfg.resid_bits;
    a.rotate = cfg.rotate;
    a.scale_mode = cfg.scale_mode;
    a.chained = cfg.anchor_mode;
    std::memcpy(a.sigma, &c->sigma[(size_t)layer * 4], sizeof(a.sigma));
    if (L.paged) {
        const int sb = prepare_blocks(c, a.pos0, n, st);
        if (sb != RQ_OK) return sb;
    }
    int s = cuda_status(launch_append(a, st));
    if (s != RQ_OK) return s;
    int w0 = 0x7FFFFFFF;
    for (int b = 0; b < cfg.batch; b++) w0 = std::min(w0, a.pos0.v[b]);
    c->wstart[slot] = w0;
    grow(c, slot, n);
    for (int jj = 0; jj < L.Lg - 1; jj++) c->ntail[(size_t)layer * cfg.num_loops + group * L.Lg + jj] = 0;
    return RQ_OK;
}

// partials == nullptr: split partials and combine counters in the cache's
// workspace (partial stride splits_max).  Otherwise in the caller's scratch
// (stride = the split count this call uses).
// app_k != nullptr: append app_n tokens to the loop first (rq_append_decode_attn).
static int decode_common(rq_cache *c, int layer, int loop, const void *q, float *out, float scale,
                         void *stream, bool bf16, float *partials = nullptr, size_t partial_floats = 0,
                         int *counters = nullptr, size_t max_units = 0, const void *app_k = nullptr,
                         const void *app_v = nullptr, int app_n = 0) {
    if (!c || !q || !out) return RQ_ERR_INVALID;
    if (!on_cache_device(c)) return RQ_ERR_INVALID;
    const Layout &L = c->lay;
    const rq_config &cfg = L.cfg;
    if (layer < 0 || layer >= cfg.num_layers || loop < 0 || loop >= cfg.num_loops) return RQ_ERR_INVALID;
    if ((cfg.format == RQ_FMT_BF16) != bf16) return RQ_ERR_STATE;
    cudaStream_t st = (cudaStream_t)stream;
    DecodeArgs a;
    std::memset(&a, 0, sizeof(a));
    a.q = (const uint16_t *)q;
    a.out = out;
    a.partials = (float *)(c->base + L.off_partials);
    a.counters = (int *)(c->base + L.off_counters);
    a.err = (int *)(c->base + L.off_err);
    a.B = cfg.batch;
    a.H = cfg.num_kv_heads;
    a.Hq = cfg.num_q_heads;
    a.G = cfg.num_q_heads / cfg.num_kv_heads;
    a.Tp = L.Tp;
    a.pg = pages_of(c);
    a.splits_max = L.splits_max;
    a.g = cfg.group_size;
    a.scale_log2 = resolve_scale(scale) * 1.4426950408889634f;
    a.rotate = cfg.rotate;
    a.tail_cap = L.tail_cap;
    std::memcpy(a.sigma, &c->sigma[(size_t)layer * 4], sizeof(a.sigma));
    if (bf16) {
        a.T = c->len[(size_t)layer * cfg.num_loops + loop];
        fill_lens(seq_lens(c, (size_t)layer * cfg.num_loops + loop), cfg.batch, &a.seqT);
        a.bf[0] = bf16_ptr(c, layer, loop, 0);
        a.bf[1] = bf16_ptr(c, layer, loop, 1);
    } else {
        const int group = loop / L.Lg, j = loop % L.Lg;
        a.T = c->len[(size_t)layer * L.groups + group];
        fill_lens(seq_lens(c, (size_t)layer * L.groups + group), cfg.batch, &a.seqT);
        for (int kv = 0; kv < 2; kv++) {
            a.a_codes[kv] = anchor_codes(c, layer, group, kv);
            a.a_meta[kv] = anchor_meta(c, layer, group, kv);
        }
        a.vmax_a = vmax_ptr(c, layer, group, L.Lg - 1);
        a.stable = c->wstart[(size_t)layer * L.groups + group];
        if (L.paged && c->table_dirty) {
            // the table may have changed in the kernel just before this one
            a.stable = 0;
            c->table_dirty = false;
        }
        if (!is_commit_loop(L, loop)) {
            a.n_tail = c->ntail[(size_t)layer * cfg.num_loops + loop];
            a.tail_k = (const uint16_t *)tail_ptr(c, layer, group, j, 0);
            a.tail_v = (const uint16_t *)tail_ptr(c, layer, group, j, 1);
        }
        // residual records read: the loop's own (shared reference), or the
        // chain of records 0 .. slot (chained reference)
        const int slot = record_slot(L, loop);
        const int r0 = cfg.anchor_mode == 1 ? 0 : slot;
        a.nr = slot < 0 ? 0 : slot - r0 + 1;
        if (!decode_rq_supported(cfg.anchor_bits, cfg.resid_bits, a.nr)) return RQ_ERR_UNSUPPORTED;
        for (int r = 0; r < a.nr; r++) {
            a.vmax_r[r] = vmax_ptr(c, layer, group, r0 + r);
            for (int kv = 0; kv < 2; kv++) {
                a.r_codes[r][kv] = resid_codes(c, layer, group, r0 + r, kv);
                a.r_meta[r][kv] = resid_meta(c, layer, group, r0 + r, kv);
                a.r_coef[r][kv] = (const uint16_t *)resid_coef(c, layer, group, r0 + r, kv);
            }
        }
    }
    const int units = a.B * a.H * (a.G > 2 ? a.G / 2 : 1);
    choose_splits(c, a.T, units, bf16 ? 0 : a.nr, &a.S, &a.chunk);
    if (partials) {
        a.splits_max = std::max(a.S, 1);
        if ((size_t)a.B * a.Hq * a.splits_max * kPartialStride > partial_floats) return RQ_ERR_CAPACITY;
        if ((size_t)a.B * a.Hq > max_units) return RQ_ERR_CAPACITY;
        a.partials = partials;
        a.counters = counters;
    }
    if (app_k) {
        // one launch when the loop keeps the tokens in its tail and the split
        // kernel runs (it writes the rows, then merges them); else append first
        if (!(!bf16 && !is_commit_loop(L, loop) && a.S > 0)) {
            int s = rq_append(c, layer, loop, app_k, app_v, app_n, stream);
            if (s != RQ_OK) return s;
            return decode_common(c, layer, loop, q, out, scale, stream, bf16);
        }
        int &nt = c->ntail[(size_t)layer * cfg.num_loops + loop];
        if (nt + app_n > L.tail_cap) return RQ_ERR_CAPACITY;
        const int group = loop / L.Lg, j = loop % L.Lg;
        a.new_k = (const uint16_t *)app_k;
        a.new_v = (const uint16_t *)app_v;
        a.tail_k_w = (uint16_t *)tail_ptr(c, layer, group, j, 0);
        a.tail_v_w = (uint16_t *)tail_ptr(c, layer, group, j, 1);
        a.n_new = app_n;
        a.tail_pos = nt;
        a.n_tail = nt + app_n;
        int s = cuda_status(launch_decode_rq(a, cfg.anchor_bits, cfg.resid_bits, st));
        if (s == RQ_OK) nt += app_n;
        return s;
    }
    if (!bf16 && a.S > 0)   // the decode kernel merges its splits and the tail itself
        return cuda_status(launch_decode_rq(a, cfg.anchor_bits, cfg.resid_bits, st));
    if (bf16 && a.S > 0) {
        cudaError_t e = launch_decode_bf16(a, st);
        if (e != cudaSuccess) return RQ_ERR_CUDA;
    }
    CombineArgs cb;
    std::memset(&cb, 0, sizeof(cb));
    cb.partials = a.partials;
    cb.q = a.q;
    cb.out = out;
    cb.tail_k = a.tail_k;
    cb.tail_v = a.tail_v;
    cb.B = a.B;
    cb.H = a.H;
    cb.Hq = a.Hq;
    cb.G = a.G;
    cb.S = a.S;
    cb.splits_max = a.splits_max;
    cb.n_tail = a.n_tail;
    cb.tail_cap = L.tail_cap;
    cb.scale_log2 = a.scale_log2;
    return cuda_status(launch_combine(cb, st));
}

}  // extern "C"

namespace rq {
int cache_device(const rq_cache *c) { return c->device; }

int decode_with_scratch(rq_cache *c, int layer, int loop, const void *q, float *out, float scale, void *stream,
                        float *partials, size_t partial_floats, int *counters, size_t max_units) {
    if (!partials || !counters) return RQ_ERR_INVALID;
    return decode_common(c, layer, loop, q, out, scale, stream, false, partials, partial_floats, counters,
                         max_units);
}
}  // namespace rq

extern "C" {

int rq_decode_attn(rq_cache *c, int layer, int loop, const void *q, float *out, float scale, void *stream) {
    return decode_common(c, layer, loop, q, out, scale, stream, false);
}

int rq_append_decode_attn(rq_cache *c, int layer, int loop, const void *k, const void *v, int n,
                          const void *q, float *out, float scale, void *stream) {
    if (!c || !k || !v || n <= 0) return RQ_ERR_INVALID;
    if (c->lay.cfg.format != RQ_FMT_RESIDUAL) return RQ_ERR_STATE;
    return decode_common(c, layer, loop, q, out, scale, stream, false, nullptr, 0, nullptr, 0, k, v, n);
}

int rq_decode_attn_bf16(rq_cache *c, int layer, int loop, const void *q, float *out, float scale,
                        void *stream) {
    return decode_common(c, layer, loop, q, out, scale, stream, true);
}

int rq_prefill_attn(rq_cache *c, int layer, int loop, const void *q, int n, float *out, float scale,
                    void *stream) {
    if (!c || !q || !out || n <= 0) return RQ_ERR_INVALID;
    if (!on_cache_device(c)) return RQ_ERR_INVALID;
    const Layout &L = c->lay;
    const rq_config &cfg = L.cfg;
    if (layer < 0 || layer >= cfg.num_layers || loop < 0 || loop >= cfg.num_loops) return RQ_ERR_INVALID;
    if (cfg.format != RQ_FMT_RESIDUAL) return RQ_ERR_STATE;
    // the multi-token kernel is built for INT4/INT2, INT2/INT2 and INT4/INT4,
    // the last-loop reference (contiguous or paged records)
    if (cfg.anchor_bits == 2 && cfg.resid_bits == 4) return RQ_ERR_UNSUPPORTED;
    if (cfg.anchor_mode != 0) return RQ_ERR_UNSUPPORTED;
    PrefillArgs a;
    std::memset(&a, 0, sizeof(a));
    const int group = loop / L.Lg, j = loop % L.Lg;
    const size_t slot = (size_t)layer * L.groups + group;
    const int T = c->len[slot];
    fill_lens(seq_lens(c, slot), cfg.batch, &a.seqT);
    a.pg = pages_of(c);
    for (int kv = 0; kv < 2; kv++) {
        a.a_codes[kv] = anchor_codes(c, layer, group, kv);
        a.a_meta[kv] = anchor_meta(c, layer, group, kv);
    }
    if (!is_commit_loop(L, loop)) {
        for (int kv = 0; kv < 2; kv++) {
            a.r_codes[kv] = resid_codes(c, layer, group, j, kv);
            a.r_meta[kv] = resid_meta(c, layer, group, j, kv);
            a.r_coef[kv] = (const uint16_t *)resid_coef(c, layer, group, j, kv);
        }
        a.n_tail = c->ntail[(size_t)layer * cfg.num_loops + loop];
        a.tail_k = (const uint16_t *)tail_ptr(c, layer, group, j, 0);
        a.tail_v = (const uint16_t *)tail_ptr(c, layer, group, j, 1);
    }
    // the n new tokens must be the most recent of every sequence
    for (int b = 0; b < cfg.batch; b++)
        if (a.seqT.v[b] + a.n_tail < n) return RQ_ERR_STATE;
    a.q = (const uint16_t *)q;
    a.out = out;
    a.B = cfg.batch;
    a.H = cfg.num_kv_heads;
    a.Hq = cfg.num_q_heads;
    a.G = cfg.num_q_heads / cfg.num_kv_heads;
    a.n = n;
    a.tail_cap = L.tail_cap;
    a.Tp = L.Tp;
    a.g = cfg.group_size;
    a.scale_log2 = resolve_scale(scale) * 1.4426950408889634f;
    a.rotate = cfg.rotate;
    std::memcpy(a.sigma, &c->sigma[(size_t)layer * 4], sizeof(a.sigma));
    if (n > 65535) return RQ_ERR_UNSUPPORTED;   // grid limit
    prefill_plan(&a, T, cfg.anchor_bits, cfg.resid_bits, c->sms);
    if ((long)a.B * a.nqb > 65535) return RQ_ERR_UNSUPPORTED;
    const size_t need = (size_t)a.B * n * a.Hq * std::max(a.S, 1) * kPartialStride;
    if (need > c->prefill_ws_floats) {
        if (c->prefill_ws) {
            if (cudaDeviceSynchronize() != cudaSuccess) return RQ_ERR_CUDA;
            cudaFree(c->prefill_ws);
            c->prefill_ws = nullptr;
            c->prefill_ws_floats = 0;
        }
        void *p = nullptr;
        if (cudaMalloc(&p, need * sizeof(float)) != cudaSuccess) {
            cudaGetLastError();
            return RQ_ERR_NOMEM;
        }
        c->prefill_ws = (float *)p;
        c->prefill_ws_floats = need;
    }
    a.partials = c->prefill_ws;
    a.counters = nullptr;
    if (a.S > 0) {
        const size_t units = (size_t)a.B * a.H * a.nqb;
        if (units > c->prefill_cnt_n) {
            if (c->prefill_cnt) {
                if (cudaDeviceSynchronize() != cudaSuccess) return RQ_ERR_CUDA;
                cudaFree(c->prefill_cnt);
                c->prefill_cnt = nullptr;
                c->prefill_cnt_n = 0;
            }
            void *p = nullptr;
            if (cudaMalloc(&p, units * sizeof(int)) != cudaSuccess) {
                cudaGetLastError();
                return RQ_ERR_NOMEM;
            }
            if (cudaMemset(p, 0, units * sizeof(int)) != cudaSuccess) {
                cudaFree(p);
                return RQ_ERR_CUDA;
            }
            c->prefill_cnt = (int *)p;
            c->prefill_cnt_n = units;
        }
        a.counters = c->prefill_cnt;
    }
    a.err = (int *)(c->base + L.off_err);
    return cuda_status(launch_prefill(a, cfg.anchor_bits, cfg.resid_bits, (cudaStream_t)stream));
}

int rq_cache_length(const rq_cache *c, int layer, int group, int *len) {
    if (!c || !len) return RQ_ERR_INVALID;
    const Layout &L = c->lay;
    int ngroups = L.cfg.format == RQ_FMT_RESIDUAL ? L.groups : L.cfg.num_loops;
    if (layer < 0 || layer >= L.cfg.num_layers || group < 0 || group >= ngroups) return RQ_ERR_INVALID;
    *len = c->len[(size_t)layer * ngroups + group];
    return RQ_OK;
}

int rq_cache_tail_length(const rq_cache *c, int layer, int loop, int *n) {
    if (!c || !n) return RQ_ERR_INVALID;
    const Layout &L = c->lay;
    if (layer < 0 || layer >= L.cfg.num_layers || loop < 0 || loop >= L.cfg.num_loops) return RQ_ERR_INVALID;
    *n = c->ntail[(size_t)layer * L.cfg.num_loops + loop];
    return RQ_OK;
}

int rq_cache_truncate(rq_cache *c, int layer, int group, int new_len) {
    if (!c) return RQ_ERR_INVALID;
    const Layout &L = c->lay;
    int ngroups = L.cfg.format == RQ_FMT_RESIDUAL ? L.groups : L.cfg.num_loops;
    if (layer < 0 || layer >= L.cfg.num_layers || group < 0 || group >= ngroups) return RQ_ERR_INVALID;
    const size_t slot = (size_t)layer * ngroups + group;
    if (new_len < 0 || new_len > c->len[slot]) return RQ_ERR_INVALID;
    if (L.cfg.format == RQ_FMT_RESIDUAL)
        for (int jj = 0; jj < L.Lg - 1; jj++)
            if (c->ntail[(size_t)layer * L.cfg.num_loops + group * L.Lg + jj] != 0) return RQ_ERR_STATE;
    int *v = seq_lens(c, slot), mx = 0;
    for (int b = 0; b < L.cfg.batch; b++) mx = std::max(mx, v[b] = std::min(v[b], new_len));
    c->len[slot] = mx;
    if (L.paged)
        for (int b = 0; b < L.cfg.batch; b++) release_blocks(c, b, blocks_needed(c, b));
    return RQ_OK;
}

int rq_cache_truncate_seq(rq_cache *c, int layer, int group, int seq, int new_len) {
    if (!c) return RQ_ERR_INVALID;
    const Layout &L = c->lay;
    int ngroups = L.cfg.format == RQ_FMT_RESIDUAL ? L.groups : L.cfg.num_loops;
    if (layer < 0 || layer >= L.cfg.num_layers || group < 0 || group >= ngroups || seq < 0 || seq >= L.cfg.batch)
        return RQ_ERR_INVALID;
    const size_t slot = (size_t)layer * ngroups + group;
    int *v = seq_lens(c, slot);
    if (new_len < 0 || new_len > v[seq]) return RQ_ERR_INVALID;
    if (L.cfg.format == RQ_FMT_RESIDUAL)
        for (int jj = 0; jj < L.Lg - 1; jj++)
            if (c->ntail[(size_t)layer * L.cfg.num_loops + group * L.Lg + jj] != 0) return RQ_ERR_STATE;
    v[seq] = new_len;
    int mx = 0;
    for (int b = 0; b < L.cfg.batch; b++) mx = std::max(mx, v[b]);
    c->len[slot] = mx;
    if (L.paged) release_blocks(c, seq, blocks_needed(c, seq));
    return RQ_OK;
}

int rq_cache_length_seq(const rq_cache *c, int layer, int group, int seq, int *len) {
    if (!c || !len) return RQ_ERR_INVALID;
    const Layout &L = c->lay;
    int ngroups = L.cfg.format == RQ_FMT_RESIDUAL ? L.groups : L.cfg.num_loops;
    if (layer < 0 || layer >= L.cfg.num_layers || group < 0 || group >= ngroups || seq < 0 || seq >= L.cfg.batch)
        return RQ_ERR_INVALID;
    *len = seq_lens(c, (size_t)layer * ngroups + group)[seq];
    return RQ_OK;
}

int rq_cache_export(const rq_cache *c, int layer, int loop, void *host_codes, void *host_meta, void *host_coef,
                    void *stream) {
    if (!c || !host_codes || !host_meta) return RQ_ERR_INVALID;
    if (!on_cache_device(c)) return RQ_ERR_INVALID;
    const Layout &L = c->lay;
    const rq_config &cfg = L.cfg;
    if (cfg.format != RQ_FMT_RESIDUAL) return RQ_ERR_STATE;
    if (layer < 0 || layer >= cfg.num_layers || loop < 0 || loop >= cfg.num_loops) return RQ_ERR_INVALID;
    const int group = loop / L.Lg, j = record_slot(L, loop);
    const bool anchor = j < 0;
    if (!anchor && !host_coef) return RQ_ERR_INVALID;
    const int len = c->len[(size_t)layer * L.groups + group];
    const size_t bh = (size_t)cfg.batch * cfg.num_kv_heads;
    cudaStream_t st = (cudaStream_t)stream;
    if (len == 0) return RQ_OK;
    const size_t crec = anchor ? L.rec.a_codes : L.rec.r_codes;
    // one array [blocks][H][BT][rec] -> host [B][H][len][rec]: contiguous
    // caches copy each sequence's block whole; paged ones every allocated
    // block of every sequence (rows past a sequence's length are left as they are)
    auto copy_array = [&](uint8_t *host, const uint8_t *dev, size_t rec) -> cudaError_t {
        const int H = cfg.num_kv_heads;
        if (!L.paged)
            return cudaMemcpy2DAsync(host, len * rec, dev, (size_t)L.BT * rec, len * rec, bh, cudaMemcpyDeviceToHost,
                                     st);
        for (int b = 0; b < cfg.batch; b++)
            for (int k = 0; k * L.BT < len; k++) {
                const int blk = c->table[(size_t)b * L.MB + k];
                if (blk < 0) continue;
                const size_t cnt = std::min(L.BT, len - k * L.BT);
                cudaError_t e = cudaMemcpy2DAsync(host + ((size_t)b * H * len + (size_t)k * L.BT) * rec, len * rec,
                                                  dev + (size_t)blk * H * L.BT * rec, (size_t)L.BT * rec, cnt * rec,
                                                  H, cudaMemcpyDeviceToHost, st);
                if (e != cudaSuccess) return e;
            }
        return cudaSuccess;
    };
    for (int kv = 0; kv < 2; kv++) {
        const uint8_t *codes = anchor ? anchor_codes(c, layer, group, kv) : resid_codes(c, layer, group, j, kv);
        const uint8_t *meta = anchor ? anchor_meta(c, layer, group, kv) : resid_meta(c, layer, group, j, kv);
        uint8_t *hc = (uint8_t *)host_codes + kv * bh * len * crec;
        uint8_t *hm = (uint8_t *)host_meta + kv * bh * len * L.rec.meta;
        cudaError_t e = copy_array(hc, codes, crec);
        if (e == cudaSuccess) e = copy_array(hm, meta, L.rec.meta);
        if (e == cudaSuccess && !anchor) {
            uint8_t *hf = (uint8_t *)host_coef + kv * bh * len * 2;
            e = copy_array(hf, resid_coef(c, layer, group, j, kv), 2);
        }
        if (e != cudaSuccess) return RQ_ERR_CUDA;
    }
    return cuda_status(cudaStreamSynchronize(st));
}

size_t rq_decode_bytes(const rq_cache *c, int layer, int loop) {
    if (!c) return 0;
    const Layout &L = c->lay;
    const rq_config &cfg = L.cfg;
    if (layer < 0 || layer >= cfg.num_layers || loop < 0 || loop >= cfg.num_loops) return 0;
    const size_t bh = (size_t)cfg.batch * cfg.num_kv_heads;
    const size_t qo = (size_t)cfg.batch * cfg.num_q_heads * kHeadDim * (2 + 4);
    auto tokens = [&](size_t slot) {   // committed tokens summed over the sequences
        size_t t = 0;
        for (int b = 0; b < cfg.batch; b++) t += (size_t)seq_lens(c, slot)[b];
        return t;
    };
    if (cfg.format == RQ_FMT_BF16)
        return tokens((size_t)layer * cfg.num_loops + loop) * cfg.num_kv_heads * 2 * kHeadDim * 2 + qo;
    const int group = loop / L.Lg;
    const size_t T = tokens((size_t)layer * L.groups + group);
    size_t per = 2 * (size_t)(L.rec.a_codes + L.rec.meta);
    size_t tail = 0;
    // residual records read: the loop's own (last-loop reference) or all up
    // to its own (chained reference)
    const int slot = record_slot(L, loop);
    const int nres = slot < 0 ? 0 : cfg.anchor_mode == 1 ? slot + 1 : 1;
    per += 2 * (size_t)nres * (L.rec.r_codes + L.rec.meta + 2);
    if (!is_commit_loop(L, loop))
        tail = (size_t)c->ntail[(size_t)layer * cfg.num_loops + loop] * bh * 2 * kHeadDim * 2;
    return T * cfg.num_kv_heads * per + tail + qo;
}

int rq_cache_fork_seq(rq_cache *c, int src, int dst, void *stream) {
    if (!c) return RQ_ERR_INVALID;
    if (!on_cache_device(c)) return RQ_ERR_INVALID;
    const Layout &L = c->lay;
    const rq_config &cfg = L.cfg;
    if (!L.paged) return RQ_ERR_UNSUPPORTED;
    if (src < 0 || src >= cfg.batch || dst < 0 || dst >= cfg.batch || src == dst) return RQ_ERR_INVALID;
    for (int nt : c->ntail)
        if (nt != 0) return RQ_ERR_STATE;
    for (size_t slot = 0; slot < c->len.size(); slot++)
        if (c->seq[slot * cfg.batch + dst] != 0) return RQ_ERR_STATE;
    cudaStream_t st = (cudaStream_t)stream;
    PendingOps ops;
    for (int k = 0; k < L.MB; k++) {
        const int e = c->table[(size_t)src * L.MB + k];
        if (e < 0) continue;
        ops.sets.push_back({dst * L.MB + k, e});
    }
    // the largest V scales of dst's streams are src's: [layer][group][Lg][B][H] rows of H ints
    const size_t H = cfg.num_kv_heads;
    int *vm = (int *)(c->base + L.off_vmax);
    const size_t rows = (size_t)cfg.num_layers * L.groups * L.Lg;
    if (cudaMemcpy2DAsync(vm + dst * H, cfg.batch * H * sizeof(int), vm + src * H, cfg.batch * H * sizeof(int),
                          H * sizeof(int), rows, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return RQ_ERR_CUDA;
    int s = flush_ops(c, ops, st);
    if (s != RQ_OK) return s;
    for (int k = 0; k < L.MB; k++) {
        const int e = c->table[(size_t)src * L.MB + k];
        if (e < 0) continue;
        c->table[(size_t)dst * L.MB + k] = e;
        c->ref[e]++;
    }
    for (size_t slot = 0; slot < c->len.size(); slot++) c->seq[slot * cfg.batch + dst] = c->seq[slot * cfg.batch + src];
    return RQ_OK;
}

int rq_cache_shuffle_free_blocks(rq_cache *c, uint64_t seed) {
    if (!c) return RQ_ERR_INVALID;
    if (!c->lay.paged) return RQ_ERR_UNSUPPORTED;
    // Fisher-Yates with splitmix64 draws
    std::vector<int> &f = c->free_blocks;
    for (size_t i = f.size(); i > 1; i--) {
        const size_t j = (size_t)(splitmix64(seed + i) % i);
        std::swap(f[i - 1], f[j]);
    }
    return RQ_OK;
}

int rq_cache_free_blocks(const rq_cache *c, int *n) {
    if (!c || !n) return RQ_ERR_INVALID;
    if (!c->lay.paged) return RQ_ERR_UNSUPPORTED;
    *n = (int)c->free_blocks.size();
    return RQ_OK;
}

int rq_cache_seq_blocks(const rq_cache *c, int seq, int32_t *host_blocks, int max_blocks, int *n) {
    if (!c || !n) return RQ_ERR_INVALID;
    const Layout &L = c->lay;
    if (!L.paged) return RQ_ERR_UNSUPPORTED;
    if (seq < 0 || seq >= L.cfg.batch) return RQ_ERR_INVALID;
    int cnt = 0;
    while (cnt < L.MB && c->table[(size_t)seq * L.MB + cnt] >= 0) cnt++;
    *n = cnt;
    if (host_blocks)
        for (int k = 0; k < std::min(cnt, max_blocks); k++) host_blocks[k] = c->table[(size_t)seq * L.MB + k];
    return RQ_OK;
}

int rq_check(rq_cache *c) {
    if (!c) return RQ_ERR_INVALID;
    if (!on_cache_device(c)) return RQ_ERR_INVALID;
    if (cudaDeviceSynchronize() != cudaSuccess) return RQ_ERR_CUDA;
    int err = 0;
    if (cudaMemcpy(&err, c->base + c->lay.off_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return RQ_ERR_CUDA;
    if (err != 0) {
        // A call whose bounded wait gave up still counts every CTA's arrival
        // (consumers finish their pass over the data they have and reach the
        // counter), so its counters return to zero; they are cleared here
        // anyway, with the error word -- the cache's and the allocation-free
        // entry point's -- so that the next call starts clean whatever
        // happened.
        cudaMemset(c->base + c->lay.off_counters, 0, c->lay.off_err + sizeof(int) - c->lay.off_counters);
        noalloc_reset_counters();
        if (c->prefill_cnt) cudaMemset(c->prefill_cnt, 0, c->prefill_cnt_n * sizeof(int));
        if (cudaDeviceSynchronize() != cudaSuccess) return RQ_ERR_CUDA;
        return RQ_ERR_TIMEOUT;
    }
    // every completed rq_prefill_attn leaves its split-arrival counters at zero
    if (c->prefill_cnt) {
        std::vector<int> cnt(c->prefill_cnt_n);
        if (cudaMemcpy(cnt.data(), c->prefill_cnt, cnt.size() * sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
            return RQ_ERR_CUDA;
        for (int v : cnt) {
            if (v != 0) {
                cudaMemset(c->prefill_cnt, 0, c->prefill_cnt_n * sizeof(int));
                if (cudaDeviceSynchronize() != cudaSuccess) return RQ_ERR_CUDA;
                return RQ_ERR_STATE;
            }
        }
    }
    return RQ_OK;
}

}  // extern "C"
