// decode_rq.cu -- split-KV decode attention over the ResidualQuant cache
// (arXiv 2610.10381; ai4snews summary, paragraph 3: shared-anchor
// reconstruction needs two cache reads -- the anchor record and the loop's
// own residual record).
//
// Algebra.  For a committed token t of a non-anchor loop,
//   k_t = s_t * a_t + R^T y_t      (a_t anchor, y_t rotated residual)
// so  q.k_t = s_t (q.a_t) + (R q).y_t : q is rotated once per CTA instead of
// rotating every key.  Per 16-element segment of a quantization group
// (FP8 scale sc, FP8 minimum mn, integer codes c):
//   q_seg . x_hat_seg = mn * sum(q_seg) + sc * sum(q_i c_i)
// The V sum is accumulated the same way: the anchor part in the original
// basis, the residual part in the rotated basis; R^T is applied once per CTA
// to the rotated accumulator.
//
// Arithmetic.  The per-code products run on the integer dot-product units,
// which consume packed codes with no conversion to floating point:
//  - logits: q (and R q) are converted once per CTA to 24-bit fixed point
//    (power-of-two scale, |q| < 2^22) split into three byte planes, and
//    sum_i q_i c_i is three dp4a (4 products each) per 4 codes, exact;
//  - values: each weight p_t s_t sc_{g,t} becomes fixed point with a
//    power-of-two scale chosen from a bound of every weight of the chunk
//    (max |s_t| of the chunk times the largest V scale the encoder has
//    written to the (sequence, head) stream; mapped into [2^21, 2^22)),
//    split into 16-bit halves; sum_t w_t c_t,i is two dp2a (2 products each)
//    per 2 codes, exact.  The high halves are nonzero only for the largest
//    weights, and skipped when a warp has none for a token pair.
// The fixed-point rounding of q and of the weights is the only departure from
// fp32 arithmetic (relative 2^-21 of max|q|; absolute 2^-22 of the bound,
// which follows the actual V scales, so small-magnitude V keeps its relative
// precision).
//
// Programmatic launch.  The kernel may start while the previous kernel on
// its stream is still running (the host launches it with programmatic stream
// serialization): the producer streams committed records below a.stable --
// which no in-flight work writes -- before its grid-dependency wait; every
// other global access (q, the V scale bounds, records from a.stable on, the
// tail, partials, counters, out) comes after the wait.  A thread signals
// that the next kernel may start only after its own wait has returned, so at
// most one earlier kernel is ever still running.
// Per-group scales, minima, softmax and the final rotation stay in fp32.
//
// Data movement.  Each CTA owns a chunk of one (sequence, kv head) (the
// sequence's 64-token tiles dealt evenly over the splits) and streams it in
// 128-token items through a byte-addressed shared-memory ring filled by one
// producer warp with 1-D bulk asynchronous copies (cp.async.bulk, completion
// counted on mbarriers; no multicast): first the K records of every item
// (pass 1: logits), then the anchor V codes + meta, then the residual V codes
// + meta (pass 2: values).  Only the V coefficients of the chunk (2 bytes per
// token) are fetched once up front; the producer warp's other lanes take
// their maximum for the weights' fixed point.  Every mbarrier wait is
// bounded: on timeout the kernel records an error word, stops issuing copies,
// drains what it issued and finishes without touching further data.
//
// Split combine.  Each CTA writes its partial (max, sum, o); the last CTA of
// a (sequence, kv head) -- found with a device-wide counter, no waiting --
// merges all partials plus the loop's BF16 tail tokens and writes the output.
//
// Thread map (both passes): 4 consumer warps x 16 tokens of each 64-token
// tile of an item; lane 8s+j takes head_dim segment j (elements 16j..16j+15)
// of tokens s, s+4, s+8, s+12 of its warp's 16.
#include <math_constants.h>

#include "combine.cuh"
#include "common.cuh"
#include "rq_internal.h"
#include "sync.cuh"

#ifdef RQ_FAULT_INJECT
// Test builds only (never the shipped library): when set, the next decode
// launch's CTA (0, 0, 0) leaves the mbarrier of its second ring item unarmed
// -- it issues no copy for it -- so its consumers' bounded wait runs out.
__device__ int g_rq_fault_once;
extern "C" int rq_test_arm_fault(void) {
    const int one = 1;
    return cudaMemcpyToSymbol(g_rq_fault_once, &one, sizeof(int)) == cudaSuccess ? 0 : -6;
}
#endif

namespace rq {
namespace {

constexpr int kTile = 64;   // tokens of one thread-map pass: 4 consumer warps x 16
#ifndef RQ_DECODE_ITEM_TILES
#define RQ_DECODE_ITEM_TILES 2
#endif
constexpr int kItemTiles = RQ_DECODE_ITEM_TILES;   // tiles per ring item
constexpr int kItem = kTile * kItemTiles;          // tokens per ring item
#ifndef RQ_DECODE_PAIR_VOTE
#define RQ_DECODE_PAIR_VOTE 1
#endif
#ifndef RQ_DECODE_PRODUCER_SLEEP_NS
#define RQ_DECODE_PRODUCER_SLEEP_NS 0
#endif
#ifndef RQ_DECODE_RING_BYTES
#define RQ_DECODE_RING_BYTES 39936
#endif
#ifndef RQ_DECODE_MIN_CTAS
#define RQ_DECODE_MIN_CTAS 4
#endif
constexpr int kRingBytes = RQ_DECODE_RING_BYTES;   // byte ring of one CTA (multiple of 128)
constexpr int kSlots = 16;                         // mbarrier pairs: at most 16 items in flight
static_assert(kRingBytes % 128 == 0, "ring must be a multiple of 128 bytes");
constexpr int kConsumers = 128;
constexpr int kThreads = kConsumers + 32;
constexpr float kRsqrt128 = 0.088388347648318440f;
constexpr int kWeightTop = 22;                          // V weight bound in [2^21, 2^22) (fixed point)
#ifndef RQ_DECODE_PDL
#define RQ_DECODE_PDL 1
#endif

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
// Grid-dependency control (programmatic dependent launch): wait for the
// previous kernel on the stream to complete (its writes visible), then allow
// the next one to start.  Both are no-ops without a programmatic launch.
__device__ __forceinline__ void griddep_wait_then_release() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }

struct ConsumerSync {
    __device__ __forceinline__ void operator()() const { consumer_sync(); }
};

// ---------------------------------------------------------------- codes
// A 16-element segment: BITS=4 -> 2 words (elements 0-7, 8-15), BITS=2 -> 1 word.
template <int BITS>
struct Seg {
    uint32_t w[BITS / 2];
};

template <int BITS>
__device__ __forceinline__ Seg<BITS> lds_seg(const uint8_t *p) {
    Seg<BITS> s;
    if (BITS == 4) {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        s.w[0] = v.x;
        s.w[BITS / 2 - 1] = v.y;
    } else {
        s.w[0] = *reinterpret_cast<const uint32_t *>(p);
    }
    return s;
}

// Unpacked code word r of a segment holds four codes, one per byte;
// elem_of<BITS>(r, m) is the segment element in byte m of word r.
//   BITS=4: r = 2u + hi: nibbles of word u; bytes = elements 8u + hi + {0,2,4,6}
//   BITS=2: r = c: (w >> 2c) & 0x03030303; bytes = elements c + {0,4,8,12}
template <int BITS>
__device__ __forceinline__ int elem_of(int r, int m) {
    return BITS == 4 ? 8 * (r >> 1) + (r & 1) + 2 * m : r + 4 * m;
}

// Inverse of elem_of: the (word, byte) slot 4r + m of segment element i.
template <int BITS>
__device__ __forceinline__ int slot_of(int i) {
    return BITS == 4 ? 4 * (2 * (i >> 3) + (i & 1)) + ((i & 7) >> 1) : 4 * (i & 3) + (i >> 2);
}

template <int BITS>
__device__ __forceinline__ uint32_t unpack_word(const Seg<BITS> &s, int r) {
    if (BITS == 4) return (r & 1) ? ((s.w[r >> 1] >> 4) & 0x0F0F0F0Fu) : (s.w[r >> 1] & 0x0F0F0F0Fu);
    return (s.w[0] >> (2 * r)) & 0x03030303u;
}

// q of one segment in 24-bit fixed point as three byte planes laid out like
// the unpacked code words: planes 0 and 1 unsigned, plane 2 signed.
struct QPlanes {
    uint32_t p[3][4];
};

// sum_i q_i c_i of one segment, exact in int32 (|q| < 2^22).
template <int BITS>
__device__ __forceinline__ int dot_seg(const Seg<BITS> &s, const QPlanes &q) {
    unsigned lo = 0, mid = 0;
    int hi = 0;
#pragma unroll
    for (int r = 0; r < 4; r++) {
        const uint32_t c = unpack_word<BITS>(s, r);
        lo = __dp4a(q.p[0][r], c, lo);
        mid = __dp4a(q.p[1][r], c, mid);
        hi = __dp4a((int)q.p[2][r], (int)c, hi);
    }
    return (int)(((unsigned)hi << 16) + (mid << 8) + lo);
}

// dp2a with signed 16-bit halves of a and UNSIGNED bytes of b (the masked
// codes reach 240, beyond int8).
__device__ __forceinline__ int dp2a_lo_su(int a, uint32_t b, int c) {
    int d;
    asm("dp2a.lo.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ int dp2a_hi_su(int a, uint32_t b, int c) {
    int d;
    asm("dp2a.hi.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

template <int BITS>
__host__ __device__ constexpr int acc_shift(int e) {
    return BITS == 4 ? ((e & 1) ? 4 : 0) : 2 * (e & 3);
}

// The code words of one segment for a pair of tokens, masked in place:
// word i feeds the dp2a of elements pair_elem(i) (low half of the word) and
// pair_elem(i) + pair_step (high half), codes of both tokens side by side.
template <int BITS>
struct PairCodes {
    uint32_t c[8];
};
template <int BITS>
__host__ __device__ constexpr int pair_elem(int i) {
    return BITS == 4 ? 8 * (i >> 2) + ((i & 3) < 2 ? (i & 3) : (i & 3) + 2) : (i < 4 ? i : i + 4);
}
template <int BITS>
__host__ __device__ constexpr int pair_step() {
    return BITS == 4 ? 2 : 4;
}

template <int BITS>
__device__ __forceinline__ PairCodes<BITS> pair_codes(const Seg<BITS> &a, const Seg<BITS> &b) {
    PairCodes<BITS> p;
    if (BITS == 4) {
#pragma unroll
        for (int u = 0; u < 2; u++) {
            const uint32_t X = __byte_perm(a.w[u], b.w[u], 0x5140);   // bytes 0,1 of both tokens
            const uint32_t Y = __byte_perm(a.w[u], b.w[u], 0x7362);   // bytes 2,3 of both tokens
            p.c[4 * u + 0] = X & 0x0F0F0F0Fu;   // elements 8u+0, 8u+2
            p.c[4 * u + 1] = X & 0xF0F0F0F0u;   // elements 8u+1, 8u+3 (x16)
            p.c[4 * u + 2] = Y & 0x0F0F0F0Fu;   // elements 8u+4, 8u+6
            p.c[4 * u + 3] = Y & 0xF0F0F0F0u;   // elements 8u+5, 8u+7 (x16)
        }
    } else {
        const uint32_t X = __byte_perm(a.w[0], b.w[0], 0x5140);   // bytes 0,1: elements 0-7
        const uint32_t Y = __byte_perm(a.w[0], b.w[0], 0x7362);   // bytes 2,3: elements 8-15
#pragma unroll
        for (int c = 0; c < 4; c++) {
            p.c[c] = X & (0x03030303u << (2 * c));       // elements c, 4+c (x4^c)
            p.c[4 + c] = Y & (0x03030303u << (2 * c));   // elements 8+c, 12+c (x4^c)
        }
    }
    return p;
}

// accLo[i] += 2^acc_shift(i) (w0 * c0_i + w1 * c1_i) with the low 16-bit
// halves wlo = (w0 & 0xFFFF) | (w1 << 16); acc_hi the same with the signed
// high halves whi = (w0 >> 16) | (w1 >> 16) << 16.  Codes are masked in
// place rather than shifted down, so element i's sums carry the factor
// 2^acc_shift(i), removed once at the end (the sums stay below 2^30 for the
// 64 tokens a lane takes per chunk).
template <int BITS>
__device__ __forceinline__ void acc_lo(const PairCodes<BITS> &p, uint32_t wlo, unsigned accLo[16]) {
#pragma unroll
    for (int i = 0; i < 8; i++) {
        constexpr int s = pair_step<BITS>();
        const int e = pair_elem<BITS>(i);
        accLo[e] = __dp2a_lo(wlo, p.c[i], accLo[e]);
        accLo[e + s] = __dp2a_hi(wlo, p.c[i], accLo[e + s]);
    }
}
template <int BITS>
__device__ __forceinline__ void acc_hi(const PairCodes<BITS> &p, uint32_t whi, int accHi[16]) {
#pragma unroll
    for (int i = 0; i < 8; i++) {
        constexpr int s = pair_step<BITS>();
        const int e = pair_elem<BITS>(i);
        accHi[e] = dp2a_lo_su((int)whi, p.c[i], accHi[e]);
        accHi[e + s] = dp2a_hi_su((int)whi, p.c[i], accHi[e + s]);
    }
}

// (scale, min) of an FP8 pair stored little-endian as scale | min << 8.
__device__ __forceinline__ float2 meta_pair(uint32_t m16) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)m16, __NV_E4M3);
    return __half22float2(__half2(h));
}

// power-of-two scale 2^F putting a positive bound into [2^(top-1), 2^top)
__device__ __forceinline__ float fixed_scale(float bound, int top) {
    if (!(bound > 0.f)) return 1.f;
    int e;
    frexpf(bound, &e);                       // bound = m 2^e, m in [0.5, 1)
    const int F = max(-100, min(100, top - e));
    return ldexpf(1.f, F);
}

// Shared-memory plan of one CTA (bytes).  Items are kItem tokens; they are placed
// back to back in a byte ring (an item never straddles its end), so the
// number in flight follows their size: about 4 K items, 7 anchor V items or
// 12 residual V items at once.
template <int BA, int BR, int GS, int NR>
struct Plan {
    static constexpr bool RESID = NR > 0;
    static constexpr int A_C = 16 * BA;              // anchor codes per record
    static constexpr int R_C = 16 * BR;              // residual codes per record
    static constexpr int MR = 2 * (kHeadDim / GS);   // meta bytes per record
    // K item: anchor codes | anchor meta | then per residual record k of the
    // chain: codes | meta | coefficients
    static constexpr int K_AM = kItem * A_C;
    static constexpr int K_R0 = K_AM + kItem * MR;
    static constexpr int K_RS = kItem * (R_C + MR + 2);
    __host__ __device__ static constexpr int K_RC(int k) { return K_R0 + k * K_RS; }
    __host__ __device__ static constexpr int K_RM(int k) { return K_RC(k) + kItem * R_C; }
    __host__ __device__ static constexpr int K_CF(int k) { return K_RM(k) + kItem * MR; }
    static constexpr int K_BYTES = K_R0 + NR * K_RS;
    // V items: codes | meta, anchor items then residual items
    static constexpr int VA_M = kItem * A_C;
    static constexpr int VA_BYTES = VA_M + kItem * MR;
    static constexpr int VR_M = kItem * R_C;
    static constexpr int VR_BYTES = VR_M + kItem * MR;
    // at least two K items in flight
    static constexpr int RING = 2 * K_BYTES > kRingBytes ? 2 * K_BYTES : kRingBytes;
    static_assert(K_BYTES % 128 == 0 && VA_BYTES % 128 == 0 && VR_BYTES % 128 == 0, "item alignment");
    static_assert(K_BYTES <= RING && VA_BYTES <= RING, "ring too small");
    // pass 0: K items; pass 1: anchor V items; pass 2 + k: residual V items of record k
    __host__ __device__ static constexpr int item_bytes(int pass) {
        return pass == 0 ? K_BYTES : pass == 1 ? VA_BYTES : VR_BYTES;
    }
    // ring offset of the item after one of `cur` bytes at offset `off`, when the next has `next` bytes
    __host__ __device__ static int advance(int off, int cur, int next) {
        off += cur;
        return off + next > RING ? 0 : off;
    }
    // then: V coefficients [NR][chunk], logits -> residual weights of the last
    // record [GK][chunk], anchor weights [GK][chunk], residual weights of the
    // other records [NR - 1][GK][chunk]
    __host__ __device__ static int coef_bytes(int chunk) { return RESID ? (chunk * 2 + 127) / 128 * 128 : 0; }
    __host__ __device__ static size_t smem(int GK, int chunk) {
        return (size_t)RING + (size_t)NR * coef_bytes(chunk) +
               (size_t)(1 + (NR > 1 ? NR : 1)) * GK * chunk * sizeof(float);
    }
};

// NR: residual records the loop's reconstruction reads (0 for the anchor's
// own loop, 1 for the shared reference, 1..3 along a chained reference).
// PG: records in a pool of blocks behind a block table (a.pg.table set); the
// contiguous instantiation carries none of the block arithmetic.
template <int GK, int BA, int BR, int GS, int NR, bool PG>
__global__ void __launch_bounds__(kThreads, GK == 1 ? RQ_DECODE_MIN_CTAS : 3) decode_rq_kernel(const DecodeArgs a) {
    using P = Plan<BA, BR, GS, NR>;
    constexpr bool RESID = NR > 0;
    constexpr int NW = NR > 1 ? NR : 1;   // residual weight arrays
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bar_full[kSlots];
    __shared__ __align__(8) uint64_t bar_empty[kSlots];
    __shared__ __align__(8) uint64_t bar_cf;
    __shared__ __align__(8) uint64_t bar_cfmax;   // the chunk's max |s_hat(V)| is known
    __shared__ int s_abort, s_last;
    __shared__ int s_blk[PG ? kMaxChunk / kTokTile + 1 : 1];   // paged: physical blocks of the chunk
    __shared__ unsigned s_cfmax[NW];
    __shared__ float s_q[GK][2][kHeadDim];
    __shared__ __align__(16) uint8_t s_qp[GK][2][3][kHeadDim];   // q byte planes, [plane][segment][word][byte]
    __shared__ int s_qsum[GK][2][8];                             // sum of each segment's fixed-point q
    __shared__ float s_red[4][2 * GK + 2];
    __shared__ __align__(16) float s_acc[4][GK][2][kHeadDim];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, h = blockIdx.y;
    const int npairs = a.G / GK;
    const int b = blockIdx.z / npairs, pair = blockIdx.z % npairs;
    const int hq0 = h * a.G + pair * GK;
    int t0, n;   // this split's tokens of its sequence (none when the sequence is short)
    split_range(split, a.S, a.seqT.v[b], &t0, &n);
    const int ntiles = (n + kTile - 1) / kTile;
    // paged: ring items start on item-size boundaries of the sequence (a
    // split may begin inside one), so that no item straddles two blocks; the
    // item grid then begins sh tiles before the split, which stay empty
    const int sh = (PG && ntiles > 0) ? (t0 / kTile) % kItemTiles : 0;
    const int ntv = ntiles + sh;   // tiles of the item grid
    const size_t bh = (size_t)b * a.H + h;
    uint8_t *ring = smem;
    const uint16_t *s_cf = reinterpret_cast<const uint16_t *>(smem + P::RING);   // V coefficients [NR][cstride]
    const int cstride = P::coef_bytes(a.chunk) / 2;
    float *s_sc = reinterpret_cast<float *>(smem + P::RING + NR * P::coef_bytes(a.chunk));  // logits -> weights
    float *s_P = s_sc + GK * a.chunk;                        // [GK][chunk] anchor weights
    // residual weights of record k: s_sc for the last one, s_P + (k + 1) * GK * chunk for the others
    auto s_W = [&](int k) { return k == NR - 1 ? s_sc : s_P + (size_t)(k + 1) * GK * a.chunk; };

    if (tid == 0) {
        for (int i = 0; i < kSlots; i++) {
            mbar_init(&bar_full[i], 1);
            mbar_init(&bar_empty[i], kConsumers);   // every consumer thread arrives
        }
        mbar_init(&bar_cf, 1);
        mbar_init(&bar_cfmax, 31);
        s_abort = 0;
        for (int k = 0; k < NW; k++) s_cfmax[k] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // ------------------------------------------------------------ producer
    if (warp == 4) {
        // paged records: the chunk's physical blocks, read once into shared
        // memory (through L2).  Before the grid dependency wait only when the
        // whole chunk lies below a.stable: the host sets a.stable to 0 when a
        // block-table change may be in flight, so such rows are settled.
        constexpr bool paged = PG;
        const bool early = paged && t0 + ntiles * kTile <= a.stable;
        const int blk0 = t0 >> a.pg.shift;
        if (paged) {
            if (!early) griddep_wait_then_release();
            const int nblk = ntiles > 0 ? ((t0 + ntiles * kTile - 1) >> a.pg.shift) - blk0 + 1 : 0;
            if (lane < nblk) s_blk[lane] = __ldcg(a.pg.table + (size_t)b * a.pg.mb + blk0 + lane);
            __syncwarp();
        }
        if (lane == 0) {
            // record row of token t of this (sequence, head)
            auto row_of = [&](int t) -> size_t {
                if (!paged) return bh * a.pg.bt + (size_t)t;
                return (((size_t)s_blk[(t >> a.pg.shift) - blk0] * a.H + h) << a.pg.shift) +
                       (size_t)(t & (a.pg.bt - 1));
            };
            // bulk copies of tokens [t, t + cnt) of an array with rec bytes per
            // record, one per block the run touches
            auto copy_rows = [&](uint8_t *dst, const void *base, int rec, int t, int cnt, uint64_t *bar) {
                const uint8_t *src = static_cast<const uint8_t *>(base);
                while (cnt > 0) {
                    const int c = paged ? min(cnt, a.pg.bt - (t & (a.pg.bt - 1))) : cnt;
                    bulk_g2s(dst, src + row_of(t) * rec, (uint32_t)(c * rec), bar);
                    dst += c * rec;
                    t += c;
                    cnt -= c;
                }
            };
            // records of tokens [.., tok_end) may be read before the grid
            // dependency wait only if all of them lie below a.stable (padding
            // beyond the sequence's length is read but never used)
            bool waited = paged && !early;
            auto dep = [&](int tok_end) {
                if (!waited && t0 + tok_end > a.stable) {
                    griddep_wait_then_release();
                    waited = true;
                }
            };
            dep(RESID && ntiles > 0 ? n : 0);
            if (RESID && ntiles > 0) {
                mbar_expect_tx(&bar_cf, (uint32_t)(NR * ntiles * kTile * 2));
#pragma unroll
                for (int k = 0; k < NR; k++)
                    copy_rows(smem + P::RING + k * P::coef_bytes(a.chunk), a.r_coef[k][1], 2, t0, ntiles * kTile,
                             &bar_cf);
            } else if (RESID) {
                mbar_arrive(&bar_cf);   // nothing to fetch
            }
            // Items in order: K items, anchor V items, residual V items.  Item it
            // occupies [virt, virt + bytes) of an unbounded virtual byte
            // sequence, padded so that no item straddles the ring's end; its
            // ring offset is phys = virt mod RING.  Before it is issued, every
            // older item starting below virt + bytes - RING must have been
            // released, and at most kSlots items may be outstanding.  The
            // loop keeps all of this in running counters (no division).
            const int npass = 2 + NR;
            int it = 0, virt = 0, phys = 0;
            const int nitems = (ntv + kItemTiles - 1) / kItemTiles;   // items per pass
            int rel = 0, vrel = 0, rphys = 0, ritem = 0, rpass = 0, rbytes = P::K_BYTES;   // oldest unreleased item
            bool ok = true;
            for (int pass = 0; pass < npass && ok; pass++) {
                const int bytes = P::item_bytes(pass);
                for (int j = 0; j < nitems; j++, it++) {
                    if (phys + bytes > P::RING) {
                        virt += P::RING - phys;
                        phys = 0;
                    }
                    if (rel < it && (it - rel >= kSlots || vrel < virt + bytes - P::RING))
                        dep(0x7FFFFFFF);   // about to block on the consumers, who run after their wait
                    dep(min((j + 1) * kItem - sh * kTile, n));
                    while (rel < it && (it - rel >= kSlots || vrel < virt + bytes - P::RING)) {
                        if (!mbar_wait<RQ_DECODE_PRODUCER_SLEEP_NS>(&bar_empty[rel % kSlots], (rel / kSlots) & 1,
                                                                    &s_abort)) {
                            ok = false;
                            break;
                        }
                        vrel += rbytes;
                        rphys += rbytes;
                        if (++ritem == nitems) {
                            ritem = 0;
                            rbytes = P::item_bytes(++rpass);
                        }
                        if (rphys + rbytes > P::RING) {
                            vrel += P::RING - rphys;
                            rphys = 0;
                        }
                        rel++;
                    }
                    if (!ok) {
                        s_abort = 1;
                        atomicExch(a.err, 1);
                        break;
                    }
                    // the first and the last item of a pass may hold fewer tiles:
                    // copy only those, to their places in the item
                    const int v0 = max(j * kItemTiles, sh), v1 = min((j + 1) * kItemTiles, ntv);
                    const int toks = (v1 - v0) * kTile;
                    const int tj = t0 + (v0 - sh) * kTile;
                    const int skip = (v0 - j * kItemTiles) * kTile;   // empty token slots before them
                    uint8_t *st = ring + phys;
                    uint64_t *bar = &bar_full[it % kSlots];
#ifdef RQ_FAULT_INJECT
                    if (it == 1 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 &&
                        atomicExch(&g_rq_fault_once, 0) == 1) {
                        virt += bytes;   // the item keeps its place in the ring, unarmed
                        phys += bytes;
                        continue;
                    }
#endif
                    // paged: one run per stream, at a row found once per item (an
                    // item lies inside one block: items follow the 128-token grid,
                    // blocks hold 128 or 256 tokens)
                    const size_t prow = PG ? row_of(tj) : 0;
                    auto copy_run = [&](uint8_t *dst, const void *base, int rec, int t, int cnt, uint64_t *bar) {
                        if (PG) {
                            bulk_g2s(dst, static_cast<const uint8_t *>(base) + prow * rec, (uint32_t)(cnt * rec), bar);
                        } else {
                            copy_rows(dst, base, rec, t, cnt, bar);
                        }
                    };
                    if (pass == 0) {
                        mbar_expect_tx(bar, (uint32_t)(toks * (P::A_C + P::MR + NR * (P::R_C + P::MR + 2))));
                        copy_run(st + skip * P::A_C, a.a_codes[0], P::A_C, tj, toks, bar);
                        copy_run(st + P::K_AM + skip * P::MR, a.a_meta[0], P::MR, tj, toks, bar);
#pragma unroll
                        for (int k = 0; k < NR; k++) {
                            copy_run(st + P::K_RC(k) + skip * P::R_C, a.r_codes[k][0], P::R_C, tj, toks, bar);
                            copy_run(st + P::K_RM(k) + skip * P::MR, a.r_meta[k][0], P::MR, tj, toks, bar);
                            copy_run(st + P::K_CF(k) + skip * 2, a.r_coef[k][0], 2, tj, toks, bar);
                        }
                    } else if (pass == 1) {
                        mbar_expect_tx(bar, (uint32_t)(toks * (P::A_C + P::MR)));
                        copy_run(st + skip * P::A_C, a.a_codes[1], P::A_C, tj, toks, bar);
                        copy_run(st + P::VA_M + skip * P::MR, a.a_meta[1], P::MR, tj, toks, bar);
                    } else {
                        mbar_expect_tx(bar, (uint32_t)(toks * (P::R_C + P::MR)));
                        copy_run(st + skip * P::R_C, a.r_codes[pass - 2][1], P::R_C, tj, toks, bar);
                        copy_run(st + P::VR_M + skip * P::MR, a.r_meta[pass - 2][1], P::MR, tj, toks, bar);
                    }
                    virt += bytes;
                    phys += bytes;
                }
            }
            dep(0x7FFFFFFF);
            const int issued = it;
            // drain: every issued copy must have landed before the CTA exits
            // (the consumers stop waiting once the CTA has given up)
            if (RESID) mbar_wait<256>(&bar_cf, 0, &s_abort);
            for (int it = max(0, issued - kSlots); it < issued; it++)
                mbar_wait<256>(&bar_full[it % kSlots], (it / kSlots) & 1, &s_abort);
        } else {
            // the other lanes: the bound max |s_hat(V)| of the chunk's V
            // coefficients (for the weights' fixed point), ready before the
            // softmax needs it
            griddep_wait_then_release();
            if (RESID && mbar_wait<64>(&bar_cf, 0, &s_abort)) {
#pragma unroll
                for (int k = 0; k < NR; k++) {
                    const uint16_t *cf = reinterpret_cast<const uint16_t *>(smem + P::RING + k * P::coef_bytes(a.chunk));
                    unsigned m = 0;
                    for (int t = lane - 1; t < n; t += 31) m = max(m, (unsigned)cf[t] & 0x7FFFu);
                    atomicMax(&s_cfmax[k], m);
                }
            }
            mbar_arrive(&bar_cfmax);
        }
        return;
    }

    // ------------------------------------------------------------ consumers
    griddep_wait_then_release();
    // upper bounds of this stream's V scales (anchor; the loop's residual)
    const float vA = e4m3_to_f32((uint32_t)a.vmax_a[bh]);
    float vR[NW];
#pragma unroll
    for (int k = 0; k < NW; k++) vR[k] = RESID ? e4m3_to_f32((uint32_t)a.vmax_r[k][bh]) : 0.f;
    if (a.n_new > 0 && split == 0) {
        // fused append: this unit's new tail rows (K and V, 16-byte vectors);
        // the fence before the arrival count below publishes them to the
        // CTA that combines
        const int nvec = a.n_new * 2 * (kHeadDim / 8);
        for (int i = tid; i < nvec; i += kConsumers) {
            const int vec = i % (kHeadDim / 8), r = i / (kHeadDim / 8), kv = r & 1, t = r >> 1;
            const uint4 *src = reinterpret_cast<const uint4 *>((kv ? a.new_v : a.new_k) +
                                                               (((size_t)b * a.n_new + t) * a.H + h) * kHeadDim);
            uint4 *dst = reinterpret_cast<uint4 *>((kv ? a.tail_v_w : a.tail_k_w) +
                                                   (((size_t)b * a.tail_cap + a.tail_pos + t) * a.H + h) * kHeadDim);
            dst[vec] = src[vec];
        }
    }
    const int sub = lane >> 3, seg = lane & 7;
    const int mg = (seg * 16) / GS;   // quantization group of this lane's segment

    // q (log2-domain scale folded in) and R q, then 24-bit fixed-point planes
    for (int gq = 0; gq < GK; gq++)
        s_q[gq][0][tid] = bf16_to_f32(a.q[((size_t)b * a.Hq + hq0 + gq) * kHeadDim + tid]) * a.scale_log2;
    consumer_sync();
    if (RESID && warp < GK) {
        const int gq = warp;
        float v[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            v[k] = s_q[gq][0][4 * lane + k];
            if (a.rotate && sigma_neg(a.sigma, 4 * lane + k)) v[k] = -v[k];
        }
        if (a.rotate) {
            wht128_warp<float>(v, lane);
#pragma unroll
            for (int k = 0; k < 4; k++) v[k] *= kRsqrt128;
        }
#pragma unroll
        for (int k = 0; k < 4; k++) s_q[gq][1][4 * lane + k] = v[k];
    }
    consumer_sync();
    {
        float mx = 0.f;
        for (int gq = 0; gq < GK; gq++) {
            mx = fmaxf(mx, fabsf(s_q[gq][0][tid]));
            if (RESID) mx = fmaxf(mx, fabsf(s_q[gq][1][tid]));
        }
        for (int m = 16; m >= 1; m >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, m));
        if (lane == 0) s_red[warp][0] = mx;
    }
    consumer_sync();
    const float qmax = fmaxf(fmaxf(s_red[0][0], s_red[1][0]), fmaxf(s_red[2][0], s_red[3][0]));
    const float qscale = fixed_scale(qmax, 22);  // q_int = round(q * qscale), |q_int| < 2^22
    const float qinv = 1.f / qscale;             // exact (power of two)
    // Each consumer thread converts element tid of q (and of R q) and stores
    // its three bytes where the lanes of its segment pick them up as plane
    // words; the integer sum of each segment's 16 values comes from a
    // 16-lane shuffle reduction.
    {
        const int sg = tid >> 4, i = tid & 15;
#pragma unroll
        for (int gq = 0; gq < GK; gq++) {
#pragma unroll
            for (int ab = 0; ab < (RESID ? 2 : 1); ab++) {
                const int x = __float2int_rn(s_q[gq][ab][tid] * qscale);
                uint8_t *dst = &s_qp[gq][ab][0][sg * 16 + (ab == 0 ? slot_of<BA>(i) : slot_of<BR>(i))];
                dst[0] = (uint8_t)(x & 0xFF);
                dst[kHeadDim] = (uint8_t)((x >> 8) & 0xFF);
                dst[2 * kHeadDim] = (uint8_t)((x >> 16) & 0xFF);
                int sum = x;
#pragma unroll
                for (int m = 1; m < 16; m <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, m);
                if (i == 0) s_qsum[gq][ab][sg] = sum;
            }
        }
    }
    consumer_sync();
    QPlanes qA[GK], qR[GK];
    float QA[GK], QR[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
#pragma unroll
        for (int pl = 0; pl < 3; pl++) {
            const uint4 wa = *reinterpret_cast<const uint4 *>(&s_qp[gq][0][pl][seg * 16]);
            qA[gq].p[pl][0] = wa.x;
            qA[gq].p[pl][1] = wa.y;
            qA[gq].p[pl][2] = wa.z;
            qA[gq].p[pl][3] = wa.w;
            if (RESID) {
                const uint4 wr = *reinterpret_cast<const uint4 *>(&s_qp[gq][1][pl][seg * 16]);
                qR[gq].p[pl][0] = wr.x;
                qR[gq].p[pl][1] = wr.y;
                qR[gq].p[pl][2] = wr.z;
                qR[gq].p[pl][3] = wr.w;
            }
        }
        QA[gq] = (float)s_qsum[gq][0][seg];
        QR[gq] = RESID ? (float)s_qsum[gq][1][seg] : 0.f;
    }

    // ------------------------------------------------------------ pass 1: logits
    float mloc[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) mloc[gq] = -CUDART_INF_F;
    const bool b4 = (seg & 4) != 0, b2 = (seg & 2) != 0;
    const int kown = (b4 ? 2 : 0) + (b2 ? 1 : 0);   // token (of 4) this lane ends up owning
    const int nitems = (ntv + kItemTiles - 1) / kItemTiles;   // ring items per pass
    int c_off = 0;   // ring offset of the current item (the producer's placement rule)
    for (int j = 0; j < nitems; j++) {
        const int slot = j % kSlots;
        const bool ok = mbar_wait(&bar_full[slot], (j / kSlots) & 1, &s_abort);
        if (!ok) {
            s_abort = 1;
            atomicExch(a.err, 2);
        }
        const uint8_t *st = ring + c_off;
        float part[kItemTiles][GK][4];
#pragma unroll
        for (int u = 0; u < kItemTiles; u++) {
            if (j * kItemTiles + u >= ntv) break;   // uniform: a short last item
            if (PG && j * kItemTiles + u < sh) continue;   // uniform: an empty first tile
#pragma unroll
            for (int k = 0; k < 4; k++) {
                const int tok = u * kTile + 16 * warp + sub + 4 * k;   // token within the item
                const Seg<BA> ca = lds_seg<BA>(st + tok * P::A_C + seg * (2 * BA));
                const float2 ma =
                    meta_pair(*reinterpret_cast<const uint16_t *>(st + P::K_AM + tok * P::MR + 2 * mg));
#pragma unroll
                for (int gq = 0; gq < GK; gq++)
                    part[u][gq][k] = fmaf(ma.y, QA[gq], ma.x * __int2float_rn(dot_seg<BA>(ca, qA[gq])));
                // along the chain: v <- s_hat_k v + (R q) . y_hat_k  (one step for the shared reference)
#pragma unroll
                for (int r = 0; r < NR; r++) {
                    const Seg<BR> cr = lds_seg<BR>(st + P::K_RC(r) + tok * P::R_C + seg * (2 * BR));
                    const float2 mr =
                        meta_pair(*reinterpret_cast<const uint16_t *>(st + P::K_RM(r) + tok * P::MR + 2 * mg));
                    const float shat = bf16_to_f32(*reinterpret_cast<const uint16_t *>(st + P::K_CF(r) + 2 * tok));
#pragma unroll
                    for (int gq = 0; gq < GK; gq++) {
                        const float R = fmaf(mr.y, QR[gq], mr.x * __int2float_rn(dot_seg<BR>(cr, qR[gq])));
                        part[u][gq][k] = fmaf(shat, part[u][gq][k], R);
                    }
                }
            }
        }
        mbar_arrive(&bar_empty[slot]);
        c_off = P::advance(c_off, P::K_BYTES, j + 1 < nitems ? P::K_BYTES : P::VA_BYTES);
        // reduce the 4 tokens' partials over the 8 segment lanes: lanes 2k, 2k+1 end with token k
#pragma unroll
        for (int u = 0; u < kItemTiles; u++) {
            if (j * kItemTiles + u >= ntv) break;
            if (PG && j * kItemTiles + u < sh) continue;
            const int i = j * kItemTiles + u - sh;   // tile of the chunk
            const int tl = i * kTile + 16 * warp + sub + 4 * kown;
#pragma unroll
            for (int gq = 0; gq < GK; gq++) {
                float r0 = (b4 ? part[u][gq][2] : part[u][gq][0]) +
                           __shfl_xor_sync(0xffffffffu, b4 ? part[u][gq][0] : part[u][gq][2], 4);
                float r1 = (b4 ? part[u][gq][3] : part[u][gq][1]) +
                           __shfl_xor_sync(0xffffffffu, b4 ? part[u][gq][1] : part[u][gq][3], 4);
                float r = (b2 ? r1 : r0) + __shfl_xor_sync(0xffffffffu, b2 ? r0 : r1, 2);
                r += __shfl_xor_sync(0xffffffffu, r, 1);
                r *= qinv;
                if ((seg & 1) == 0) s_sc[gq * a.chunk + tl] = r;   // tl < ntiles*64 <= chunk
                if (tl < n && ok) mloc[gq] = fmaxf(mloc[gq], r);
            }
        }
    }

    // ------------------------------------------------------------ softmax weights
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        float v = mloc[gq];
        for (int m = 16; m >= 1; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
        if (lane == 0) s_red[warp][gq] = v;
    }
    if (RESID && !mbar_wait(&bar_cf, 0, &s_abort)) {
        s_abort = 1;
        atomicExch(a.err, 3);
    }
    consumer_sync();
    float M[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++)
        M[gq] = fmaxf(fmaxf(s_red[0][gq], s_red[1][gq]), fmaxf(s_red[2][gq], s_red[3][gq]));
    // the weights' fixed-point scales: w = P * sc (anchor) or p * sc
    // (residual), |P| <= max|s_hat|, p <= 1, sc <= the stream's largest V
    // scale (powers of two)
    if (!mbar_wait(&bar_cfmax, 0, &s_abort)) {
        s_abort = 1;
        atomicExch(a.err, 3);
    }
    // record k's V weight is p times the product of the V coefficients of
    // the records after it on the chain (1 for the last), the anchor's p
    // times the product of all of them; bounds from the coefficients' maxima
    float cR[NW];
    float cfprod = 1.f;
#pragma unroll
    for (int k = NW - 1; k >= 0; k--) {
        cR[k] = fixed_scale(cfprod * vR[k], kWeightTop);
        if (RESID) cfprod *= bf16_to_f32((uint16_t)s_cfmax[k]);
    }
    const float cA = fixed_scale(cfprod * vA, kWeightTop);
    // p = exp2(z - M), zero beyond the chunk's tokens; the weights stored with their scales
    float lsum[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) lsum[gq] = 0.f;
    for (int t = tid; t < ntiles * kTile; t += kConsumers) {
        const bool valid = t < n;
#pragma unroll
        for (int gq = 0; gq < GK; gq++) {
            const float p = valid ? exp2f(s_sc[gq * a.chunk + t] - M[gq]) : 0.f;
            lsum[gq] += p;
            float pr = p;
#pragma unroll
            for (int k = NR - 1; k >= 0; k--) {
                s_W(k)[gq * a.chunk + t] = pr * cR[k];
                pr *= bf16_to_f32(s_cf[k * cstride + t]);
            }
            s_P[gq * a.chunk + t] = pr * cA;
        }
    }
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        float v = lsum[gq];
        for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
        if (lane == 0) s_red[warp][GK + gq] = v;   // beside the maxima, which are read until here
    }
    consumer_sync();
    float Lsum[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++)
        Lsum[gq] = s_red[0][GK + gq] + s_red[1][GK + gq] + s_red[2][GK + gq] + s_red[3][GK + gq];

    // ------------------------------------------------------------ pass 2: values (anchor, then residual)
    const int npass = 1 + NR;
    for (int vp = 0; vp < npass; vp++) {
        const float cW = vp == 0 ? cA : cR[vp - 1];   // the weights already carry it
        const float *wsrc = vp == 0 ? s_P : s_W(vp - 1);
        unsigned accLo[GK][16];
        int accHi[GK][16];
        float mS[GK];
#pragma unroll
        for (int gq = 0; gq < GK; gq++) {
            mS[gq] = 0.f;
#pragma unroll
            for (int e = 0; e < 16; e++) {
                accLo[gq][e] = 0u;
                accHi[gq][e] = 0;
            }
        }
        for (int j = 0; j < nitems; j++) {
            const int it = (1 + vp) * nitems + j;
            const int slot = it % kSlots;
            if (!mbar_wait(&bar_full[slot], (it / kSlots) & 1, &s_abort)) {
                s_abort = 1;
                atomicExch(a.err, 4);
            }
            const uint8_t *st = ring + c_off;
            const int last_u = min(kItemTiles, ntv - j * kItemTiles) - 1;   // a short last item
#pragma unroll
            for (int u = 0; u < kItemTiles; u++) {
                if (u > last_u) break;   // uniform
                if (PG && j * kItemTiles + u < sh) continue;   // uniform: an empty first tile
                uint32_t wlo[GK][2], whi[GK][2];
                float2 mm[4];
                float W[GK][4];
                Seg<BA> ca[4];
                Seg<BR> cr[4];
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    const int tok = u * kTile + 16 * warp + sub + 4 * k;   // token within the item
                    if (vp == 0) {
                        ca[k] = lds_seg<BA>(st + tok * P::A_C + seg * (2 * BA));
                        mm[k] = meta_pair(*reinterpret_cast<const uint16_t *>(st + P::VA_M + tok * P::MR + 2 * mg));
                    } else {
                        cr[k] = lds_seg<BR>(st + tok * P::R_C + seg * (2 * BR));
                        mm[k] = meta_pair(*reinterpret_cast<const uint16_t *>(st + P::VR_M + tok * P::MR + 2 * mg));
                    }
#pragma unroll
                    for (int gq = 0; gq < GK; gq++) W[gq][k] = wsrc[gq * a.chunk + j * kItem + tok - sh * kTile];
                }
                if (u == last_u) {   // every read of the item is done: release it
                    mbar_arrive(&bar_empty[slot]);
                    const int cur = vp == 0 ? P::VA_BYTES : P::VR_BYTES;
                    c_off = P::advance(c_off, cur, j + 1 < nitems ? cur : P::VR_BYTES);
                }
                uint32_t hi_any[2] = {0u, 0u};   // per token pair
#pragma unroll
                for (int gq = 0; gq < GK; gq++) {
                    int wi[4];
#pragma unroll
                    for (int k = 0; k < 4; k++) {
                        wi[k] = __float2int_rn(W[gq][k] * mm[k].x);   // W carries the scale 2^F
                        mS[gq] = fmaf(W[gq][k], mm[k].y, mS[gq]);
                    }
#pragma unroll
                    for (int pr = 0; pr < 2; pr++) {
                        wlo[gq][pr] = __byte_perm((uint32_t)wi[2 * pr], (uint32_t)wi[2 * pr + 1], 0x5410);
                        whi[gq][pr] = __byte_perm((uint32_t)wi[2 * pr], (uint32_t)wi[2 * pr + 1], 0x7632);
                        hi_any[pr] |= whi[gq][pr];
                    }
                }
                // small weights (most tokens of a peaked softmax) have zero high
                // halves; when no lane of the warp has one, skip their products
                bool need_hi[2];
                if (RQ_DECODE_PAIR_VOTE) {
                    need_hi[0] = __any_sync(0xffffffffu, hi_any[0] != 0);
                    need_hi[1] = __any_sync(0xffffffffu, hi_any[1] != 0);
                } else {
                    need_hi[0] = need_hi[1] = __any_sync(0xffffffffu, (hi_any[0] | hi_any[1]) != 0);
                }
#pragma unroll
                for (int pr = 0; pr < 2; pr++) {
                    if (vp == 0) {
                        const PairCodes<BA> pc = pair_codes<BA>(ca[2 * pr], ca[2 * pr + 1]);
#pragma unroll
                        for (int gq = 0; gq < GK; gq++) acc_lo<BA>(pc, wlo[gq][pr], accLo[gq]);
                        if (need_hi[pr]) {
#pragma unroll
                            for (int gq = 0; gq < GK; gq++) acc_hi<BA>(pc, whi[gq][pr], accHi[gq]);
                        }
                    } else {
                        const PairCodes<BR> pc = pair_codes<BR>(cr[2 * pr], cr[2 * pr + 1]);
#pragma unroll
                        for (int gq = 0; gq < GK; gq++) acc_lo<BR>(pc, wlo[gq][pr], accLo[gq]);
                        if (need_hi[pr]) {
#pragma unroll
                            for (int gq = 0; gq < GK; gq++) acc_hi<BR>(pc, whi[gq][pr], accHi[gq]);
                        }
                    }
                }
            }
        }
        // fixed point -> fp32 (the 2^-acc_shift and 2^-F factors and the
        // minimum term folded into one FMA), then a reduce-scatter over the
        // 4 sub-groups (lanes xor 8, xor 16): each lane ends with 4 elements
        const float iW = 1.f / cW;   // exact (power of two)
        const bool hb8 = (sub & 1) != 0, hb16 = (sub & 2) != 0;
#pragma unroll
        for (int gq = 0; gq < GK; gq++) {
            const float mSi = mS[gq] * iW;
            float v[16];
#pragma unroll
            for (int e = 0; e < 16; e++) {
                const int sh = vp == 0 ? acc_shift<BA>(e) : acc_shift<BR>(e);
                const float f = fmaf((float)accHi[gq][e], 65536.f, (float)accLo[gq][e]);
                v[e] = fmaf(f, __int_as_float((127 - sh) << 23) * iW, mSi);
            }
            float r1[8];
#pragma unroll
            for (int i = 0; i < 8; i++)
                r1[i] = (hb8 ? v[8 + i] : v[i]) + __shfl_xor_sync(0xffffffffu, hb8 ? v[i] : v[8 + i], 8);
            float4 r2;
            r2.x = (hb16 ? r1[4] : r1[0]) + __shfl_xor_sync(0xffffffffu, hb16 ? r1[0] : r1[4], 16);
            r2.y = (hb16 ? r1[5] : r1[1]) + __shfl_xor_sync(0xffffffffu, hb16 ? r1[1] : r1[5], 16);
            r2.z = (hb16 ? r1[6] : r1[2]) + __shfl_xor_sync(0xffffffffu, hb16 ? r1[2] : r1[6], 16);
            r2.w = (hb16 ? r1[7] : r1[3]) + __shfl_xor_sync(0xffffffffu, hb16 ? r1[3] : r1[7], 16);
            // residual records after the first add into the rotated basis's slot
            float4 *dst = reinterpret_cast<float4 *>(
                &s_acc[warp][gq][vp > 0 ? 1 : 0][seg * 16 + (hb8 ? 8 : 0) + (hb16 ? 4 : 0)]);
            if (vp >= 2) {
                const float4 o = *dst;
                r2.x += o.x;
                r2.y += o.y;
                r2.z += o.z;
                r2.w += o.w;
            }
            *dst = r2;
        }
    }

    // ------------------------------------------------------------ reduce over warps, write the partial
    consumer_sync();
    float oA[GK], oR[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        oA[gq] = s_acc[0][gq][0][tid] + s_acc[1][gq][0][tid] + s_acc[2][gq][0][tid] + s_acc[3][gq][0][tid];
        oR[gq] = RESID ? s_acc[0][gq][1][tid] + s_acc[1][gq][1][tid] + s_acc[2][gq][1][tid] + s_acc[3][gq][1][tid]
                       : 0.f;
    }
    if (RESID && a.rotate) {
        // o += R^T o_rot = sigma . (H o_rot) / sqrt(d)
#pragma unroll
        for (int gq = 0; gq < GK; gq++) s_q[gq][1][tid] = oR[gq];
        consumer_sync();
        if (warp < GK) {
            const int gq = warp;
            float v[4];
#pragma unroll
            for (int k = 0; k < 4; k++) v[k] = s_q[gq][1][4 * lane + k];
            wht128_warp<float>(v, lane);
#pragma unroll
            for (int k = 0; k < 4; k++) {
                float r = v[k] * kRsqrt128;
                if (sigma_neg(a.sigma, 4 * lane + k)) r = -r;
                s_q[gq][1][4 * lane + k] = r;
            }
        }
        consumer_sync();
#pragma unroll
        for (int gq = 0; gq < GK; gq++) oR[gq] = s_q[gq][1][tid];
    }
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        float *part = a.partials + (((size_t)b * a.Hq + hq0 + gq) * a.splits_max + split) * kPartialStride;
        part[tid] = oA[gq] + oR[gq];
        if (tid == 0) {
            part[kHeadDim] = M[gq];
            part[kHeadDim + 1] = Lsum[gq];
        }
    }

    // ------------------------------------------------------------ last CTA of the unit combines
    __threadfence();
    consumer_sync();
    const int unit = (b * a.H + h) * npairs + pair;
    if (tid == 0) s_last = (atomicAdd(&a.counters[unit], 1) == a.S - 1);
    consumer_sync();
    if (s_last) {
        __threadfence();
        if (tid == 0) a.counters[unit] = 0;   // ready for the next call
#pragma unroll 1
        for (int gq = 0; gq < GK; gq++) {
            const size_t row = (size_t)b * a.Hq + hq0 + gq;
            const size_t trow = ((size_t)b * a.tail_cap * a.H + h) * kHeadDim;
            combine_row(a.partials + row * a.splits_max * kPartialStride, a.S, a.q + row * kHeadDim, a.scale_log2,
                        a.tail_k ? a.tail_k + trow : nullptr, a.tail_v ? a.tail_v + trow : nullptr,
                        (size_t)a.H * kHeadDim, a.n_tail, a.out + row * kHeadDim, tid, &s_red[0][0],
                        ConsumerSync());
        }
    }
}

template <int GK, int BA, int BR, int GS, int NR, bool PG>
cudaError_t configure() {
    static bool done[kMaxDevices] = {};   // the largest dynamic shared memory any launch can ask for
    return once_per_device(done, [] {
        return cudaFuncSetAttribute(decode_rq_kernel<GK, BA, BR, GS, NR, PG>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)Plan<BA, BR, GS, NR>::smem(GK, kMaxChunk));
    });
}

template <int GK, int BA, int BR, int GS, int NR, bool PG>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t st) {
    const dim3 grid(a.S, a.H, a.B * (a.G / GK));
    cudaError_t e = configure<GK, BA, BR, GS, NR, PG>();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = dim3(kThreads);
    lc.dynamicSmemBytes = Plan<BA, BR, GS, NR>::smem(GK, a.chunk);
    lc.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = RQ_DECODE_PDL ? 1 : 0;
    e = cudaLaunchKernelEx(&lc, decode_rq_kernel<GK, BA, BR, GS, NR, PG>, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int GK, int BA, int BR, int GS, int NR, bool PG>
int occupancy_t(int chunk) {
    if (configure<GK, BA, BR, GS, NR, PG>() != cudaSuccess) return 1;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_rq_kernel<GK, BA, BR, GS, NR, PG>, kThreads,
                                                      Plan<BA, BR, GS, NR>::smem(GK, chunk)) != cudaSuccess)
        return 1;
    return n > 0 ? n : 1;
}

// Variant dispatch: one instantiation per (q heads per CTA, bits, group,
// residual records read).  Chains of two or three records (the chained
// reference) are built for the method's format, INT4 anchor / INT2 residuals.
template <int GK, int GS>
struct Dispatch {
    template <typename F>
    static auto run(int ba, int br, int nr, F f) {
        if (nr == 0) return ba == 4 ? f.template go<GK, 4, 2, GS, 0>() : f.template go<GK, 2, 2, GS, 0>();
        if (nr == 2) return f.template go<GK, 4, 2, GS, 2>();
        if (nr == 3) return f.template go<GK, 4, 2, GS, 3>();
        if (ba == 4 && br == 2) return f.template go<GK, 4, 2, GS, 1>();
        if (ba == 4 && br == 4) return f.template go<GK, 4, 4, GS, 1>();
        if (ba == 2 && br == 2) return f.template go<GK, 2, 2, GS, 1>();
        return f.template go<GK, 2, 4, GS, 1>();
    }
};

struct LaunchF {
    const DecodeArgs *a;
    cudaStream_t st;
    template <int GK, int BA, int BR, int GS, int NR>
    cudaError_t go() const {
        return a->pg.table ? launch_t<GK, BA, BR, GS, NR, true>(*a, st) : launch_t<GK, BA, BR, GS, NR, false>(*a, st);
    }
};
struct OccF {
    int chunk;
    template <int GK, int BA, int BR, int GS, int NR>
    int go() const { return occupancy_t<GK, BA, BR, GS, NR, false>(chunk); }   // same resources paged or not
};

template <typename F>
auto dispatch(int G, int g, int ba, int br, int nr, F f) {
    if (G == 1) return g == 16 ? Dispatch<1, 16>::run(ba, br, nr, f) : Dispatch<1, 32>::run(ba, br, nr, f);
    return g == 16 ? Dispatch<2, 16>::run(ba, br, nr, f) : Dispatch<2, 32>::run(ba, br, nr, f);
}

}  // namespace

bool decode_rq_supported(int ba, int br, int nr) {
    return nr >= 0 && nr <= kMaxChain && (nr <= 1 || (ba == 4 && br == 2));
}

cudaError_t launch_decode_rq(const DecodeArgs &a, int ba, int br, cudaStream_t st) {
    // G = 2, 4, 8 run as pairs of query heads per CTA
    if (!decode_rq_supported(ba, br, a.nr)) return cudaErrorInvalidValue;
    return dispatch(a.G, a.g, ba, br, a.nr, LaunchF{&a, st});
}

int decode_rq_occupancy(int G, int ba, int br, int nr, int g, int chunk) {
    if (!decode_rq_supported(ba, br, nr)) return 1;
    return dispatch(G, g, ba, br, nr, OccF{chunk});
}

}  // namespace rq
