// prefill.cu -- multi-token causal attention over the ResidualQuant cache: the
// step before decode (chunked prefill, or verifying several drafted tokens),
// which the ai4snews summary's throughput study (paragraph 4) leaves out of
// its decode timing.  Query row (i, hq) of sequence b, i < n, attends to the
// first T_b + n_tail - n + 1 + i tokens of [the group's committed tokens, the
// loop's BF16 tail tokens]: the n new tokens are the most recent ones,
// committed already at an anchor loop, in the tail at the other loops.
//
// Algebra.  A committed token's key and value are k = s a + R^T y (anchor a,
// rotated residual y, least-squares coefficient s; at an anchor loop k = a),
// and per quantization group each of a and y is sc * code + mn.  So
//   q.k   = s (q.(sc code) + sum_g mn_g Q_g) + (Rq).(sc_r code_r) + sum_g mn_rg (Rq)_g
//   sum_t p_t v_t = A + R^T Y,  A = sum_t (p_t s_t) a_t,  Y = sum_t p_t y_t
// (Q_g, (Rq)_g: sums of the group's elements).  Every product of that runs on
// the tensor cores with operands that BF16 holds exactly or nearly so:
//  - sc * code (a 4-significant-bit FP8 scale times a code below 16) and the
//    FP8 minima are exact in BF16, and so is q itself;
//  - Rq, the group sums and the probabilities p and p s are fp32 values
//    split into a BF16 high part and a BF16 low part (relative 2^-17), whose
//    two products accumulate into the same fp32 tensor-memory accumulator;
//  - the minima ride along as extra K columns of the logit products (group
//    sums of q against the minima of the keys) and as extra N rows of the
//    value products (probabilities against the minima of the values).
// R^T is applied once per CTA to the accumulated Y.  Per 32-token step and
// 64 query rows (operands with a high and a low part stacked as M = 128):
//   SA = [q | Q_g] [sc code | mn]^T                      (9 MMAs of 64x32x16)
//   SY = [Rq | (Rq)_g]_hi,lo [sc_r code_r | mn_r]^T      (9 MMAs of 128x32x16)
//   OA += (p s)_hi,lo [sc code | mn]                     (2 MMAs of 128x136x16)
//   OY += p_hi,lo [sc_r code_r | mn_r]                   (2 MMAs of 128x136x16)
// (the two row halves of SY, OA, OY are summed when they are read back)
// with logits scale_log2 (s SA + SY) and a running maximum that is only
// raised when a row's maximum grows by more than 2^8 (then that row of OA and
// OY is rescaled in tensor memory); the partial (m, l, o) of each row goes to
// global memory, and the last split of each row block to finish merges them
// (a second kernel does, with the tail tokens, only when nothing is
// committed and this kernel does not run).
//
// CTA = (split of the committed tokens, kv head, sequence x block of 64 query
// rows); 14 warps:
//  - warps 0-3: softmax -- warp w owns tensor-memory lanes 32w.. and query
//    rows 16w..16w+15 (the M=64 accumulator layout); loads the logits,
//    writes the probability operands, rescales, and at the end reads OA and
//    OY, applies R^T and writes the partial;
//  - warps 4 and 13: one thread each issues the MMAs of the anchor side
//    (SA, OA) and of the residual side (SY, OY); warp 4 allocates tensor
//    memory;
//  - warps 5-12: dequantize the step's K and V records (straight from global
//    memory; the anchor records brought into L2 two steps ahead) into the
//    swizzled operand tiles.
// Hand-offs go through mbarriers, every wait bounded (error word, abort flag):
//   kfull/vfull   dequant -> MMA       K / V operands of step j written
//   cfull[j & 3]  dequant -> softmax   coefficients of step j written
//   kdone         MMA commit           logits of step j complete (K tile free)
//   sfree         softmax -> MMA       logits of step j read (SA/SY free)
//   pfull         softmax -> MMA       probabilities of step j written
//   odone         MMA commit           values of step j complete (V and P free)
#include <math_constants.h>

#include <algorithm>

#include "combine.cuh"
#include "common.cuh"
#include "prefill.h"
#include "sync.cuh"
#include "tc.cuh"

namespace rq {
namespace {

constexpr int kRows = 64;             // query rows of a CTA (M of every MMA)
#ifndef RQ_PREFILL_PREFETCH
#define RQ_PREFILL_PREFETCH 2
#endif
constexpr int kPrefetchSteps = RQ_PREFILL_PREFETCH;   // steps of records brought into L2 ahead of their loads (0: none)
constexpr int kTok = kPrefillTile;    // committed tokens per step (N of the logits, K of the values)
constexpr int kSoftmaxWarps = 4;
constexpr int kMmaWarp = 4;            // issues the anchor-side MMAs (SA, OA); allocates tensor memory
constexpr int kMmaWarpY = 13;          // issues the residual-side MMAs (SY, OY)
constexpr int kDeqWarps = 8;
constexpr int kDeqThreads = 32 * kDeqWarps;
constexpr int kThreadsP = 32 * (kSoftmaxWarps + 2 + kDeqWarps);
static_assert(kMmaWarpY == kSoftmaxWarps + 1 + kDeqWarps, "the second MMA warp follows the dequantizing warps");
constexpr int kQBlk = kRows * 128;    // a 64-row block of 64 bf16 columns (8 KB): q
constexpr int kSBlk = 2 * kQBlk;      // a 128-row block (16 KB): stacked high / low operands (M = 128)
constexpr int kTBlk = kTok * 128;     // a block of the step's token rows (4 KB): key / value operands
static_assert(kDeqThreads == 2 * 4 * kTok, "a dequantizing thread per (K or V, record half, token)");
// Operand tiles of 3 blocks hold head_dim (blocks 0, 1) and the 16 minimum /
// group-sum columns (the first 32 bytes of each row of block 2).  Operands
// with a BF16 high and low part are stacked as the two halves of an M = 128
// operand: row 32 (r / 16) + r % 16 holds the high part of query row r, the
// row 16 after it the low part, so that both land in the tensor-memory lanes
// of the warp that owns row r.  K, V and the probabilities are
// double-buffered by step parity.
constexpr int OFF_Q = 0;                 // q (blocks 0, 1; its group sums: chunks 2, 3 of block 2 of OFF_QR)
constexpr int OFF_QR = 2 * kQBlk;        // stacked Rq hi / lo | (Rq)_g hi, lo on the high rows
constexpr int OFF_K = OFF_QR + 3 * kSBlk;   // per buffer: anchor K (sc code | mn, mn), then residual K
constexpr int kKVBytes = 6 * kTBlk;
constexpr int OFF_V = OFF_K + 2 * kKVBytes;   // per buffer: anchor V, then residual V (read MN-major)
constexpr int OFF_P = OFF_V + 2 * kKVBytes;   // per buffer: stacked (p s) hi / lo, then stacked p hi / lo
constexpr int kPBytes = 2 * kSBlk;
constexpr int kTilesBytes = OFF_P + 2 * kPBytes;
constexpr int kSmemBytes = kTilesBytes + 1024;   // + alignment of the base to 1024
// tensor-memory columns (fp32): the logits SA, SY of each step buffer, then
// the value accumulators OA, OY
constexpr uint32_t kColS = 0, kColOA = 128, kColOY = 272, kTmemCols = 512;
constexpr int kOCols = kHeadDim + 8;             // head_dim + one column per group minimum
constexpr float kRescaleLog2 = 8.f;              // raise a row's maximum only past 2^8
constexpr float kInvSqrtD = 0.08838834764831845f;   // 1 / sqrt(128)
static_assert(2 * 2 * kTok <= (int)kColOA, "two buffers of SA, SY fit before OA");

__device__ __forceinline__ uint32_t bf16_bits(float x) { return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(x)); }
__device__ __forceinline__ float bf16_val(uint32_t bits) { return __uint_as_float(bits << 16); }
// high and low BF16 parts of x, packed as the low halves of two words
__device__ __forceinline__ void split_hi_lo(float x, uint32_t &hi, uint32_t &lo) {
    hi = bf16_bits(x);
    lo = bf16_bits(x - bf16_val(hi));
}
// (x0, x1) to BF16 pairs, element 0 in the low half: one rounding each
__device__ __forceinline__ uint32_t bf16x2_rn(float x0, float x1) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(x1), "f"(x0));
    return d;
}
// high and low BF16 parts of (x0, x1) as two BF16 pairs
__device__ __forceinline__ void split_hi_lo2(float x0, float x1, uint32_t &hi, uint32_t &lo) {
    hi = bf16x2_rn(x0, x1);
    lo = bf16x2_rn(x0 - __uint_as_float(hi << 16), x1 - __uint_as_float(hi & 0xFFFF0000u));
}
// 2^x on the multi-function unit (relative error ~2^-22; 0 for x = -inf)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t fma_bf16x2(uint32_t a, uint32_t b, uint32_t c) {
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ void st_shared16(uint8_t *p, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(smem_u32(p)), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}
__device__ __forceinline__ void st_shared_u16(uint8_t *p, uint32_t x) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(smem_u32(p)), "h"((unsigned short)x) : "memory");
}
__device__ __forceinline__ void st_shared8(uint8_t *p, uint32_t x, uint32_t y) {
    asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(smem_u32(p)), "r"(x), "r"(y) : "memory");
}
// Bulk prefetch of [p, p + bytes) from global memory into L2 (p 16-byte
// aligned, bytes a multiple of 16); nothing waits for it.
__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// BF16 pair (128 + code x, 128 + code y): x in bits 0 .. BITS-1 of byte b of
// wx, y in the same bits of byte b of wy (0x4300 is 128.0 with one unit per
// code; one byte permute and one mask-and-or).
template <int BITS>
__device__ __forceinline__ uint32_t code_pair(uint32_t wx, uint32_t wy, int b) {
    constexpr uint32_t m = BITS == 4 ? 0x000F000Fu : 0x00030003u;
    return (__byte_perm(wx, wy, (uint32_t)(b | ((4 + b) << 8))) & m) | 0x43004300u;
}

// Raw bytes of half a record (head_dim elements 64 h .. 64 h + 63): its
// codes (8 BITS bytes) and the (scale, minimum) FP8 pairs of every group.
struct RawHalf {
    uint32_t w[8];
    uint32_t mw[4];
};

// Loads half `h` of a record (nothing, zeros, for a token past the step).
template <int BITS, int GS>
__device__ __forceinline__ void load_half(const uint8_t *codes, const uint8_t *meta, int h, bool ok, RawHalf &r) {
    constexpr int MR = 2 * (kHeadDim / GS);
#pragma unroll
    for (int i = 0; i < 8; i++) r.w[i] = 0u;
#pragma unroll
    for (int i = 0; i < 4; i++) r.mw[i] = 0u;
    if (!ok) return;
    const uint4 *src = reinterpret_cast<const uint4 *>(codes + 8 * BITS * h);
#pragma unroll
    for (int u = 0; u < BITS / 2; u++) {
        const uint4 v = __ldg(src + u);
        r.w[4 * u] = v.x;
        r.w[4 * u + 1] = v.y;
        r.w[4 * u + 2] = v.z;
        r.w[4 * u + 3] = v.w;
    }
    if (MR == 16) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(meta));
        r.mw[0] = v.x;
        r.mw[1] = v.y;
        r.mw[2] = v.z;
        r.mw[3] = v.w;
    } else {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(meta));
        r.mw[0] = v.x;
        r.mw[1] = v.y;
    }
}

// Writes half HALF of a loaded record into row t of a 3-block operand tile:
// sc * code per element, exact in BF16 ((128 + code) sc - 128 sc in one
// rounding); HALF 0 also writes the minimum columns (mn_0 .. mn_{NG-1},
// zeros, twice).  A token past the step (ok false) gets a zero row.
template <int BITS, int GS, int HALF, int BLK>
__device__ __forceinline__ void store_half(uint8_t *tile, int t, const RawHalf &r, bool ok) {
    constexpr int NG = kHeadDim / GS;
    uint8_t *row = tile + HALF * BLK;
    uint8_t *mrow = tile + 2 * BLK;
    if (!ok) {
#pragma unroll
        for (int c = 0; c < 8; c++) st_shared16(row + tc::sw_chunk(t, c), 0u, 0u, 0u, 0u);
        if (HALF == 0) {
            st_shared16(mrow + tc::sw_chunk(t, 0), 0u, 0u, 0u, 0u);
            st_shared16(mrow + tc::sw_chunk(t, 1), 0u, 0u, 0u, 0u);
        }
        return;
    }
    constexpr int GPH = 64 / GS;   // groups of this half
#pragma unroll
    for (int gl = 0; gl < GPH; gl++) {
        constexpr int CPG = GS / 8;   // 16-byte chunks per group
        const int gi = HALF * GPH + gl;
        const uint32_t pr = (r.mw[gi >> 1] >> (16 * (gi & 1))) & 0xFFFFu;
        const float sc = e4m3_to_f32(pr & 0xFFu);
        const uint32_t s2 = bf16_bits(sc) * 0x10001u;
        const uint32_t nb2 = bf16_bits(-128.f * sc) * 0x10001u;
#pragma unroll
        for (int cg = 0; cg < CPG; cg++) {
            const int c = gl * CPG + cg;   // chunk of the half: elements 8c .. 8c + 7
            uint32_t q[4];
            if (BITS == 4) {
                // pair k: element 8c + 2k in the low nibble of byte k of the
                // word, element 8c + 2k + 1 in its high nibble
                const uint32_t w = r.w[c];
#pragma unroll
                for (int k = 0; k < 4; k++) q[k] = code_pair<4>(w, w >> 4, k);
            } else {
                // pair k: elements 8c + 2k, 8c + 2k + 1 in bits 4(k & 1) ..
                // 4(k & 1) + 3 of byte 2(c & 1) + k / 2 of the word
                const uint32_t w = r.w[c >> 1];
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    const int b = 2 * (c & 1) + (k >> 1);
                    q[k] = (k & 1) ? code_pair<2>(w >> 4, w >> 6, b) : code_pair<2>(w, w >> 2, b);
                }
            }
            st_shared16(row + tc::sw_chunk(t, c), fma_bf16x2(q[0], s2, nb2), fma_bf16x2(q[1], s2, nb2),
                        fma_bf16x2(q[2], s2, nb2), fma_bf16x2(q[3], s2, nb2));
        }
    }
    if (HALF == 0) {
        uint32_t m[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            uint32_t lo = 0u, hi = 0u;
            if (2 * k < NG) lo = bf16_bits(e4m3_to_f32((r.mw[k] >> 8) & 0xFFu));
            if (2 * k + 1 < NG) hi = bf16_bits(e4m3_to_f32((r.mw[k] >> 24) & 0xFFu));
            m[k] = lo | (hi << 16);
        }
        st_shared16(mrow + tc::sw_chunk(t, 0), m[0], m[1], m[2], m[3]);
        st_shared16(mrow + tc::sw_chunk(t, 1), m[0], m[1], m[2], m[3]);
    }
}

// Query operands of the CTA's 64 rows (rows past nr are zero): q into OFF_Q
// and its group sums (hi, lo) into chunks 2, 3 of row r of block 2 of the
// stacked tile; for a residual loop Rq hi / lo into the stacked tile's high
// and low rows and the group sums of Rq (hi, lo) into chunks 0, 1 of the
// high row (zero on the low row).  A warp per row.
template <int GS, bool RESID>
__device__ __forceinline__ void setup_queries(const PrefillArgs &a, uint8_t *sm, int b, int h, int r0, int nr,
                                              int warp, int lane) {
    constexpr int NG = kHeadDim / GS, LPG = GS / 4;   // lanes per group
    constexpr int kWarps = kThreadsP / 32, kRowsPerWarp = (kRows + kWarps - 1) / kWarps;
    uint8_t *mblk = sm + OFF_QR + 2 * kSBlk;          // block 2 of the stacked tile
    // all of this warp's rows are fetched first, so that their latencies overlap
    uint2 raws[kRowsPerWarp];
#pragma unroll
    for (int u = 0; u < kRowsPerWarp; u++) {
        const int r = warp + u * kWarps;
        raws[u] = make_uint2(0u, 0u);
        if (r < nr) {
            const int rg = r0 + r, i = rg / a.G, gq = rg % a.G;
            const uint16_t *qrow = a.q + (((size_t)b * a.n + i) * a.Hq + h * a.G + gq) * kHeadDim;
            raws[u] = __ldg(reinterpret_cast<const uint2 *>(qrow + 4 * lane));
        }
    }
    // group sums of v (hi, lo) as elements g of chunks c0 and c0 + 1 of row `row` of block 2
    auto sums = [&](const float v[4], int row, int c0) {
        float gs = (v[0] + v[1]) + (v[2] + v[3]);
#pragma unroll
        for (int o = 1; o < LPG; o <<= 1) gs += __shfl_xor_sync(0xffffffffu, gs, o);
        if (NG < 8) {   // unused group columns are zero
            if (lane == 0) {
                st_shared16(mblk + tc::sw_chunk(row, c0), 0u, 0u, 0u, 0u);
                st_shared16(mblk + tc::sw_chunk(row, c0 + 1), 0u, 0u, 0u, 0u);
            }
            __syncwarp();
        }
        if (lane % LPG == 0) {   // the group's first lane holds its sum
            const int g = lane / LPG;
            uint32_t hi, lo;
            split_hi_lo(gs, hi, lo);
            st_shared_u16(mblk + tc::sw_chunk(row, c0) + 2 * g, hi);
            st_shared_u16(mblk + tc::sw_chunk(row, c0 + 1) + 2 * g, lo);
        }
    };
#pragma unroll
    for (int u = 0; u < kRowsPerWarp; u++) {
        const int r = warp + u * kWarps;
        if (r >= kRows) break;
        const uint2 raw = raws[u];
        float x[4];
        x[0] = bf16_val(raw.x & 0xFFFFu);
        x[1] = bf16_val(raw.x >> 16);
        x[2] = bf16_val(raw.y & 0xFFFFu);
        x[3] = bf16_val(raw.y >> 16);
        // elements 4 lane .. 4 lane + 3: block lane / 16, chunk (lane % 16) / 2, half (lane & 1)
        const int ch = (lane & 15) >> 1;
        const uint32_t in = 8u * (lane & 1);
        st_shared8(sm + OFF_Q + (lane >> 4) * kQBlk + tc::sw_chunk(r, ch) + in, raw.x, raw.y);
        sums(x, r, 2);
        if (RESID) {
            // R q = H diag(sigma) q / sqrt(d)
            float y[4];
#pragma unroll
            for (int k = 0; k < 4; k++) y[k] = (a.rotate && sigma_neg(a.sigma, 4 * lane + k)) ? -x[k] : x[k];
            if (a.rotate) {
                wht128_warp<float>(y, lane);
#pragma unroll
                for (int k = 0; k < 4; k++) y[k] *= kInvSqrtD;
            }
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int k = 0; k < 4; k++) split_hi_lo(y[k], hi[k], lo[k]);
            const int rh = 32 * (r / 16) + r % 16, rl = rh + 16;   // stacked rows
            uint8_t *blk = sm + OFF_QR + (lane >> 4) * kSBlk;
            st_shared8(blk + tc::sw_chunk(rh, ch) + in, hi[0] | hi[1] << 16, hi[2] | hi[3] << 16);
            st_shared8(blk + tc::sw_chunk(rl, ch) + in, lo[0] | lo[1] << 16, lo[2] | lo[3] << 16);
            sums(y, rh, 0);
            if (lane == 0) {
                st_shared16(mblk + tc::sw_chunk(rl, 0), 0u, 0u, 0u, 0u);
                st_shared16(mblk + tc::sw_chunk(rl, 1), 0u, 0u, 0u, 0u);
            }
        }
    }
}

// PG: records in a pool of blocks behind a block table (a.pg.table set); the
// contiguous instantiation carries none of the block arithmetic.
template <int BA, int BR, int GS, bool RESID, bool PG>
__global__ void __launch_bounds__(kThreadsP, 1) prefill_tc_kernel(const PrefillArgs a) {
    extern __shared__ uint8_t smem_raw[];
    // per step buffer b = j & 1 (k-th completion: step 2k + b); cfull per
    // coefficient slot j & 3 (k-th completion: step 4k + slot)
    __shared__ uint64_t bar_kfull[2], bar_vfull[2], bar_kdone[2], bar_sfree[2], bar_pfull[2], bar_odone[2];
    __shared__ uint64_t bar_cfull[4];
    __shared__ uint32_t s_tmem;
    __shared__ int s_abort, s_last;
    __shared__ __align__(16) float s_cK[4][kTok], s_cV[4][kTok];   // coefficients of a step (1 at an anchor loop)
    __shared__ float s_ml[kRows][2];                  // running maximum and sum of each row

    const uint32_t raw_base = smem_u32(smem_raw);
    uint8_t *sm = smem_raw + (((raw_base + 1023u) & ~1023u) - raw_base);
    const uint32_t sbase = smem_u32(sm);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, h = blockIdx.y;
    const int b = blockIdx.z / a.nqb, qb = blockIdx.z % a.nqb;
    const int r0 = qb * kRows;
    const int nr = min(kRows, a.n * a.G - r0);
    const int Tb = a.seqT.v[b];
    int t0, cnt;
    split_range(split, a.S, Tb, &t0, &cnt);
    // committed steps, then (last split of each sequence and kv head) steps
    // over the loop's BF16 tail tokens: an anchor-like step with the tokens'
    // K and V as exact BF16 operands, coefficient 1 and no residual part
    const int ntc = cnt > 0 ? (cnt + kTok - 1) / kTok : 0;
    const bool tail_here = a.tail_in_kernel && a.tail_k != nullptr && split == a.S - 1;
    const int ntl = ntc + (tail_here ? (a.n_tail + kTok - 1) / kTok : 0);
    const size_t bh = (size_t)b * a.H + h;
    constexpr int MR = 2 * (kHeadDim / GS);

    if (tid == 0) {
        for (int i = 0; i < 2; i++) {
            mbar_init(&bar_kfull[i], kDeqThreads / 2);
            mbar_init(&bar_vfull[i], kDeqThreads / 2);
            mbar_init(&bar_kdone[i], RESID ? 2 : 1);   // one commit per MMA-issuing thread
            mbar_init(&bar_sfree[i], 32 * kSoftmaxWarps);
            mbar_init(&bar_pfull[i], 32 * kSoftmaxWarps);
            mbar_init(&bar_odone[i], RESID ? 2 : 1);
        }
        for (int i = 0; i < 4; i++) mbar_init(&bar_cfull[i], kTok);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        tc::alloc(&s_tmem, kTmemCols);
        tc::relinquish();
    }
    setup_queries<GS, RESID>(a, sm, b, h, r0, nr, warp, lane);
    tc::fence_async_smem();
    tc::fence_before();
    __syncthreads();
    tc::fence_after();
    const uint32_t tmem = s_tmem;
    volatile int *abort_flag = &s_abort;
    auto wait = [&](uint64_t *bar, int parity, int code) {
        if (!mbar_wait(bar, (uint32_t)parity, abort_flag)) {
            *abort_flag = 1;
            atomicExch(a.err, code);
        }
    };
    // No barrier runs two of its phases ahead of a waiter: each next phase
    // needs work that the waiter itself releases later (the hand-offs below).

    if (warp < kSoftmaxWarps) {
        // ------------------------------------------------------- softmax
        // Thread (w, i + 16 hf) owns query row r = 16 w + i and the tokens
        // 16 hf .. 16 hf + 15 of each step.  SA (M = 64 layout: row r in
        // lane 32 w + i) is read with the 16x32bx2 access, which gives each
        // thread its own tokens; SY and the values (M = 128, stacked) hold
        // row r's high part in lane 32 w + i and its low part in lane
        // 32 w + 16 + i, i.e. thread hf = 0 reads the high, hf = 1 the low
        // part, and the pair exchanges the halves of the other's tokens.
        const int hf = lane >> 4, i16 = lane & 15;
        const int r = 16 * warp + i16;
        const int iq = (r0 + r) / a.G;
        const int lim = min(Tb, Tb + a.n_tail - a.n + 1 + iq);   // committed tokens the row may see
        const int ltail = min(a.n_tail, max(0, a.n_tail - a.n + 1 + iq));   // tail tokens it may see
        const uint32_t tl = tmem + ((uint32_t)(32 * warp) << 16);
        constexpr int kHalf = kTok / 2;                          // tokens of a thread per step
        float m_used = -CUDART_INF_F, l = 0.f;                   // l: this thread's half of the row's sum
        for (int j = 0; j < ntl; j++) {
            const int tt = j * kTok;
            const int tn = min(kTok, cnt - tt);
            const int pb = j & 1;   // step buffer
            const int cs = j & 3;   // coefficient slot
            wait(&bar_cfull[cs], (j >> 2) & 1, 21);
            wait(&bar_kdone[pb], (j >> 1) & 1, 22);
            tc::fence_after();
            // logits, and this thread's V coefficients, read before the
            // logits buffer and the coefficient slot are released
            const bool tstep = j >= ntc;   // a tail step (warp-uniform)
            float s[kHalf], cv[kHalf];
            {
                const uint32_t cS = kColS + pb * 2 * kTok;
                uint32_t sa[16];
                tc::ld16x2<kHalf>(tl + cS, sa);
                if (RESID && !tstep) {
                    uint32_t y0[16], y1[16];
                    tc::ld16(tl + cS + kTok, y0);        // this lane's part of SY, tokens 0..15
                    tc::ld16(tl + cS + kTok + 16, y1);   // tokens 16..31
                    tc::wait_ld3(sa, y0, y1);
                    float ck[kHalf];
                    const float4 *c4 = reinterpret_cast<const float4 *>(&s_cK[cs][kHalf * hf]);
#pragma unroll
                    for (int k = 0; k < kHalf; k += 4) {
                        const float4 v = c4[k / 4];
                        ck[k] = v.x;
                        ck[k + 1] = v.y;
                        ck[k + 2] = v.z;
                        ck[k + 3] = v.w;
                    }
#pragma unroll
                    for (int k = 0; k < kHalf; k++) {
                        const float own = __uint_as_float(hf ? y1[k] : y0[k]);
                        const float other = __shfl_xor_sync(0xffffffffu, __uint_as_float(hf ? y0[k] : y1[k]), 16);
                        s[k] = fmaf(ck[k], __uint_as_float(sa[k]), own + other) * a.scale_log2;
                    }
                } else {
                    tc::wait_ld(sa);
#pragma unroll
                    for (int k = 0; k < kHalf; k++) s[k] = __uint_as_float(sa[k]) * a.scale_log2;
                }
                if (RESID) {
                    const float4 *c4 = reinterpret_cast<const float4 *>(&s_cV[cs][kHalf * hf]);
#pragma unroll
                    for (int k = 0; k < kHalf; k += 4) {
                        const float4 v = c4[k / 4];
                        cv[k] = v.x;
                        cv[k + 1] = v.y;
                        cv[k + 2] = v.z;
                        cv[k + 3] = v.w;
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < kHalf; k++) cv[k] = 1.f;
                }
            }
            tc::fence_before();
            mbar_arrive(&bar_sfree[pb]);
            float mx = -CUDART_INF_F;
            if (!tstep) {
                if (tn < kTok || t0 + tt + kTok > lim) {   // the step's end is not visible to the row
#pragma unroll
                    for (int k = 0; k < kHalf; k++) {
                        const int t = kHalf * hf + k;
                        const bool ok = t < tn && t0 + tt + t < lim;
                        s[k] = ok ? s[k] : -CUDART_INF_F;
                    }
                }
            } else {
                const int jt0 = (j - ntc) * kTok;   // first tail token of the step
                if (jt0 + kTok > ltail) {
#pragma unroll
                    for (int k = 0; k < kHalf; k++) {
                        const bool ok = jt0 + kHalf * hf + k < ltail;
                        s[k] = ok ? s[k] : -CUDART_INF_F;
                    }
                }
            }
#pragma unroll
            for (int k = 0; k < kHalf; k++) mx = fmaxf(mx, s[k]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));   // the row's maximum
            const bool raise = mx > m_used + kRescaleLog2;   // false while nothing is seen (both -inf)
            const bool rescale = raise && m_used != -CUDART_INF_F;
            const float f = rescale ? exp2f(m_used - mx) : 1.f;
            if (raise) m_used = mx;
            // this step's probability buffer was last read by the values of step j - 2
            if (j >= 2) wait(&bar_odone[pb], ((j >> 1) - 1) & 1, 23);
            if (__any_sync(0xffffffffu, rescale)) {
                // O must be final: the values of step j - 1 complete
                if (j >= 1) wait(&bar_odone[pb ^ 1], ((j - 1) >> 1) & 1, 23);
                tc::fence_after();
                // this lane's part (high or low) of the row's accumulated
                // values times f (rows without a raise times 1)
#pragma unroll 1
                for (int c = 0; c < kHeadDim; c += 16) {
                    uint32_t v[16];
                    tc::ld16(tl + kColOA + c, v);
                    tc::wait_ld(v);
#pragma unroll
                    for (int k = 0; k < 16; k++) v[k] = __float_as_uint(__uint_as_float(v[k]) * f);
                    tc::st16(tl + kColOA + c, v);
                    if (RESID) {
                        tc::ld16(tl + kColOY + c, v);
                        tc::wait_ld(v);
#pragma unroll
                        for (int k = 0; k < 16; k++) v[k] = __float_as_uint(__uint_as_float(v[k]) * f);
                        tc::st16(tl + kColOY + c, v);
                    }
                }
                uint32_t v8[8];
                tc::ld8(tl + kColOA + kHeadDim, v8);
                tc::wait_ld8(v8);
#pragma unroll
                for (int k = 0; k < 8; k++) v8[k] = __float_as_uint(__uint_as_float(v8[k]) * f);
                tc::st8(tl + kColOA + kHeadDim, v8);
                if (RESID) {
                    tc::ld8(tl + kColOY + kHeadDim, v8);
                    tc::wait_ld8(v8);
#pragma unroll
                    for (int k = 0; k < 8; k++) v8[k] = __float_as_uint(__uint_as_float(v8[k]) * f);
                    tc::st8(tl + kColOY + kHeadDim, v8);
                }
                tc::wait_st();
            }
            l *= f;
            // probabilities of the step, split hi / lo, into the stacked A
            // operands (K = the step's 32 tokens: the first 64 bytes of each
            // 128-byte row)
            const float mu = m_used == -CUDART_INF_F ? 0.f : m_used;
            uint8_t *prow = sm + OFF_P + pb * kPBytes;
            const int rh = 32 * warp + i16, rl = rh + 16;
#pragma unroll
            for (int cc = 0; cc < kHalf / 8; cc++) {
                uint32_t psh[4], psl[4], ph[4], pl[4];
#pragma unroll
                for (int k = 0; k < 8; k += 2) {
                    const int u = 8 * cc + k;
                    const float p0 = ex2(s[u] - mu), p1 = ex2(s[u + 1] - mu);   // 0 if masked
                    l += p0 + p1;
                    if (RESID) {
                        split_hi_lo2(p0 * cv[u], p1 * cv[u + 1], psh[k / 2], psl[k / 2]);
                        split_hi_lo2(p0, p1, ph[k / 2], pl[k / 2]);
                    } else {
                        split_hi_lo2(p0, p1, psh[k / 2], psl[k / 2]);
                    }
                }
                const int c = (kHalf / 8) * hf + cc;
                st_shared16(prow + tc::sw_chunk(rh, c), psh[0], psh[1], psh[2], psh[3]);
                st_shared16(prow + tc::sw_chunk(rl, c), psl[0], psl[1], psl[2], psl[3]);
                if (RESID) {
                    st_shared16(prow + kSBlk + tc::sw_chunk(rh, c), ph[0], ph[1], ph[2], ph[3]);
                    st_shared16(prow + kSBlk + tc::sw_chunk(rl, c), pl[0], pl[1], pl[2], pl[3]);
                }
            }
            tc::fence_async_smem();
            tc::fence_before();
            mbar_arrive(&bar_pfull[pb]);
        }
        l += __shfl_xor_sync(0xffffffffu, l, 16);   // the row's sum
        // ------------------------------------------------------- epilogue
        // Each row's A and Y (high + low parts, plus their group minima) go
        // to shared memory (the K and V tiles are free once the last values
        // completed), with the row's running maximum and sum.
        constexpr int kEStride = kHeadDim + 4;   // padded rows: the row-per-thread stores do not conflict
        static_assert(kRows * kEStride * 4 <= 2 * kKVBytes, "staging fits in the K (and the V) tiles");
        float *sA = reinterpret_cast<float *>(sm + OFF_K);
        float *sY = reinterpret_cast<float *>(sm + OFF_V);
        if (ntl > 0) {
            // the last values complete (and with them every earlier MMA)
            wait(&bar_odone[(ntl - 1) & 1], ((ntl - 1) >> 1) & 1, 24);
            tc::fence_after();
#pragma unroll
            // OY holds something only if a committed step ran (tail steps add nothing to it)
            for (int side = 0; side < ((RESID && ntc > 0) ? 2 : 1); side++) {
                const uint32_t col = side == 0 ? kColOA : kColOY;
                float *dst = (side == 0 ? sA : sY) + r * kEStride + 8 * hf;
                // the row's group minima: high + low lane
                uint32_t m8[8];
                tc::ld8(tl + col + kHeadDim, m8);
                tc::wait_ld8(m8);
                float mn8[8];
#pragma unroll
                for (int k = 0; k < 8; k++)
                    mn8[k] = __uint_as_float(m8[k]) + __shfl_xor_sync(0xffffffffu, __uint_as_float(m8[k]), 16);
#pragma unroll
                for (int c = 0; c < kHeadDim; c += 16) {
                    uint32_t v[16];
                    tc::ld16(tl + col + c, v);
                    tc::wait_ld(v);
                    float w[16];
#pragma unroll
                    for (int k = 0; k < 16; k++)
                        w[k] = __uint_as_float(v[k]) + __shfl_xor_sync(0xffffffffu, __uint_as_float(v[k]), 16);
                    // a 16-column chunk lies in one group; thread hf stores its 8 columns
                    const float mn = mn8[c / GS];
#pragma unroll
                    for (int k = 0; k < 8; k += 4) {
                        const float a0 = hf ? w[8 + k] : w[k], a1 = hf ? w[9 + k] : w[k + 1];
                        const float a2 = hf ? w[10 + k] : w[k + 2], a3 = hf ? w[11 + k] : w[k + 3];
                        *reinterpret_cast<float4 *>(dst + c + k) = make_float4(a0 + mn, a1 + mn, a2 + mn, a3 + mn);
                    }
                }
            }
        }
        if (hf == 0) {
            s_ml[r][0] = m_used;
            s_ml[r][1] = l;
        }
    } else if (warp == kMmaWarp || warp == kMmaWarpY) {
        // ------------------------------------------------------- MMA issue
        // Two threads, in different warps (one thread issues a tcgen05.mma
        // every ~57 cycles at best; two reach the shared-memory bandwidth of
        // the operands): the anchor side (SA, OA) and the residual side (SY,
        // OY, residual loops only).  Each commits to kdone / odone, which
        // count both.  The logits of the next steps and the values of the
        // current one are issued in whichever order their operands are ready.
        const bool yside = warp == kMmaWarpY;
        if (lane == 0 && (RESID || !yside)) {
            constexpr uint32_t idA = tc::idesc_bf16(kRows, kTok, false);          // SA: q (M = 64)
            constexpr uint32_t idY = tc::idesc_bf16(2 * kRows, kTok, false);      // SY: stacked Rq (M = 128)
            constexpr uint32_t idV = tc::idesc_bf16(2 * kRows, kOCols, true);     // OA, OY: stacked p (M = 128)
            // descriptors of the operand tiles; the start address advances in
            // 16-byte units (32 bytes per K step inside a block, a block across)
            const uint64_t dQ = tc::desc_k(sbase + OFF_Q), dQm = tc::desc_k(sbase + OFF_QR + 2 * kSBlk + 32),
                           dR = tc::desc_k(sbase + OFF_QR), dK = tc::desc_k(sbase + OFF_K),
                           dP = tc::desc_k(sbase + OFF_P), dV = tc::desc_mn(sbase + OFF_V, kTBlk);
            auto kq = [](int kk) { return (uint64_t)(((kk >> 2) * kQBlk + (kk & 3) * 32) >> 4); };
            auto ks = [](int kk) { return (uint64_t)(((kk >> 2) * kSBlk + (kk & 3) * 32) >> 4); };
            auto kt = [](int kk) { return (uint64_t)(((kk >> 2) * kTBlk + (kk & 3) * 32) >> 4); };
            auto logits = [&](int j) {
                const uint64_t ka = dK + (uint64_t)(((j & 1) * kKVBytes) >> 4);
                const uint64_t ky = ka + (uint64_t)((3 * kTBlk) >> 4);
                const uint32_t cS = tmem + kColS + (j & 1) * 2 * kTok;
                if (yside && j >= ntc) {
                    // a tail step has no residual part: nothing to issue
                } else if (!yside) {
#pragma unroll
                    for (int kk = 0; kk < 8; kk++) tc::mma_bf16(cS, dQ + kq(kk), ka + kt(kk), idA, kk > 0);
                    tc::mma_bf16(cS, dQm, ka + kt(8), idA, true);   // the group sums of q against the minima
                } else {
#pragma unroll
                    for (int kk = 0; kk < 9; kk++) tc::mma_bf16(cS + kTok, dR + ks(kk), ky + kt(kk), idY, kk > 0);
                }
                tc::commit(&bar_kdone[j & 1]);
            };
            auto values = [&](int j) {
                const uint64_t pbuf = dP + (uint64_t)(((j & 1) * kPBytes + (yside ? kSBlk : 0)) >> 4);
                const uint64_t vv = dV + (uint64_t)(((j & 1) * kKVBytes + (yside ? 3 * kTBlk : 0)) >> 4);
                const uint32_t cO = tmem + (yside ? kColOY : kColOA);
                if (!(yside && j >= ntc)) {
#pragma unroll
                    for (int kk = 0; kk < kTok / 16; kk++)
                        tc::mma_bf16(cO, pbuf + (uint64_t)((kk * 32) >> 4), vv + (uint64_t)((kk * 16 * 128) >> 4),
                                     idV, j > 0 || kk > 0);
                }
                tc::commit(&bar_odone[j & 1]);
            };
            int nl = 0, nv = 0;   // steps whose logits / values are issued
            unsigned long long idle0 = 0;
            while (nv < ntl) {
                bool did = false;
                // logits of step nl: its K written, its logits buffer read by the softmax of step nl - 2
                if (nl < ntl && mbar_test(&bar_kfull[nl & 1], (nl >> 1) & 1) &&
                    (nl < 2 || mbar_test(&bar_sfree[nl & 1], ((nl >> 1) - 1) & 1))) {
                    tc::fence_after();
                    logits(nl);
                    nl++;
                    did = true;
                }
                // values of step nv: its probabilities and V written
                if (nv < nl && mbar_test(&bar_pfull[nv & 1], (nv >> 1) & 1) &&
                    mbar_test(&bar_vfull[nv & 1], (nv >> 1) & 1)) {
                    tc::fence_after();
                    values(nv);
                    nv++;
                    did = true;
                }
                if (did) {
                    idle0 = 0;
                } else if (idle0 == 0) {
                    idle0 = global_ns();
                } else if (*abort_flag || global_ns() - idle0 > kWaitNs) {
                    *abort_flag = 1;
                    atomicExch(a.err, 25);
                    break;
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------- dequantize
        // Thread (side, part, t): token t of the step, K (side 0) or V, half
        // (part & 1) of its anchor (part < 2) or residual record.  The record
        // of step j + 1 is loaded into registers while step j's is written.
        // A warp per (side, part), a lane per token; the roles are dealt so
        // that every scheduler (warp index mod 4) gets one anchor half and one
        // (costlier) residual half.
        static_assert(kTok == 32, "a lane per token of the step");
        const int dq = warp - (kSoftmaxWarps + 1);   // 0 .. 7
        const int side = dq >> 2;
        const int part = (0x31201302u >> (4 * dq)) & 0xF;   // 2, 0, 3, 1, 0, 2, 1, 3
        const int t = lane;
        // record row of the first token of committed step j (a step lies in
        // one block of a paged cache: splits start on 64-token tiles and
        // blocks hold 128 or 256 tokens)
        auto step_row = [&](int j) -> size_t {
            const int tok = t0 + j * kTok;
            if (!PG) return bh * a.Tp + (size_t)tok;
            const int blk = __ldg(a.pg.table + (size_t)b * a.pg.mb + (tok >> a.pg.shift));
            return (((size_t)blk * a.H + h) << a.pg.shift) + (size_t)(tok & (a.pg.bt - 1));
        };
        auto load = [&](int j, RawHalf &r, uint16_t *cf) {
            const bool ok = t < min(kTok, cnt - j * kTok);
            const size_t rec = step_row(j) + t;
            if (part < 2) {
                load_half<BA, GS>(ok ? a.a_codes[side] + rec * (16 * BA) : nullptr,
                                  ok ? a.a_meta[side] + rec * MR : nullptr, part, ok, r);
                if (RESID && part == 0 && side == 0) {
                    cf[0] = ok ? __ldg(a.r_coef[0] + rec) : 0;
                    cf[1] = ok ? __ldg(a.r_coef[1] + rec) : 0;
                }
            } else if (RESID) {
                load_half<BR, GS>(ok ? a.r_codes[side] + rec * (16 * BR) : nullptr,
                                  ok ? a.r_meta[side] + rec * MR : nullptr, part - 2, ok, r);
            }
        };
        // Lane 0 of the warps of part 0 brings the anchor records (codes and
        // meta) of step j + 1 + kPrefetchSteps of its side into L2 while step
        // j is written, so that the register loads of that step find them
        // there: a whole step (the padded token capacity of a sequence is a
        // multiple of 64 tokens and a block holds 128 or 256, so a full step
        // never leaves the sequence's records or its block).  The
        // residual records are not prefetched: that made residual loops
        // slower 1 or 2 steps ahead and gained nothing 3 steps ahead.
        auto prefetch = [&](int j) {
            if (kPrefetchSteps <= 0 || lane != 0 || part != 0 || j >= ntc) return;
            const size_t rec = step_row(j);
            prefetch_l2(a.a_codes[side] + rec * (16 * BA), kTok * 16 * BA);
            prefetch_l2(a.a_meta[side] + rec * MR, kTok * MR);
        };
        RawHalf raw;
        uint16_t cf[2] = {0, 0};
        if (ntc > 0) load(0, raw, cf);
        for (int i = 1; i <= kPrefetchSteps; i++) prefetch(i);
        for (int j = 0; j < ntl; j++) {
            const bool tstep = j >= ntc;
            const bool ok = !tstep && t < min(kTok, cnt - j * kTok);
            const int pb = j & 1;
            // the buffer was last read by the logits (K) / values (V) of step j - 2
            if (j >= 2) wait(side == 0 ? &bar_kdone[pb] : &bar_odone[pb], ((j >> 1) - 1) & 1, 29);
            uint8_t *ta = sm + (side == 0 ? OFF_K : OFF_V) + pb * kKVBytes;
            uint8_t *ty = ta + 3 * kTBlk;
            if (tstep) {
                // tail token jt's K or V half, BF16 as it is; minima zero
                if (part < 2) {
                    const int jt = (j - ntc) * kTok + t;
                    const bool tok = jt < a.n_tail;
                    const uint16_t *src =
                        (side == 0 ? a.tail_k : a.tail_v) + (((size_t)b * a.tail_cap + (tok ? jt : 0)) * a.H + h) * kHeadDim;
                    uint8_t *row = ta + part * kTBlk;
#pragma unroll
                    for (int c = 0; c < 8; c++) {
                        const uint4 v = tok ? __ldcg(reinterpret_cast<const uint4 *>(src + 64 * part) + c)
                                            : make_uint4(0u, 0u, 0u, 0u);
                        st_shared16(row + tc::sw_chunk(t, c), v.x, v.y, v.z, v.w);
                    }
                    if (part == 0) {
                        st_shared16(ta + 2 * kTBlk + tc::sw_chunk(t, 0), 0u, 0u, 0u, 0u);
                        st_shared16(ta + 2 * kTBlk + tc::sw_chunk(t, 1), 0u, 0u, 0u, 0u);
                    }
                }
            } else if (part == 0) store_half<BA, GS, 0, kTBlk>(ta, t, raw, ok);
            else if (part == 1) store_half<BA, GS, 1, kTBlk>(ta, t, raw, ok);
            else if (RESID) {
                if (part == 2) store_half<BR, GS, 0, kTBlk>(ty, t, raw, ok);
                else store_half<BR, GS, 1, kTBlk>(ty, t, raw, ok);
            }
            if (side == 0 && part == 0) {
                // slot j & 3 was last read by the softmax of step j - 4, before
                // it released the logits of that step, which the logits of
                // step j - 2 (hence this K buffer) waited for
                s_cK[j & 3][t] = RESID && ok ? bf16_to_f32(cf[0]) : 1.f;
                s_cV[j & 3][t] = RESID && ok ? bf16_to_f32(cf[1]) : 1.f;
                mbar_arrive(&bar_cfull[j & 3]);
            }
            tc::fence_async_smem();
            mbar_arrive(side == 0 ? &bar_kfull[pb] : &bar_vfull[pb]);
            if (j + 1 < ntc) load(j + 1, raw, cf);
            prefetch(j + 1 + kPrefetchSteps);
        }
    }

    // ------------------------------------------------------- partials
    // Every warp takes rows of the staged A and Y (warp w: rows w, w + 14,
    // ...; two rows at a time, so that their transforms overlap), applies
    // R^T to Y with the in-warp transform and writes the row's partial
    // (m, l, o), 4 consecutive elements per lane.
    tc::fence_before();
    __syncthreads();
    {
        constexpr int kEStride = kHeadDim + 4;
        const float *sA = reinterpret_cast<const float *>(sm + OFF_K);
        const float *sY = reinterpret_cast<const float *>(sm + OFF_V);
        constexpr int kWarps = kThreadsP / 32;
        for (int row0 = warp; row0 < nr; row0 += 2 * kWarps) {
            float o[2][4];
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int row = min(row0 + u * kWarps, kRows - 1);   // a row past nr is computed, not written
#pragma unroll
                for (int k = 0; k < 4; k++) o[u][k] = 0.f;
                if (ntc > 0 && RESID) {
                    const float4 y = *reinterpret_cast<const float4 *>(sY + row * kEStride + 4 * lane);
                    o[u][0] = y.x;
                    o[u][1] = y.y;
                    o[u][2] = y.z;
                    o[u][3] = y.w;
                }
            }
            if (ntc > 0 && RESID && a.rotate) {
                // R^T Y = diag(sigma) H Y / sqrt(d)
                wht128_warp2<float>(o[0], o[1], lane);
#pragma unroll
                for (int u = 0; u < 2; u++)
#pragma unroll
                    for (int k = 0; k < 4; k++) o[u][k] *= sigma_neg(a.sigma, 4 * lane + k) ? -kInvSqrtD : kInvSqrtD;
            }
#pragma unroll
            for (int u = 0; u < 2; u++) {
                const int row = row0 + u * kWarps;
                if (row >= nr) break;
                if (ntl > 0) {
                    const float4 x = *reinterpret_cast<const float4 *>(sA + row * kEStride + 4 * lane);
                    o[u][0] += x.x;
                    o[u][1] += x.y;
                    o[u][2] += x.z;
                    o[u][3] += x.w;
                }
                const int rg = r0 + row, i = rg / a.G, gq = rg % a.G;
                const size_t prow = ((size_t)b * a.n + i) * a.Hq + h * a.G + gq;
                float *part = a.partials + (prow * a.S + split) * kPartialStride;
                *reinterpret_cast<float4 *>(part + 4 * lane) = make_float4(o[u][0], o[u][1], o[u][2], o[u][3]);
                if (lane == 0) {
                    part[kHeadDim] = ntl > 0 ? s_ml[row][0] : -CUDART_INF_F;
                    part[kHeadDim + 1] = ntl > 0 ? s_ml[row][1] : 0.f;
                }
            }
        }
    }
    // ------------------------------------------------------- split merge
    // The last split of the row block to arrive merges every split's partial
    // of its rows (a split with no key has m = -inf: weight 0) and writes the
    // output rows; it leaves the counter at zero for the next launch.
    if (a.counters) {
        __threadfence();
        __syncthreads();
        const int unit = (b * a.H + h) * a.nqb + qb;
        if (tid == 0) s_last = atomicAdd(a.counters + unit, 1) == a.S - 1;
        __syncthreads();
        if (s_last) {
            __threadfence();
            for (int row = warp; row < nr; row += kThreadsP / 32) {
                const int rg = r0 + row, i = rg / a.G, gq = rg % a.G;
                const size_t prow = ((size_t)b * a.n + i) * a.Hq + h * a.G + gq;
                const float *part = a.partials + prow * a.S * kPartialStride;
                float M = -CUDART_INF_F, l = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
                for (int sp = 0; sp < a.S; sp++) {
                    const float *p = part + (size_t)sp * kPartialStride;
                    const float m = __ldcg(p + kHeadDim), ls = __ldcg(p + kHeadDim + 1);
                    const float4 v = __ldcg(reinterpret_cast<const float4 *>(p) + lane);
                    if (m == -CUDART_INF_F) continue;   // uniform over the warp
                    const float Mn = fmaxf(M, m);
                    const float c0 = exp2f(M - Mn), c = exp2f(m - Mn);   // c0 = 0 while M = -inf
                    l = fmaf(ls, c, l * c0);
                    o[0] = fmaf(v.x, c, o[0] * c0);
                    o[1] = fmaf(v.y, c, o[1] * c0);
                    o[2] = fmaf(v.z, c, o[2] * c0);
                    o[3] = fmaf(v.w, c, o[3] * c0);
                    M = Mn;
                }
                *reinterpret_cast<float4 *>(a.out + prow * kHeadDim + 4 * lane) =
                    l > 0.f ? make_float4(o[0] / l, o[1] / l, o[2] / l, o[3] / l) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            if (tid == 0) a.counters[unit] = 0;
        }
    }
    if (warp == kMmaWarp) {
        tc::fence_after();
        tc::dealloc(tmem, kTmemCols);
    }
}

// One CTA per (q head, query token, sequence): the row's split partials,
// then the tail tokens it may see, 128 at a time: their logits (a warp per
// token, 4 elements per lane), the chunk's maximum, then o += sum 2^(z - M) v
// with thread tid owning element tid.
__global__ void __launch_bounds__(128) prefill_combine_kernel(const PrefillArgs a) {
    constexpr int kChunk = 128;
    __shared__ float s_z[kChunk];
    __shared__ float s_red[4];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int hq = blockIdx.x, i = blockIdx.y, b = blockIdx.z;
    const int h = hq / a.G;
    const size_t row = ((size_t)b * a.n + i) * a.Hq + hq;
    // of [committed, tail] the row sees T_b + n_tail - n + 1 + i tokens: all
    // committed ones when the new tokens are in the tail
    const int nt = (a.tail_k && !a.tail_in_kernel) ? max(0, a.n_tail - a.n + 1 + i) : 0;
    const size_t tstride = (size_t)a.H * kHeadDim;
    const uint16_t *tk = a.tail_k ? a.tail_k + ((size_t)b * a.tail_cap * a.H + h) * kHeadDim : nullptr;
    const uint16_t *tv = a.tail_v ? a.tail_v + ((size_t)b * a.tail_cap * a.H + h) * kHeadDim : nullptr;
    float q4[4] = {0.f, 0.f, 0.f, 0.f};
    if (nt > 0) {
        const uint2 qr = *reinterpret_cast<const uint2 *>(a.q + row * kHeadDim + 4 * lane);
        q4[0] = bf16_to_f32(qr.x & 0xFFFFu) * a.scale_log2;
        q4[1] = bf16_to_f32(qr.x >> 16) * a.scale_log2;
        q4[2] = bf16_to_f32(qr.y & 0xFFFFu) * a.scale_log2;
        q4[3] = bf16_to_f32(qr.y >> 16) * a.scale_log2;
    }
    float M, l, o;
    merge_partials(a.partials + row * a.S * kPartialStride, a.S, tid, M, l, o);
    for (int c0 = 0; c0 < nt; c0 += kChunk) {
        const int cn = min(kChunk, nt - c0);
        // logits of the chunk (L2 loads: the tail rows may just have been written)
#pragma unroll 4
        for (int jj = warp; jj < cn; jj += 4) {
            const uint2 kr = __ldcg(reinterpret_cast<const uint2 *>(tk + (size_t)(c0 + jj) * tstride + 4 * lane));
            float z = q4[0] * bf16_to_f32(kr.x & 0xFFFFu);
            z = fmaf(q4[1], bf16_to_f32(kr.x >> 16), z);
            z = fmaf(q4[2], bf16_to_f32(kr.y & 0xFFFFu), z);
            z = fmaf(q4[3], bf16_to_f32(kr.y >> 16), z);
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) z += __shfl_xor_sync(0xffffffffu, z, m);
            if (lane == 0) s_z[jj] = z;
        }
        __syncthreads();
        float mc = tid < cn ? s_z[tid] : -CUDART_INF_F;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, m));
        if (lane == 0) s_red[warp] = mc;
        __syncthreads();
        const float Mn = fmaxf(M, fmaxf(fmaxf(s_red[0], s_red[1]), fmaxf(s_red[2], s_red[3])));
        const float c = exp2f(M - Mn);   // 0 while M = -inf
        l *= c;
        o *= c;
#pragma unroll 8
        for (int j = 0; j < cn; j++) {
            const float w = exp2f(s_z[j] - Mn);
            l += w;
            o = fmaf(w, bf16_to_f32(__ldcg(tv + (size_t)(c0 + j) * tstride + tid)), o);
        }
        M = Mn;
        __syncthreads();   // s_z and s_red are rewritten by the next chunk
    }
    a.out[row * kHeadDim + tid] = (l > 0.f) ? o / l : 0.f;
}

template <int BA, int BR, int GS, bool RESID, bool PG>
struct Variant {
    static cudaError_t configure() {
        static bool done[kMaxDevices];
        return once_per_device(done, [] {
            return cudaFuncSetAttribute(prefill_tc_kernel<BA, BR, GS, RESID, PG>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        });
    }
    static cudaError_t launch(const PrefillArgs &a, cudaStream_t st) {
        cudaError_t e = configure();
        if (e != cudaSuccess) return e;
        if (a.S > 0)
            prefill_tc_kernel<BA, BR, GS, RESID, PG><<<dim3(a.S, a.H, a.B * a.nqb), kThreadsP, kSmemBytes, st>>>(a);
        return cudaGetLastError();
    }
};

template <int BA, int BR, int GS>
cudaError_t launch_bits(const PrefillArgs &a, cudaStream_t st) {
    if (a.pg.table)
        return a.r_codes[0] ? Variant<BA, BR, GS, true, true>::launch(a, st) : Variant<BA, BR, GS, false, true>::launch(a, st);
    return a.r_codes[0] ? Variant<BA, BR, GS, true, false>::launch(a, st) : Variant<BA, BR, GS, false, false>::launch(a, st);
}

template <int GS>
cudaError_t launch_group(const PrefillArgs &a, int ba, int br, cudaStream_t st) {
    if (ba == 2 && br == 2) return launch_bits<2, 2, GS>(a, st);
    if (ba == 4 && br == 4) return launch_bits<4, 4, GS>(a, st);
    return launch_bits<4, 2, GS>(a, st);
}

}  // namespace

// Row blocks of 64 query rows per kv head; splits: the count with the least
// wave-quantised work (waves x 64-token steps of the largest split, plus a
// fixed cost of RQ_PREFILL_STEP_OVERHEAD steps per CTA), one CTA per SM (the tiles take 193 KB of shared memory
// and the accumulators all 512 tensor-memory columns).
#ifndef RQ_PREFILL_STEP_OVERHEAD
#define RQ_PREFILL_STEP_OVERHEAD 3
#endif
void prefill_plan(PrefillArgs *a, int T, int ba, int br, int sms) {
    (void)ba;
    (void)br;
    const int nq = a->n * a->G;
    a->nqb = (nq + kRows - 1) / kRows;
    a->S = 0;
    a->tail_in_kernel = 0;
    if (T <= 0) return;   // nothing committed: the combine kernel takes the tail
    a->tail_in_kernel = 1;
    const long slots = (long)std::max(1, sms);
    const long units = (long)a->B * a->H * a->nqb;
    const int nt = (T + kTokTile - 1) / kTokTile;
    long best = -1;
    for (int S = 1; S <= std::min(nt, kMaxSplits); S++) {
        const long waves = (S * units + slots - 1) / slots;
        const long cost = waves * ((nt + S - 1) / S + RQ_PREFILL_STEP_OVERHEAD);
        if (best < 0 || cost < best) {
            best = cost;
            a->S = S;
        }
    }
}

cudaError_t launch_prefill(const PrefillArgs &a, int ba, int br, cudaStream_t st) {
    if (!((ba == 4 && br == 2) || (ba == 2 && br == 2) || (ba == 4 && br == 4))) return cudaErrorInvalidValue;
    if (a.g != 16 && a.g != 32) return cudaErrorInvalidValue;
    cudaError_t e = a.g == 16 ? launch_group<16>(a, ba, br, st) : launch_group<32>(a, ba, br, st);
    if (e != cudaSuccess) return e;
    if (!a.counters) prefill_combine_kernel<<<dim3(a.Hq, a.n, a.B), 128, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace rq
