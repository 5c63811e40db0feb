// prefill.cu -- multi-token causal attention over the ResidualQuant cache: the
// step before decode (chunked prefill, or verifying several drafted tokens),
// which the ai4snews summary's throughput study (paragraph 4) leaves out of
// its decode timing.  Query row (i, hq) of sequence b, i < n, attends to the
// first T_b + n_tail - n + 1 + i tokens of [the group's committed tokens, the
// loop's BF16 tail tokens]: the n new tokens are the most recent ones,
// committed already at an anchor loop, in the tail at the other loops.
//
// Design.  With n query tokens per sequence the keys are shared by n * G
// query rows, so a CTA dequantizes each record once into shared memory in
// fp32 (k_hat = s_hat a_hat + R^T y_hat; the inverse rotation is one warp
// Walsh-Hadamard transform per token, cheaper than rotating n * G queries
// once the rows outnumber a few) and runs both products, logits and p V, on
// the FP32 pipes from shared memory:
//  - CTA = (split of the committed tokens, kv head, sequence x block of
//    8 RPW query rows, RPW in {1, 2, 4, 8} the fewest that hold a kv head's
//    n * G rows), 8 warps; warp w owns rows w, w + 8, ...;
//  - per 32-token step: dequantize K (warp per token), logits (lane = token,
//    a row's 32 logits in one warp), online softmax per row, dequantize V,
//    o += p V (lane = 4 columns of head_dim); the raw records of the next
//    step are copied into a second shared buffer (cp.async) meanwhile;
//  - each CTA writes a partial (m, l, o) per row; a second kernel merges the
//    partials and the tail tokens of each row (combine_row) under the row's
//    causal limit.
// This is a CUDA-core kernel: the contraction per step is at most 64 x 32 x
// 128 twice, on fp32 reconstructions; BF16 tensor-core operands would add a
// rounding of every reconstructed key and value.
#include <math_constants.h>

#include <algorithm>

#include "combine.cuh"
#include "common.cuh"
#include "prefill.h"

namespace rq {
namespace {

constexpr int kThreadsP = 256;
constexpr int kQStride = kHeadDim + 4;   // float4-aligned query rows
constexpr int kKStride = kHeadDim + 1;   // lane = token reads a column without bank conflicts
constexpr int kPStride = kPrefillTile + 1;
// shared floats of a CTA of `rows` query rows: q, one reconstructed tile, probabilities
__host__ __device__ constexpr int float_smem(int rows) {
    return rows * kQStride + kPrefillTile * kKStride + rows * kPStride;
}
constexpr float kInvSqrtD = 0.08838834764831845f;   // 1 / sqrt(128)

// Raw records of one 32-token tile, K then V, each side laid out
// [anchor codes][anchor meta][residual codes][residual meta][coefficients]
// (meta sized for the largest, group 16); two such stages are in flight.
template <int BA, int BR>
struct Stage {
    static constexpr int A_C = 16 * BA, R_C = 16 * BR, MR_MAX = 16;
    static constexpr int SIDE = kPrefillTile * (A_C + R_C + 2 * MR_MAX) + 2 * kPrefillTile;
    static constexpr int BYTES = 2 * SIDE;
    static constexpr size_t smem(int rows) { return (size_t)float_smem(rows) * sizeof(float) + 2 * (size_t)BYTES; }
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// bytes (a multiple of 16, both addresses 16-byte aligned) spread over the CTA
__device__ __forceinline__ void copy_async(uint8_t *dst, const uint8_t *src, int bytes, int tid) {
    for (int o = 16 * tid; o < bytes; o += 16 * kThreadsP) cp_async16(dst + o, src + o);
}

// Issue the copies of the tile whose first record is rec0 (a multiple of 32:
// every source is 16-byte aligned, and a whole tile lies inside the stream's
// padded capacity).
template <int BA, int BR>
__device__ __forceinline__ void stage_tile(const PrefillArgs &a, uint8_t *st, size_t rec0, int MR, bool resid,
                                           int tid) {
    using SG = Stage<BA, BR>;
    constexpr int TT = kPrefillTile;
#pragma unroll
    for (int kv = 0; kv < 2; kv++) {
        uint8_t *d = st + kv * SG::SIDE;
        copy_async(d, a.a_codes[kv] + rec0 * SG::A_C, TT * SG::A_C, tid);
        copy_async(d + TT * SG::A_C, a.a_meta[kv] + rec0 * MR, TT * MR, tid);
        if (resid) {
            copy_async(d + TT * (SG::A_C + MR), a.r_codes[kv] + rec0 * SG::R_C, TT * SG::R_C, tid);
            copy_async(d + TT * (SG::A_C + MR + SG::R_C), a.r_meta[kv] + rec0 * MR, TT * MR, tid);
            copy_async(d + TT * (SG::A_C + SG::R_C + 2 * MR), reinterpret_cast<const uint8_t *>(a.r_coef[kv] + rec0),
                       2 * TT, tid);
        }
    }
}

// The codes of elements 4 lane .. 4 lane + 3 of a record, LSB first.
template <int BITS>
__device__ __forceinline__ uint32_t lane_codes(const uint8_t *rec, int lane) {
    if (BITS == 4) return *reinterpret_cast<const uint16_t *>(rec + 2 * lane);
    return rec[lane];
}

// Reconstruct side kv of the staged tile, tokens 0 .. tn - 1, into rows
// 0 .. tn - 1 of sK (rows tn .. 31 zeroed); warp per token, lane holds
// elements 4 lane .. 4 lane + 3.
template <int BA, int BR>
__device__ __forceinline__ void dequant_tile(const PrefillArgs &a, const uint8_t *st, int kv, int MR, bool resid,
                                             int tn, float *sK, int warp, int lane) {
    using SG = Stage<BA, BR>;
    constexpr int TT = kPrefillTile;
    const uint8_t *d = st + kv * SG::SIDE;
    const int gi = (4 * lane) / a.g;   // quantization group of this lane's elements
#pragma unroll
    for (int u = warp; u < TT; u += kThreadsP / 32) {
        float x[4] = {0.f, 0.f, 0.f, 0.f};
        if (u < tn) {
            const uint32_t w = lane_codes<BA>(d + u * SG::A_C, lane);
            const uint8_t *mp = d + TT * SG::A_C + u * MR + 2 * gi;
            const float sc = e4m3_to_f32(mp[0]), mn = e4m3_to_f32(mp[1]);
#pragma unroll
            for (int k = 0; k < 4; k++) x[k] = fmaf((float)((w >> (BA * k)) & ((1u << BA) - 1)), sc, mn);
            if (resid) {
                const float sh =
                    bf16_to_f32(reinterpret_cast<const uint16_t *>(d + TT * (SG::A_C + SG::R_C + 2 * MR))[u]);
                const uint32_t wr = lane_codes<BR>(d + TT * (SG::A_C + MR) + u * SG::R_C, lane);
                const uint8_t *mr = d + TT * (SG::A_C + MR + SG::R_C) + u * MR + 2 * gi;
                const float rs = e4m3_to_f32(mr[0]), rm = e4m3_to_f32(mr[1]);
                float y[4];
#pragma unroll
                for (int k = 0; k < 4; k++) y[k] = fmaf((float)((wr >> (BR * k)) & ((1u << BR) - 1)), rs, rm);
                if (a.rotate) {
                    // R^T y = diag(sigma) H y / sqrt(d)
                    wht128_warp(y, lane);
#pragma unroll
                    for (int k = 0; k < 4; k++) y[k] *= sigma_neg(a.sigma, 4 * lane + k) ? -kInvSqrtD : kInvSqrtD;
                }
#pragma unroll
                for (int k = 0; k < 4; k++) x[k] = fmaf(sh, x[k], y[k]);
            }
        }
#pragma unroll
        for (int k = 0; k < 4; k++) sK[u * kKStride + 4 * lane + k] = x[k];
    }
}

// RPW query rows per warp (8 RPW per CTA); fewer rows leave room for more CTAs per SM
template <int BA, int BR, int RPW>
__global__ void __launch_bounds__(kThreadsP, RPW <= 2 ? 4 : RPW == 4 ? 3 : 2) prefill_rq_kernel(const PrefillArgs a) {
    using SG = Stage<BA, BR>;
    constexpr int ROWS = 8 * RPW;
    extern __shared__ __align__(16) float smem[];
    float *sQ = smem;                                  // [ROWS][kQStride] q * scale * log2(e)
    float *sK = sQ + ROWS * kQStride;                  // [32][kKStride] reconstructed K, then V
    float *sP = sK + kPrefillTile * kKStride;          // [ROWS][kPStride] probabilities of the step
    uint8_t *sRaw = reinterpret_cast<uint8_t *>(smem + float_smem(ROWS));   // 2 stages of raw records

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, h = blockIdx.y;
    const int b = blockIdx.z / a.nqb, qb = blockIdx.z % a.nqb;
    const int r0 = qb * ROWS;                                   // first query row (i * G + gq) of the CTA
    const int nr = min(ROWS, a.n * a.G - r0);                   // rows of the CTA
    const int Tb = a.seqT.v[b];
    int t0, cnt;
    split_range(split, a.S, Tb, &t0, &cnt);
    const size_t bh = (size_t)b * a.H + h;
    const int MR = 2 * (kHeadDim / a.g);
    const bool resid = a.r_codes[0] != nullptr;
    const int ntl = (cnt + kPrefillTile - 1) / kPrefillTile;

    if (ntl > 0) stage_tile<BA, BR>(a, sRaw, bh * a.Tp + t0, MR, resid, tid);
    cp_async_commit();

    for (int idx = tid; idx < ROWS * kHeadDim; idx += kThreadsP) {
        const int r = idx / kHeadDim, d = idx % kHeadDim;
        float v = 0.f;
        if (r < nr) {
            const int rg = r0 + r, i = rg / a.G, gq = rg % a.G;
            v = bf16_to_f32(a.q[(((size_t)b * a.n + i) * a.Hq + h * a.G + gq) * kHeadDim + d]) * a.scale_log2;
        }
        sQ[r * kQStride + d] = v;
    }
    // this warp's rows: warp + 8 j for j < jn
    const int jn = nr > warp ? (nr - warp + 7) / 8 : 0;
    int lim[RPW];   // committed tokens each row may see
    float m[RPW], l[RPW], acc[RPW][4];
#pragma unroll
    for (int j = 0; j < RPW; j++) {
        const int i = (r0 + warp + 8 * j) / a.G;
        lim[j] = min(Tb, Tb + a.n_tail - a.n + 1 + i);
        m[j] = -CUDART_INF_F;
        l[j] = 0.f;
#pragma unroll
        for (int k = 0; k < 4; k++) acc[j][k] = 0.f;
    }

    for (int kt = 0; kt < ntl; kt++) {
        const int tt = kt * kPrefillTile;
        const int tn = min(kPrefillTile, cnt - tt);
        const uint8_t *st = sRaw + (kt & 1) * SG::BYTES;
        // the next tile's copies overlap this tile's work; its stage was
        // released by the barrier that ended the step before
        if (kt + 1 < ntl)
            stage_tile<BA, BR>(a, sRaw + ((kt + 1) & 1) * SG::BYTES, bh * a.Tp + t0 + tt + kPrefillTile, MR,
                               resid, tid);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();   // this tile's records (and, first time, sQ) are visible
        dequant_tile<BA, BR>(a, st, 0, MR, resid, tn, sK, warp, lane);
        __syncthreads();
        // logits of token lane for the warp's rows
        float s[RPW];
#pragma unroll
        for (int j = 0; j < RPW; j++) s[j] = 0.f;
        const float *kr = sK + lane * kKStride;
#pragma unroll 2
        for (int d = 0; d < kHeadDim; d += 4) {
            const float k0 = kr[d], k1 = kr[d + 1], k2 = kr[d + 2], k3 = kr[d + 3];
#pragma unroll
            for (int j = 0; j < RPW; j++) {
                if (j < jn) {
                    const float4 qv = *reinterpret_cast<const float4 *>(sQ + (warp + 8 * j) * kQStride + d);
                    s[j] = fmaf(qv.x, k0, fmaf(qv.y, k1, fmaf(qv.z, k2, fmaf(qv.w, k3, s[j]))));
                }
            }
        }
        // online softmax per row (log2 domain); masked tokens weigh 0
        const int tabs = t0 + tt + lane;
#pragma unroll
        for (int j = 0; j < RPW; j++) {
            if (j < jn) {
                const bool valid = lane < tn && tabs < lim[j];
                const float z = valid ? s[j] : -CUDART_INF_F;
                float mx = z;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                const float mn = fmaxf(m[j], mx);
                float p = 0.f, alpha = 1.f;
                if (mn != -CUDART_INF_F) {
                    alpha = exp2f(m[j] - mn);   // 0 while nothing was seen
                    p = valid ? exp2f(z - mn) : 0.f;
                }
                float ps = p;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
                l[j] = fmaf(l[j], alpha, ps);
                m[j] = mn;
#pragma unroll
                for (int k = 0; k < 4; k++) acc[j][k] *= alpha;
                sP[(warp + 8 * j) * kPStride + lane] = p;
            }
        }
        __syncthreads();   // every logit has read sK; sP is complete
        dequant_tile<BA, BR>(a, st, 1, MR, resid, tn, sK, warp, lane);
        __syncthreads();
        for (int t = 0; t < tn; t++) {
            const float *vr = sK + t * kKStride;
            const float v0 = vr[lane], v1 = vr[lane + 32], v2 = vr[lane + 64], v3 = vr[lane + 96];
#pragma unroll
            for (int j = 0; j < RPW; j++) {
                if (j < jn) {
                    const float p = sP[(warp + 8 * j) * kPStride + t];
                    acc[j][0] = fmaf(p, v0, acc[j][0]);
                    acc[j][1] = fmaf(p, v1, acc[j][1]);
                    acc[j][2] = fmaf(p, v2, acc[j][2]);
                    acc[j][3] = fmaf(p, v3, acc[j][3]);
                }
            }
        }
        __syncthreads();   // sK, sP and this stage are rewritten by the next steps
    }
    cp_async_wait<0>();

#pragma unroll
    for (int j = 0; j < RPW; j++) {
        if (j < jn) {
            const int rg = r0 + warp + 8 * j, i = rg / a.G, gq = rg % a.G;
            const size_t row = ((size_t)b * a.n + i) * a.Hq + h * a.G + gq;
            float *part = a.partials + (row * a.S + split) * kPartialStride;
#pragma unroll
            for (int k = 0; k < 4; k++) part[lane + 32 * k] = acc[j][k];
            if (lane == 0) {
                part[kHeadDim] = m[j];
                part[kHeadDim + 1] = l[j];
            }
        }
    }
}

struct Sync128 {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

// One CTA per (q head, query token, sequence): the row's partials, then the
// tail tokens it may see.
__global__ void __launch_bounds__(128) prefill_combine_kernel(const PrefillArgs a) {
    __shared__ float s_red[4];
    const int hq = blockIdx.x, i = blockIdx.y, b = blockIdx.z;
    const int h = hq / a.G;
    const size_t row = ((size_t)b * a.n + i) * a.Hq + hq;
    // of [committed, tail] the row sees T_b + n_tail - n + 1 + i tokens: all
    // committed ones when the new tokens are in the tail
    const int nt = a.tail_k ? max(0, a.n_tail - a.n + 1 + i) : 0;
    const size_t trow = ((size_t)b * a.tail_cap * a.H + h) * kHeadDim;
    combine_row(a.partials + row * a.S * kPartialStride, a.S, a.q + row * kHeadDim, a.scale_log2,
                a.tail_k ? a.tail_k + trow : nullptr, a.tail_v ? a.tail_v + trow : nullptr,
                (size_t)a.H * kHeadDim, nt, a.out + row * kHeadDim, threadIdx.x, s_red, Sync128());
}

template <int BA, int BR, int RPW>
struct Variant {
    static cudaError_t configure() {
        static bool done = false;
        if (done) return cudaSuccess;
        cudaError_t e = cudaFuncSetAttribute(prefill_rq_kernel<BA, BR, RPW>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)Stage<BA, BR>::smem(8 * RPW));
        if (e == cudaSuccess) done = true;
        return e;
    }
    static int occupancy() {
        static int occ = 0;
        if (occ == 0 && configure() == cudaSuccess &&
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, prefill_rq_kernel<BA, BR, RPW>, kThreadsP,
                                                          Stage<BA, BR>::smem(8 * RPW)) != cudaSuccess)
            occ = 0;
        return occ > 0 ? occ : 1;
    }
    static cudaError_t launch(const PrefillArgs &a, cudaStream_t st) {
        cudaError_t e = configure();
        if (e != cudaSuccess) return e;
        if (a.S > 0)
            prefill_rq_kernel<BA, BR, RPW>
                <<<dim3(a.S, a.H, a.B * a.nqb), kThreadsP, Stage<BA, BR>::smem(8 * RPW), st>>>(a);
        return cudaGetLastError();
    }
};

// f(Variant) for the (bits, rows per warp) of a
template <typename F>
auto with_variant(int ba, int br, int rpw, F f) -> decltype(f(Variant<4, 2, 1>())) {
#define RQ_PREFILL_RPW(BA, BR)                      \
    switch (rpw) {                                  \
        case 1: return f(Variant<BA, BR, 1>());     \
        case 2: return f(Variant<BA, BR, 2>());     \
        case 4: return f(Variant<BA, BR, 4>());     \
        default: return f(Variant<BA, BR, 8>());    \
    }
    if (ba == 2 && br == 2) RQ_PREFILL_RPW(2, 2)
    if (ba == 4 && br == 4) RQ_PREFILL_RPW(4, 4)
    RQ_PREFILL_RPW(4, 2)
#undef RQ_PREFILL_RPW
}

}  // namespace

// Rows per warp: the fewest that hold every query row of a kv head (at most
// 8, 64 rows per CTA).  Splits: the count with the least wave-quantised work
// (waves x 64-token tiles of the largest split, plus one tile of fixed cost),
// waves counted from the variant's measured occupancy.
void prefill_plan(PrefillArgs *a, int T, int ba, int br, int sms) {
    const int nq = a->n * a->G;
    a->rpw = nq <= 8 ? 1 : nq <= 16 ? 2 : nq <= 32 ? 4 : 8;
    a->nqb = (nq + 8 * a->rpw - 1) / (8 * a->rpw);
    a->S = 0;
    if (T <= 0) return;
    const int occ = with_variant(ba, br, a->rpw, [](auto v) { return decltype(v)::occupancy(); });
    const long slots = (long)std::max(1, occ) * std::max(1, sms);
    const long units = (long)a->B * a->H * a->nqb;
    const int nt = (T + kTokTile - 1) / kTokTile;
    long best = -1;
    for (int S = 1; S <= std::min(nt, kMaxSplits); S++) {
        const long waves = (S * units + slots - 1) / slots;
        const long cost = waves * ((nt + S - 1) / S + 1);
        if (best < 0 || cost < best) {
            best = cost;
            a->S = S;
        }
    }
}

cudaError_t launch_prefill(const PrefillArgs &a, int ba, int br, cudaStream_t st) {
    if (!((ba == 4 && br == 2) || (ba == 2 && br == 2) || (ba == 4 && br == 4))) return cudaErrorInvalidValue;
    cudaError_t e = with_variant(ba, br, a.rpw, [&](auto v) { return decltype(v)::launch(a, st); });
    if (e != cudaSuccess) return e;
    prefill_combine_kernel<<<dim3(a.Hq, a.n, a.B), 128, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace rq
