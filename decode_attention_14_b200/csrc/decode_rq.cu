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
// basis, the residual part in the rotated basis, and R^T is applied once per
// CTA to the rotated accumulator.
//
// Arithmetic.  The per-code products run on the integer dot-product unit
// (dp2a: two 16-bit x 8-bit products per instruction): q (and R q) are
// converted once per CTA to 16-bit fixed point with a power-of-two scale,
// and the V weights p_t * s_t * sc_{g,t} to 16-bit fixed point with one
// power-of-two scale per quantization group, chosen from the chunk's largest
// weight bound (so every weight keeps >= 14 significant bits).  Per-group
// scales, minima, softmax and the final rotation stay in fp32.
//
// Data movement.  Each CTA owns a chunk of one (sequence, kv head), streamed
// in 64-token tiles through a 3-stage shared-memory ring filled by one
// producer warp with 1-D bulk asynchronous copies (cp.async.bulk, completion
// counted on mbarriers; no multicast).  Pass 1 streams the K records and
// writes the chunk's logits; pass 2 streams the V codes (the V scales,
// minima and coefficients were fetched once at CTA start) and sums
// exp2(z - chunk max) * v.  Every mbarrier wait is bounded: on timeout the
// kernel records an error word, stops issuing copies, drains what it issued
// and finishes without touching further data.
//
// Thread map (pass 1 and 2): 4 consumer warps x 16 tokens of each tile;
// lane 8s+j takes head_dim segment j (elements 16j..16j+15) of tokens
// s, s+4, s+8, s+12 of its warp's 16.
#include <math_constants.h>

#include "common.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

constexpr int kTile = 64;
constexpr int kStages = 3;
constexpr int kConsumers = 128;
constexpr int kThreads = kConsumers + 32;
constexpr float kRsqrt128 = 0.088388347648318440f;
constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23: float(x) + kMagic holds round(x) in its low bits
constexpr unsigned long long kWaitNs = 1000000000ull;   // 1 s per wait

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Bounded wait on an mbarrier phase; gives up after kWaitNs or as soon as
// another warp of the CTA has given up.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (global_ns() - t0 > kWaitNs) return false;
    }
}
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }

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

// Which two segment elements sit in the 16-bit halves of q pair register r,
// matching the byte lanes the unpacking below produces (dp2a .lo uses code
// bytes 0,1; .hi bytes 2,3).
template <int BITS>
__device__ __forceinline__ void qpair_index(int r, int &i0, int &i1) {
    if (BITS == 4) {
        // lo nibbles of word u: bytes = elements 8u+{0,2,4,6}; hi nibbles: 8u+{1,3,5,7}
        const int u = r >> 2, hi = (r >> 1) & 1, upper = r & 1;
        i0 = 8 * u + hi + 4 * upper;
        i1 = i0 + 2;
    } else {
        // (w >> 2c) & 0x03030303: bytes = elements c, 4+c, 8+c, 12+c
        const int c = r >> 1, upper = r & 1;
        i0 = c + 8 * upper;
        i1 = i0 + 4;
    }
}

// sum_i q_i c_i over a segment, q as 16-bit pairs in the order of qpair_index.
template <int BITS>
__device__ __forceinline__ int dot_seg(const Seg<BITS> &s, const uint32_t qp[8]) {
    int acc = 0;
    if (BITS == 4) {
#pragma unroll
        for (int u = 0; u < 2; u++) {
            const int lo = (int)(s.w[u] & 0x0F0F0F0Fu);
            const int hi = (int)((s.w[u] >> 4) & 0x0F0F0F0Fu);
            acc = __dp2a_lo((int)qp[4 * u + 0], lo, acc);
            acc = __dp2a_hi((int)qp[4 * u + 1], lo, acc);
            acc = __dp2a_lo((int)qp[4 * u + 2], hi, acc);
            acc = __dp2a_hi((int)qp[4 * u + 3], hi, acc);
        }
    } else {
#pragma unroll
        for (int c = 0; c < 4; c++) {
            const int b = (int)((s.w[0] >> (2 * c)) & 0x03030303u);
            acc = __dp2a_lo((int)qp[2 * c + 0], b, acc);
            acc = __dp2a_hi((int)qp[2 * c + 1], b, acc);
        }
    }
    return acc;
}

// acc[i] += w0 * c0_i + w1 * c1_i for the 16 elements of a segment, codes of
// two tokens, weights packed as (w0 | w1 << 16).
template <int BITS>
__device__ __forceinline__ void acc_pair(const Seg<BITS> &a, const Seg<BITS> &b, uint32_t wp, int acc[16]) {
    const int W = (int)wp;
    if (BITS == 4) {
#pragma unroll
        for (int u = 0; u < 2; u++) {
            const uint32_t X = __byte_perm(a.w[u], b.w[u], 0x5140);   // bytes 0,1 of both tokens
            const uint32_t Y = __byte_perm(a.w[u], b.w[u], 0x7362);   // bytes 2,3 of both tokens
            const int xl = (int)(X & 0x0F0F0F0Fu), xh = (int)((X >> 4) & 0x0F0F0F0Fu);
            const int yl = (int)(Y & 0x0F0F0F0Fu), yh = (int)((Y >> 4) & 0x0F0F0F0Fu);
            acc[8 * u + 0] = __dp2a_lo(W, xl, acc[8 * u + 0]);
            acc[8 * u + 2] = __dp2a_hi(W, xl, acc[8 * u + 2]);
            acc[8 * u + 1] = __dp2a_lo(W, xh, acc[8 * u + 1]);
            acc[8 * u + 3] = __dp2a_hi(W, xh, acc[8 * u + 3]);
            acc[8 * u + 4] = __dp2a_lo(W, yl, acc[8 * u + 4]);
            acc[8 * u + 6] = __dp2a_hi(W, yl, acc[8 * u + 6]);
            acc[8 * u + 5] = __dp2a_lo(W, yh, acc[8 * u + 5]);
            acc[8 * u + 7] = __dp2a_hi(W, yh, acc[8 * u + 7]);
        }
    } else {
        const uint32_t X = __byte_perm(a.w[0], b.w[0], 0x5140);   // bytes 0,1: elements 0-7
        const uint32_t Y = __byte_perm(a.w[0], b.w[0], 0x7362);   // bytes 2,3: elements 8-15
#pragma unroll
        for (int c = 0; c < 4; c++) {
            const int x = (int)((X >> (2 * c)) & 0x03030303u);
            const int y = (int)((Y >> (2 * c)) & 0x03030303u);
            acc[c] = __dp2a_lo(W, x, acc[c]);
            acc[4 + c] = __dp2a_hi(W, x, acc[4 + c]);
            acc[8 + c] = __dp2a_lo(W, y, acc[8 + c]);
            acc[12 + c] = __dp2a_hi(W, y, acc[12 + c]);
        }
    }
}

// (scale, min) of an FP8 pair stored little-endian as scale | min << 8.
__device__ __forceinline__ float2 meta_pair(uint32_t m16) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)m16, __NV_E4M3);
    return __half22float2(__half2(h));
}

// exact int -> float for |x| < 2^22 on the ALU pipes
__device__ __forceinline__ float i2f_exact(int x) { return __int_as_float(x + 0x4B400000) - kMagic; }

// round(x * y) (|x * y| < 2^15) in the low 16 bits, one rounding, ties to even
__device__ __forceinline__ uint32_t fix16_bits_fma(float x, float y) { return __float_as_uint(fmaf(x, y, kMagic)); }

// power-of-two scale 2^F putting a positive bound into [2^(top-1), 2^top)
__device__ __forceinline__ float fixed_scale(float bound, int top) {
    if (!(bound > 0.f)) return 1.f;
    int e;
    frexpf(bound, &e);                       // bound = m 2^e, m in [0.5, 1)
    const int F = max(-100, min(100, top - e));
    return ldexpf(1.f, F);
}

struct Layout2 {
    int A_C, R_C, MR;
    int k_am, k_rc, k_rm, k_cf, k_bytes;
    int v_rc, v_bytes;
    int stage_bytes;
    int vm_r, vm_cf, vm_bytes;   // retained V meta: anchor meta, resid meta, coef
    int sc_off;
};

template <int BA, int BR, bool RESID>
__device__ __forceinline__ Layout2 make_layout2(int g, int chunk_tiles) {
    Layout2 L;
    L.A_C = 16 * BA;
    L.R_C = 16 * BR;
    L.MR = 256 / g;
    L.k_am = kTile * L.A_C;
    L.k_rc = L.k_am + kTile * L.MR;
    L.k_rm = L.k_rc + (RESID ? kTile * L.R_C : 0);
    L.k_cf = L.k_rm + (RESID ? kTile * L.MR : 0);
    L.k_bytes = L.k_cf + (RESID ? kTile * 2 : 0);
    L.v_rc = kTile * L.A_C;
    L.v_bytes = L.v_rc + (RESID ? kTile * L.R_C : 0);
    L.stage_bytes = ((max(L.k_bytes, L.v_bytes) + 127) / 128) * 128;
    const int ct = chunk_tiles * kTile;
    L.vm_r = ct * L.MR;
    L.vm_cf = L.vm_r + (RESID ? ct * L.MR : 0);
    L.vm_bytes = L.vm_cf + (RESID ? ct * 2 : 0);
    L.sc_off = kStages * L.stage_bytes + ((L.vm_bytes + 127) / 128) * 128;
    return L;
}

template <int GK, int BA, int BR, bool RESID>
__global__ void __launch_bounds__(kThreads) decode_rq_kernel(const DecodeArgs a) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ __align__(8) uint64_t bar_full[kStages];
    __shared__ __align__(8) uint64_t bar_empty[kStages];
    __shared__ __align__(8) uint64_t bar_vm;
    __shared__ int s_abort;
    __shared__ float s_q[GK][2][kHeadDim];
    __shared__ float s_red[4][2 * GK + 16];
    __shared__ float s_acc[4][GK][2][kHeadDim];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int split = blockIdx.x, h = blockIdx.y;
    const int npairs = a.G / GK;
    const int b = blockIdx.z / npairs, pair = blockIdx.z % npairs;
    const int hq0 = h * a.G + pair * GK;
    const int t0 = split * a.chunk;
    const int n = min(a.chunk, a.T - t0);
    const int ntiles = (n + kTile - 1) / kTile;
    const int chunk_tiles = a.chunk / kTile;
    const size_t bh = (size_t)b * a.H + h;
    const Layout2 L = make_layout2<BA, BR, RESID>(a.g, chunk_tiles);
    uint8_t *ring = smem;
    uint8_t *vm = smem + kStages * L.stage_bytes;
    float *s_sc = reinterpret_cast<float *>(smem + L.sc_off);   // [GK][chunk] logits, then p
    float *s_P = s_sc + GK * a.chunk;                           // [GK][chunk] p * s_hat(V)

    if (tid == 0) {
        for (int i = 0; i < kStages; i++) {
            mbar_init(&bar_full[i], 1);
            mbar_init(&bar_empty[i], 4);
        }
        mbar_init(&bar_vm, 1);
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    // ------------------------------------------------------------ producer
    if (warp == 4) {
        if (lane == 0) {
            const size_t tok0 = bh * a.Tp + (size_t)t0;
            const uint32_t ntok = (uint32_t)(ntiles * kTile);
            // V scales/minima (+ coefficients) of the whole chunk, fetched once
            {
                uint32_t bytes = ntok * L.MR + (RESID ? ntok * (L.MR + 2) : 0);
                mbar_expect_tx(&bar_vm, bytes);
                bulk_g2s(vm, a.a_meta[1] + tok0 * L.MR, ntok * L.MR, &bar_vm);
                if (RESID) {
                    bulk_g2s(vm + L.vm_r, a.r_meta[1] + tok0 * L.MR, ntok * L.MR, &bar_vm);
                    bulk_g2s(vm + L.vm_cf, a.r_coef[1] + tok0, ntok * 2, &bar_vm);
                }
            }
            int issued = 0;
            for (int it = 0; it < 2 * ntiles; it++) {
                const int stage = it % kStages;
                if (it >= kStages && !mbar_wait(&bar_empty[stage], ((it / kStages) - 1) & 1, &s_abort)) {
                    s_abort = 1;
                    atomicExch(a.err, 1);
                    break;
                }
                uint8_t *st = ring + stage * L.stage_bytes;
                const bool kpass = it < ntiles;
                const size_t tk = tok0 + (size_t)(kpass ? it : it - ntiles) * kTile;
                if (kpass) {
                    mbar_expect_tx(&bar_full[stage], (uint32_t)L.k_bytes);
                    bulk_g2s(st, a.a_codes[0] + tk * L.A_C, kTile * L.A_C, &bar_full[stage]);
                    bulk_g2s(st + L.k_am, a.a_meta[0] + tk * L.MR, kTile * L.MR, &bar_full[stage]);
                    if (RESID) {
                        bulk_g2s(st + L.k_rc, a.r_codes[0] + tk * L.R_C, kTile * L.R_C, &bar_full[stage]);
                        bulk_g2s(st + L.k_rm, a.r_meta[0] + tk * L.MR, kTile * L.MR, &bar_full[stage]);
                        bulk_g2s(st + L.k_cf, a.r_coef[0] + tk, kTile * 2, &bar_full[stage]);
                    }
                } else {
                    mbar_expect_tx(&bar_full[stage], (uint32_t)L.v_bytes);
                    bulk_g2s(st, a.a_codes[1] + tk * L.A_C, kTile * L.A_C, &bar_full[stage]);
                    if (RESID) bulk_g2s(st + L.v_rc, a.r_codes[1] + tk * L.R_C, kTile * L.R_C, &bar_full[stage]);
                }
                issued = it + 1;
            }
            // drain: every issued copy must have landed before the CTA exits
            mbar_wait(&bar_vm, 0, &s_abort);
            for (int it = max(0, issued - kStages); it < issued; it++)
                mbar_wait(&bar_full[it % kStages], (it / kStages) & 1, &s_abort);
        }
        return;
    }

    // ------------------------------------------------------------ consumers
    const int sub = lane >> 3, seg = lane & 7;
    const int mgrp = (seg * 16) / a.g;

    // q (log2-domain scale folded in) and R q, then 16-bit fixed point
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
    const float qscale = fixed_scale(qmax, 14);  // q_int = round(q * qscale), |q_int| <= 2^14
    const float qinv = 1.f / qscale;             // exact (power of two)
    uint32_t qpA[GK][8], qpR[GK][8];
    float QA[GK], QR[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        QA[gq] = QR[gq] = 0.f;
#pragma unroll
        for (int r = 0; r < 8; r++) {
            int i0, i1;
            qpair_index<BA>(r, i0, i1);
            const float x0 = rintf(s_q[gq][0][seg * 16 + i0] * qscale);
            const float x1 = rintf(s_q[gq][0][seg * 16 + i1] * qscale);
            QA[gq] += x0 + x1;
            qpA[gq][r] = ((uint32_t)(int)x0 & 0xFFFFu) | ((uint32_t)(int)x1 << 16);
            if (RESID) {
                qpair_index<BR>(r, i0, i1);
                const float y0 = rintf(s_q[gq][1][seg * 16 + i0] * qscale);
                const float y1 = rintf(s_q[gq][1][seg * 16 + i1] * qscale);
                QR[gq] += y0 + y1;
                qpR[gq][r] = ((uint32_t)(int)y0 & 0xFFFFu) | ((uint32_t)(int)y1 << 16);
            } else {
                qpR[gq][r] = 0;
            }
        }
    }

    // ------------------------------------------------------------ pass 1: logits
    float mloc[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) mloc[gq] = -CUDART_INF_F;
    for (int i = 0; i < ntiles; i++) {
        const int stage = i % kStages;
        const bool ok = mbar_wait(&bar_full[stage], (i / kStages) & 1, &s_abort);
        if (!ok) {
            s_abort = 1;
            atomicExch(a.err, 2);
        }
        const uint8_t *st = ring + stage * L.stage_bytes;
        float part[GK][4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const int tok = 16 * warp + sub + 4 * k;
            const Seg<BA> ca = lds_seg<BA>(st + tok * L.A_C + seg * (2 * BA));
            const float2 ma = meta_pair(*reinterpret_cast<const uint16_t *>(st + L.k_am + tok * L.MR + 2 * mgrp));
            float shat = 1.f;
            Seg<BR> cr;
            float2 mr = make_float2(0.f, 0.f);
            if (RESID) {
                cr = lds_seg<BR>(st + L.k_rc + tok * L.R_C + seg * (2 * BR));
                mr = meta_pair(*reinterpret_cast<const uint16_t *>(st + L.k_rm + tok * L.MR + 2 * mgrp));
                shat = bf16_to_f32(*reinterpret_cast<const uint16_t *>(st + L.k_cf + 2 * tok));
            }
#pragma unroll
            for (int gq = 0; gq < GK; gq++) {
                const float A = fmaf(ma.y, QA[gq], ma.x * i2f_exact(dot_seg<BA>(ca, qpA[gq])));
                float v = A;
                if (RESID) {
                    const float R = fmaf(mr.y, QR[gq], mr.x * i2f_exact(dot_seg<BR>(cr, qpR[gq])));
                    v = fmaf(shat, A, R);
                }
                part[gq][k] = v;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_empty[stage]);
        // reduce the 4 tokens' partials over the 8 segment lanes: lanes 2k, 2k+1 end with token k
        const bool b4 = (seg & 4) != 0, b2 = (seg & 2) != 0;
#pragma unroll
        for (int gq = 0; gq < GK; gq++) {
            float r0 = (b4 ? part[gq][2] : part[gq][0]) + __shfl_xor_sync(0xffffffffu, b4 ? part[gq][0] : part[gq][2], 4);
            float r1 = (b4 ? part[gq][3] : part[gq][1]) + __shfl_xor_sync(0xffffffffu, b4 ? part[gq][1] : part[gq][3], 4);
            float r = (b2 ? r1 : r0) + __shfl_xor_sync(0xffffffffu, b2 ? r0 : r1, 2);
            r += __shfl_xor_sync(0xffffffffu, r, 1);
            r *= qinv;
            const int k = (b4 ? 2 : 0) + (b2 ? 1 : 0);
            const int tl = i * kTile + 16 * warp + sub + 4 * k;
            if (tl < n && ok) {
                if ((seg & 1) == 0) s_sc[gq * a.chunk + tl] = r;
                mloc[gq] = fmaxf(mloc[gq], r);
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
    const bool vm_ok = mbar_wait(&bar_vm, 0, &s_abort);
    if (!vm_ok) {
        s_abort = 1;
        atomicExch(a.err, 3);
    }
    consumer_sync();
    float M[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++)
        M[gq] = fmaxf(fmaxf(s_red[0][gq], s_red[1][gq]), fmaxf(s_red[2][gq], s_red[3][gq]));
    consumer_sync();   // everyone has read s_red
    // p = exp2(z - M); the scores buffer is overwritten with P = p * s_hat(V);
    // bounds of |s_hat| and of every group's scale for the fixed-point V weights
    float lsum[GK];
    uint32_t cf_max = 0, sc_max_a = 0, sc_max_r = 0;   // |coef| bits, scale bytes (per group: thread's group = tid & 7)
#pragma unroll
    for (int gq = 0; gq < GK; gq++) lsum[gq] = 0.f;
    const int G8 = 128 / a.g;   // groups per record
    for (int t = tid; t < n; t += kConsumers) {
        const float shv = RESID ? bf16_to_f32(reinterpret_cast<const uint16_t *>(vm + L.vm_cf)[t]) : 1.f;
#pragma unroll
        for (int gq = 0; gq < GK; gq++) {
            const float p = exp2f(s_sc[gq * a.chunk + t] - M[gq]);
            lsum[gq] += p;
            s_sc[gq * a.chunk + t] = p;                       // residual V weight
            s_P[gq * a.chunk + t] = p * shv;                  // anchor V weight (carries s_hat)
        }
        if (RESID) cf_max = max(cf_max, (uint32_t)reinterpret_cast<const uint16_t *>(vm + L.vm_cf)[t] & 0x7FFFu);
    }
    // scale-byte maxima: thread handles group (tid % G8) of tokens tid/G8, +128/G8, ...
    {
        const int grp = tid % G8;
        for (int t = tid / G8; t < n; t += kConsumers / G8) {
            sc_max_a = max(sc_max_a, (uint32_t)vm[t * L.MR + 2 * grp]);
            if (RESID) sc_max_r = max(sc_max_r, (uint32_t)vm[L.vm_r + t * L.MR + 2 * grp]);
        }
    }
    // reduce: lsum over all; cf_max over all; scale maxima over threads with the same group
    {
#pragma unroll
        for (int gq = 0; gq < GK; gq++) {
            float v = lsum[gq];
            for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
            lsum[gq] = v;
        }
        for (int m = 16; m >= 1; m >>= 1) cf_max = max(cf_max, __shfl_xor_sync(0xffffffffu, cf_max, m));
        for (int m = 16; m >= G8; m >>= 1) {
            sc_max_a = max(sc_max_a, __shfl_xor_sync(0xffffffffu, sc_max_a, m));
            sc_max_r = max(sc_max_r, __shfl_xor_sync(0xffffffffu, sc_max_r, m));
        }
        if (lane == 0) {
#pragma unroll
            for (int gq = 0; gq < GK; gq++) s_red[warp][gq] = lsum[gq];
            s_red[warp][GK] = __uint_as_float(cf_max);
        }
        if (lane < G8) {
            s_red[warp][2 * GK + lane] = __uint_as_float(sc_max_a);
            s_red[warp][2 * GK + 8 + lane] = __uint_as_float(sc_max_r);
        }
    }
    consumer_sync();
    float Lsum[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) Lsum[gq] = s_red[0][gq] + s_red[1][gq] + s_red[2][gq] + s_red[3][gq];
    float cA, cR;   // fixed-point scales of this lane's group: anchor and residual V weights
    {
        uint32_t cfm = 0, sa = 0, sr = 0;
#pragma unroll
        for (int w = 0; w < 4; w++) {
            cfm = max(cfm, __float_as_uint(s_red[w][GK]));
            sa = max(sa, __float_as_uint(s_red[w][2 * GK + mgrp]));
            sr = max(sr, __float_as_uint(s_red[w][2 * GK + 8 + mgrp]));
        }
        const float shmax = RESID ? bf16_to_f32((uint16_t)cfm) : 1.f;
        // the bound is an exact product of a BF16 and an FP8 value (<= 12
        // significant bits), so bound * 2^F <= 2^15 - 8 and no rounded weight
        // can reach 2^15
        cA = fixed_scale(shmax * e4m3_to_f32(sa), 15);
        cR = fixed_scale(e4m3_to_f32(sr), 15);
    }

    // ------------------------------------------------------------ pass 2: values
    int accA[GK][16], accR[GK][16];
    float mA[GK], mR[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        mA[gq] = mR[gq] = 0.f;
#pragma unroll
        for (int e = 0; e < 16; e++) accA[gq][e] = accR[gq][e] = 0;
    }
    for (int i = 0; i < ntiles; i++) {
        const int it = ntiles + i;
        const int stage = it % kStages;
        if (!mbar_wait(&bar_full[stage], (it / kStages) & 1, &s_abort)) {
            s_abort = 1;
            atomicExch(a.err, 4);
        }
        const uint8_t *st = ring + stage * L.stage_bytes;
        Seg<BA> ca[4];
        Seg<BR> cr[4];
        float P[GK][4], p[GK][4];
        float2 ma[4], mr[4];
#pragma unroll
        for (int k = 0; k < 4; k++) {
            const int tok = 16 * warp + sub + 4 * k;
            const bool valid = (i * kTile + tok) < n;
            const int tl = min(i * kTile + tok, n - 1);     // weights of tokens >= n are zero
            ca[k] = lds_seg<BA>(st + tok * L.A_C + seg * (2 * BA));
            ma[k] = meta_pair(*reinterpret_cast<const uint16_t *>(vm + tl * L.MR + 2 * mgrp));
            if (RESID) {
                cr[k] = lds_seg<BR>(st + L.v_rc + tok * L.R_C + seg * (2 * BR));
                mr[k] = meta_pair(*reinterpret_cast<const uint16_t *>(vm + L.vm_r + tl * L.MR + 2 * mgrp));
            }
#pragma unroll
            for (int gq = 0; gq < GK; gq++) {
                P[gq][k] = valid ? s_P[gq * a.chunk + tl] : 0.f;
                p[gq][k] = valid ? s_sc[gq * a.chunk + tl] : 0.f;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_empty[stage]);
#pragma unroll
        for (int gq = 0; gq < GK; gq++) {
            uint32_t wa[4], wr[4];
#pragma unroll
            for (int k = 0; k < 4; k++) {
                wa[k] = fix16_bits_fma(P[gq][k] * cA, ma[k].x);
                mA[gq] = fmaf(P[gq][k], ma[k].y, mA[gq]);
            }
            acc_pair<BA>(ca[0], ca[1], __byte_perm(wa[0], wa[1], 0x5410), accA[gq]);
            acc_pair<BA>(ca[2], ca[3], __byte_perm(wa[2], wa[3], 0x5410), accA[gq]);
            if (RESID) {
#pragma unroll
                for (int k = 0; k < 4; k++) {
                    wr[k] = fix16_bits_fma(p[gq][k] * cR, mr[k].x);
                    mR[gq] = fmaf(p[gq][k], mr[k].y, mR[gq]);
                }
                acc_pair<BR>(cr[0], cr[1], __byte_perm(wr[0], wr[1], 0x5410), accR[gq]);
                acc_pair<BR>(cr[2], cr[3], __byte_perm(wr[2], wr[3], 0x5410), accR[gq]);
            }
        }
    }

    // ------------------------------------------------------------ reduce and write the partial
    const float iA = 1.f / cA, iR = 1.f / cR;
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
#pragma unroll
        for (int e = 0; e < 16; e++) {
            float va = fmaf((float)accA[gq][e], iA, mA[gq]);
            float vr = RESID ? fmaf((float)accR[gq][e], iR, mR[gq]) : 0.f;
            va += __shfl_xor_sync(0xffffffffu, va, 8);
            va += __shfl_xor_sync(0xffffffffu, va, 16);
            vr += __shfl_xor_sync(0xffffffffu, vr, 8);
            vr += __shfl_xor_sync(0xffffffffu, vr, 16);
            if (sub == 0) {
                s_acc[warp][gq][0][seg * 16 + e] = va;
                s_acc[warp][gq][1][seg * 16 + e] = vr;
            }
        }
    }
    consumer_sync();
    float oA[GK], oR[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        oA[gq] = s_acc[0][gq][0][tid] + s_acc[1][gq][0][tid] + s_acc[2][gq][0][tid] + s_acc[3][gq][0][tid];
        oR[gq] = s_acc[0][gq][1][tid] + s_acc[1][gq][1][tid] + s_acc[2][gq][1][tid] + s_acc[3][gq][1][tid];
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
        part[tid] = oA[gq] + (RESID ? oR[gq] : 0.f);
        if (tid == 0) {
            part[kHeadDim] = M[gq];
            part[kHeadDim + 1] = Lsum[gq];
        }
    }
}

template <int GK, int BA, int BR, bool RESID>
size_t smem_bytes(int g, int chunk) {
    const int A_C = 16 * BA, R_C = 16 * BR, MR = 256 / g;
    int k_bytes = kTile * (A_C + MR) + (RESID ? kTile * (R_C + MR + 2) : 0);
    int v_bytes = kTile * A_C + (RESID ? kTile * R_C : 0);
    int stage = ((std::max(k_bytes, v_bytes) + 127) / 128) * 128;
    int vm = chunk * MR + (RESID ? chunk * (MR + 2) : 0);
    return (size_t)kStages * stage + ((vm + 127) / 128) * 128 + (size_t)2 * GK * chunk * sizeof(float);
}

template <int GK, int BA, int BR, bool RESID>
cudaError_t configure() {
    static bool configured = false;   // the largest dynamic shared memory any launch can ask for
    if (configured) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(decode_rq_kernel<GK, BA, BR, RESID>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem_bytes<GK, BA, BR, RESID>(16, kMaxChunk));
    if (e == cudaSuccess) configured = true;
    return e;
}

template <int GK, int BA, int BR, bool RESID>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t st) {
    const dim3 grid(a.S, a.H, a.B * (a.G / GK));
    const size_t smem = smem_bytes<GK, BA, BR, RESID>(a.g, a.chunk);
    cudaError_t e = configure<GK, BA, BR, RESID>();
    if (e != cudaSuccess) return e;
    decode_rq_kernel<GK, BA, BR, RESID><<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

template <int GK, int BA, int BR, bool RESID>
int occupancy_t(int g, int chunk) {
    if (configure<GK, BA, BR, RESID>() != cudaSuccess) return 1;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_rq_kernel<GK, BA, BR, RESID>, kThreads,
                                                      smem_bytes<GK, BA, BR, RESID>(g, chunk)) != cudaSuccess)
        return 1;
    return n > 0 ? n : 1;
}

template <int GK>
int occupancy_g(int ba, int br, bool resid, int g, int chunk) {
    if (!resid) return ba == 4 ? occupancy_t<GK, 4, 2, false>(g, chunk) : occupancy_t<GK, 2, 2, false>(g, chunk);
    if (ba == 4 && br == 2) return occupancy_t<GK, 4, 2, true>(g, chunk);
    if (ba == 4 && br == 4) return occupancy_t<GK, 4, 4, true>(g, chunk);
    if (ba == 2 && br == 2) return occupancy_t<GK, 2, 2, true>(g, chunk);
    return occupancy_t<GK, 2, 4, true>(g, chunk);
}

template <int GK>
cudaError_t launch_g(const DecodeArgs &a, int ba, int br, bool resid, cudaStream_t st) {
    if (!resid) return ba == 4 ? launch_t<GK, 4, 2, false>(a, st) : launch_t<GK, 2, 2, false>(a, st);
    if (ba == 4 && br == 2) return launch_t<GK, 4, 2, true>(a, st);
    if (ba == 4 && br == 4) return launch_t<GK, 4, 4, true>(a, st);
    if (ba == 2 && br == 2) return launch_t<GK, 2, 2, true>(a, st);
    return launch_t<GK, 2, 4, true>(a, st);
}

}  // namespace

cudaError_t launch_decode_rq(const DecodeArgs &a, int ba, int br, bool resid, cudaStream_t st) {
    if (a.G == 1) return launch_g<1>(a, ba, br, resid, st);
    return launch_g<2>(a, ba, br, resid, st);   // G = 2, 4, 8: pairs of query heads
}

int decode_rq_occupancy(int G, int ba, int br, bool resid, int g, int chunk) {
    return G == 1 ? occupancy_g<1>(ba, br, resid, g, chunk) : occupancy_g<2>(ba, br, resid, g, chunk);
}

}  // namespace rq
