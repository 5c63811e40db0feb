// decode_rq.cu -- split-KV decode attention over the ResidualQuant cache
// (arXiv 2610.10381; ai4snews summary, paragraph 3: shared-anchor
// reconstruction needs two cache reads -- the anchor record and the loop's
// own residual record).
//
// For a committed token t of a non-anchor loop,
//   k_t = s_t * a_t + R^T y_t      (a_t anchor, y_t rotated residual)
// so the logit factors as  q.k_t = s_t (q.a_t) + (R q).y_t : q is rotated once
// per CTA instead of rotating every key.  Per 16-element segment of a
// quantization group (scale sc, minimum mn, codes c):
//   q_seg . x_hat_seg = mn * sum(q_seg) + sc * sum(q_i c_i)
// The V side accumulates the anchor part in the original basis and the
// residual part in the rotated basis; R^T is applied once per CTA.
//
// Each CTA owns a chunk of one (sequence, kv head): pass 1 computes all the
// chunk's logits (K records), pass 2 the softmax-weighted V sum with weights
// exp2(z - chunk max) <= 1.  Partial (max, sum, o) triples are merged with the
// BF16 tail tokens by the combine kernel.
//
// Thread map: 4 warps; in a warp, lanes 8s..8s+7 ("sub-group" s) work on one
// token, lane 8s+j on head_dim elements 16j..16j+15.
#include <math_constants.h>

#include "common.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

constexpr float kRsqrt128 = 0.088388347648318440f;

// 16 codes of `BITS` bits from one segment (BITS=4: 8 bytes, BITS=2: 4 bytes).
template <int BITS>
__device__ __forceinline__ uint2 load_seg(const uint8_t *p) {
    if (BITS == 4) return __ldg(reinterpret_cast<const uint2 *>(p));
    return make_uint2(__ldg(reinterpret_cast<const uint32_t *>(p)), 0u);
}

template <int BITS>
__device__ __forceinline__ float code_at(uint2 w, int i) {
    if (BITS == 4) return (float)(((i < 8 ? w.x : w.y) >> (4 * (i & 7))) & 0xFu);
    return (float)((w.x >> (2 * i)) & 0x3u);
}

template <int BITS>
__device__ __forceinline__ float dot16(const float q[16], uint2 w) {
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 16; i++) acc = fmaf(q[i], code_at<BITS>(w, i), acc);
    return acc;
}

template <int GK, int BA, int BR, bool RESID>
__global__ void __launch_bounds__(128) decode_rq_kernel(const DecodeArgs a) {
    extern __shared__ float s_scores[];                // [GK][chunk]
    __shared__ float s_q[GK][kHeadDim];
    __shared__ float s_qr[GK][kHeadDim];
    __shared__ float s_red[4][GK];
    __shared__ float s_acc[4][GK][2][kHeadDim];

    const int split = blockIdx.x, h = blockIdx.y;
    const int npairs = a.G / GK;
    const int b = blockIdx.z / npairs, pair = blockIdx.z % npairs;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, sub = lane >> 3, seg = lane & 7;
    const int hq0 = h * a.G + pair * GK;
    const int t0 = split * a.chunk;
    const int n = min(a.chunk, a.T - t0);
    const size_t bh = (size_t)b * a.H + h;
    const int meta_rec = 2 * (kHeadDim / a.g);
    const int mgrp = (seg * 16) / a.g;                  // quantization group of this segment

    // ---- q (log2-domain scale folded in) and R q
#pragma unroll
    for (int gq = 0; gq < GK; gq++)
        s_q[gq][tid] = bf16_to_f32(a.q[((size_t)b * a.Hq + hq0 + gq) * kHeadDim + tid]) * a.scale_log2;
    __syncthreads();
    if (RESID) {
        for (int gq = warp; gq < GK; gq += 4) {
            float v[4];
#pragma unroll
            for (int k = 0; k < 4; k++) {
                v[k] = s_q[gq][4 * lane + k];
                if (a.rotate && sigma_neg(a.sigma, 4 * lane + k)) v[k] = -v[k];
            }
            if (a.rotate) {
                wht128_warp<float>(v, lane);
#pragma unroll
                for (int k = 0; k < 4; k++) v[k] *= kRsqrt128;
            }
#pragma unroll
            for (int k = 0; k < 4; k++) s_qr[gq][4 * lane + k] = v[k];
        }
    }
    __syncthreads();
    float qa[GK][16], qr[GK][16], Qa[GK], Qr[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        Qa[gq] = 0.f;
        Qr[gq] = 0.f;
#pragma unroll
        for (int i = 0; i < 16; i++) {
            qa[gq][i] = s_q[gq][seg * 16 + i];
            Qa[gq] += qa[gq][i];
            qr[gq][i] = RESID ? s_qr[gq][seg * 16 + i] : 0.f;
            Qr[gq] += qr[gq][i];
        }
    }

    // ---- pass 1: logits
    float mloc[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) mloc[gq] = -CUDART_INF_F;
    for (int it = warp * 4; it < n; it += 16) {
        const int tl = it + sub;
        const bool valid = tl < n;
        const size_t rec = bh * a.Tp + (size_t)min(t0 + tl, a.T - 1);   // loads stay on committed tokens
        const uint2 ca = load_seg<BA>(a.a_codes[0] + rec * (16 * BA) + seg * (2 * BA));
        const uint32_t ma = __ldg(reinterpret_cast<const uint16_t *>(a.a_meta[0] + rec * meta_rec) + mgrp);
        const float sa = e4m3_to_f32(ma & 0xFF), mna = e4m3_to_f32(ma >> 8);
        float part[GK];
#pragma unroll
        for (int gq = 0; gq < GK; gq++) part[gq] = fmaf(mna, Qa[gq], sa * dot16<BA>(qa[gq], ca));
        if (RESID) {
            const uint2 cr = load_seg<BR>(a.r_codes[0] + rec * (16 * BR) + seg * (2 * BR));
            const uint32_t mr = __ldg(reinterpret_cast<const uint16_t *>(a.r_meta[0] + rec * meta_rec) + mgrp);
            const float sr = e4m3_to_f32(mr & 0xFF), mnr = e4m3_to_f32(mr >> 8);
            const float shat = bf16_to_f32(__ldg(a.r_coef[0] + rec));
#pragma unroll
            for (int gq = 0; gq < GK; gq++)
                part[gq] = fmaf(shat, part[gq], fmaf(mnr, Qr[gq], sr * dot16<BR>(qr[gq], cr)));
        }
#pragma unroll
        for (int gq = 0; gq < GK; gq++) {
            float v = part[gq];
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            v += __shfl_xor_sync(0xffffffffu, v, 4);
            if (valid) {
                if (seg == 0) s_scores[gq * a.chunk + tl] = v;
                mloc[gq] = fmaxf(mloc[gq], v);
            }
        }
    }
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        float v = mloc[gq];
        for (int m = 16; m >= 1; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
        if (lane == 0) s_red[warp][gq] = v;
    }
    __syncthreads();
    float M[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++)
        M[gq] = fmaxf(fmaxf(s_red[0][gq], s_red[1][gq]), fmaxf(s_red[2][gq], s_red[3][gq]));

    // ---- pass 2: values
    float accA[GK][16], accR[GK][16], mA[GK], mR[GK], lsum[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        mA[gq] = mR[gq] = lsum[gq] = 0.f;
#pragma unroll
        for (int i = 0; i < 16; i++) accA[gq][i] = accR[gq][i] = 0.f;
    }
    for (int it = warp * 4; it < n; it += 16) {
        const int tl = it + sub;
        const bool valid = tl < n;
        const size_t rec = bh * a.Tp + (size_t)min(t0 + tl, a.T - 1);
        float p[GK];
#pragma unroll
        for (int gq = 0; gq < GK; gq++) p[gq] = valid ? exp2f(s_scores[gq * a.chunk + tl] - M[gq]) : 0.f;
        const uint2 ca = load_seg<BA>(a.a_codes[1] + rec * (16 * BA) + seg * (2 * BA));
        const uint32_t ma = __ldg(reinterpret_cast<const uint16_t *>(a.a_meta[1] + rec * meta_rec) + mgrp);
        const float sa = e4m3_to_f32(ma & 0xFF), mna = e4m3_to_f32(ma >> 8);
        const float shat = RESID ? bf16_to_f32(__ldg(a.r_coef[1] + rec)) : 1.f;
#pragma unroll
        for (int gq = 0; gq < GK; gq++) {
            const float w = p[gq] * shat;
            const float ws = w * sa;
#pragma unroll
            for (int i = 0; i < 16; i++) accA[gq][i] = fmaf(ws, code_at<BA>(ca, i), accA[gq][i]);
            mA[gq] = fmaf(w, mna, mA[gq]);
            lsum[gq] += p[gq];
        }
        if (RESID) {
            const uint2 cr = load_seg<BR>(a.r_codes[1] + rec * (16 * BR) + seg * (2 * BR));
            const uint32_t mr = __ldg(reinterpret_cast<const uint16_t *>(a.r_meta[1] + rec * meta_rec) + mgrp);
            const float sr = e4m3_to_f32(mr & 0xFF), mnr = e4m3_to_f32(mr >> 8);
#pragma unroll
            for (int gq = 0; gq < GK; gq++) {
                const float ws = p[gq] * sr;
#pragma unroll
                for (int i = 0; i < 16; i++) accR[gq][i] = fmaf(ws, code_at<BR>(cr, i), accR[gq][i]);
                mR[gq] = fmaf(p[gq], mnr, mR[gq]);
            }
        }
    }
    // ---- reduce: sub-groups (lanes xor 8, 16), then warps through shared memory
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
#pragma unroll
        for (int i = 0; i < 16; i++) {
            float va = accA[gq][i] + mA[gq];
            float vr = accR[gq][i] + mR[gq];
            va += __shfl_xor_sync(0xffffffffu, va, 8);
            va += __shfl_xor_sync(0xffffffffu, va, 16);
            vr += __shfl_xor_sync(0xffffffffu, vr, 8);
            vr += __shfl_xor_sync(0xffffffffu, vr, 16);
            if (sub == 0) {
                s_acc[warp][gq][0][seg * 16 + i] = va;
                s_acc[warp][gq][1][seg * 16 + i] = vr;
            }
        }
        float l = lsum[gq];
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        if (lane == 0) s_red[warp][gq] = l;
    }
    __syncthreads();
    float oA[GK], oR[GK], L[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        oA[gq] = s_acc[0][gq][0][tid] + s_acc[1][gq][0][tid] + s_acc[2][gq][0][tid] + s_acc[3][gq][0][tid];
        oR[gq] = s_acc[0][gq][1][tid] + s_acc[1][gq][1][tid] + s_acc[2][gq][1][tid] + s_acc[3][gq][1][tid];
        L[gq] = s_red[0][gq] + s_red[1][gq] + s_red[2][gq] + s_red[3][gq];
    }
    if (RESID && a.rotate) {
        // o += R^T o_rot = sigma . (H o_rot) / sqrt(d)
#pragma unroll
        for (int gq = 0; gq < GK; gq++) s_qr[gq][tid] = oR[gq];
        __syncthreads();
        for (int gq = warp; gq < GK; gq += 4) {
            float v[4];
#pragma unroll
            for (int k = 0; k < 4; k++) v[k] = s_qr[gq][4 * lane + k];
            wht128_warp<float>(v, lane);
#pragma unroll
            for (int k = 0; k < 4; k++) {
                float r = v[k] * kRsqrt128;
                if (sigma_neg(a.sigma, 4 * lane + k)) r = -r;
                s_qr[gq][4 * lane + k] = r;
            }
        }
        __syncthreads();
#pragma unroll
        for (int gq = 0; gq < GK; gq++) oR[gq] = s_qr[gq][tid];
    }
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        float *part = a.partials + (((size_t)b * a.Hq + hq0 + gq) * a.splits_max + split) * kPartialStride;
        part[tid] = oA[gq] + (RESID ? oR[gq] : 0.f);
        if (tid == 0) {
            part[kHeadDim] = M[gq];
            part[kHeadDim + 1] = L[gq];
        }
    }
}

template <int GK, int BA, int BR, bool RESID>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t st) {
    const dim3 grid(a.S, a.H, a.B * (a.G / GK));
    const size_t smem = (size_t)GK * a.chunk * sizeof(float);
    auto kern = decode_rq_kernel<GK, BA, BR, RESID>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    kern<<<grid, 128, smem, st>>>(a);
    return cudaGetLastError();
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

}  // namespace rq
