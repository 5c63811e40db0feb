// decode_bf16.cu -- uncompressed split-KV decode attention over a BF16 cache:
// the comparison kernel (the role BF16 FlashAttention decode plays in the
// ResidualQuant throughput study, ai4snews summary, paragraph 4), and the
// split-combine kernel shared by both decode paths.
//
// Same CTA structure as the compressed kernel: a CTA owns a chunk of one
// (sequence, kv head); pass 1 writes the chunk's logits, pass 2 sums
// exp2(z - chunk max) * v; the combine kernel merges the partials and the
// BF16 tail tokens.
#include <math_constants.h>

#include "combine.cuh"
#include "common.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

__device__ __forceinline__ void load16_bf16(const uint16_t *p, float v[16]) {
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint4 b = __ldg(reinterpret_cast<const uint4 *>(p) + 1);
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int k = 0; k < 8; k++) {
        v[2 * k] = __uint_as_float(w[k] << 16);
        v[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
    }
}

template <int GK>
__global__ void __launch_bounds__(128) decode_bf16_kernel(const DecodeArgs a) {
    extern __shared__ float s_scores[];   // [GK][chunk]
    __shared__ float s_q[GK][kHeadDim];
    __shared__ float s_red[4][GK], s_lsum[4][GK];
    __shared__ float s_acc[4][GK][kHeadDim];

    const int split = blockIdx.x, h = blockIdx.y;
    const int npairs = a.G / GK;
    const int b = blockIdx.z / npairs, pair = blockIdx.z % npairs;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, sub = lane >> 3, seg = lane & 7;
    const int hq0 = h * a.G + pair * GK;
    const int Tb = a.seqT.v[b];   // this sequence's committed tokens
    int t0, n;
    split_range(split, a.S, Tb, &t0, &n);
    const size_t bh = (size_t)b * a.H + h;

#pragma unroll
    for (int gq = 0; gq < GK; gq++)
        s_q[gq][tid] = bf16_to_f32(a.q[((size_t)b * a.Hq + hq0 + gq) * kHeadDim + tid]) * a.scale_log2;
    __syncthreads();
    float qa[GK][16];
#pragma unroll
    for (int gq = 0; gq < GK; gq++)
#pragma unroll
        for (int i = 0; i < 16; i++) qa[gq][i] = s_q[gq][seg * 16 + i];

    float mloc[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) mloc[gq] = -CUDART_INF_F;
    for (int it = warp * 4; it < n; it += 16) {
        const int tl = it + sub;
        const bool valid = tl < n;
        const size_t rec = bh * a.Tp + (size_t)min(t0 + tl, Tb - 1);
        float k[16];
        load16_bf16(a.bf[0] + rec * kHeadDim + seg * 16, k);
#pragma unroll
        for (int gq = 0; gq < GK; gq++) {
            float v = 0.f;
#pragma unroll
            for (int i = 0; i < 16; i++) v = fmaf(qa[gq][i], k[i], v);
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

    float acc[GK][16], lsum[GK];
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        lsum[gq] = 0.f;
#pragma unroll
        for (int i = 0; i < 16; i++) acc[gq][i] = 0.f;
    }
    for (int it = warp * 4; it < n; it += 16) {
        const int tl = it + sub;
        const bool valid = tl < n;
        const size_t rec = bh * a.Tp + (size_t)min(t0 + tl, Tb - 1);
        float v[16];
        load16_bf16(a.bf[1] + rec * kHeadDim + seg * 16, v);
#pragma unroll
        for (int gq = 0; gq < GK; gq++) {
            const float p = valid ? exp2f(s_scores[gq * a.chunk + tl] - M[gq]) : 0.f;
#pragma unroll
            for (int i = 0; i < 16; i++) acc[gq][i] = fmaf(p, v[i], acc[gq][i]);
            lsum[gq] += p;
        }
    }
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
#pragma unroll
        for (int i = 0; i < 16; i++) {
            float x = acc[gq][i];
            x += __shfl_xor_sync(0xffffffffu, x, 8);
            x += __shfl_xor_sync(0xffffffffu, x, 16);
            if (sub == 0) s_acc[warp][gq][seg * 16 + i] = x;
        }
        float l = lsum[gq];
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        if (lane == 0) s_lsum[warp][gq] = l;
    }
    __syncthreads();
#pragma unroll
    for (int gq = 0; gq < GK; gq++) {
        float *part = a.partials + (((size_t)b * a.Hq + hq0 + gq) * a.splits_max + split) * kPartialStride;
        part[tid] = s_acc[0][gq][tid] + s_acc[1][gq][tid] + s_acc[2][gq][tid] + s_acc[3][gq][tid];
        if (tid == 0) {
            part[kHeadDim] = M[gq];
            part[kHeadDim + 1] = s_lsum[0][gq] + s_lsum[1][gq] + s_lsum[2][gq] + s_lsum[3][gq];
        }
    }
}

struct BlockSync {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

// One CTA per (sequence, query head): merges the split partials and the BF16
// tail tokens (combine_row) and writes o / l (zero when nothing was attended).
__global__ void __launch_bounds__(128) combine_kernel(const CombineArgs a) {
    __shared__ float s_red[4];
    const int hq = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    const int h = hq / a.G;
    const size_t row = (size_t)b * a.Hq + hq;
    const size_t trow = ((size_t)b * a.tail_cap * a.H + h) * kHeadDim;
    combine_row(a.partials + row * a.splits_max * kPartialStride, a.S, a.q + row * kHeadDim, a.scale_log2,
                a.tail_k ? a.tail_k + trow : nullptr, a.tail_v ? a.tail_v + trow : nullptr, (size_t)a.H * kHeadDim,
                a.n_tail, a.out + row * kHeadDim, tid, s_red, BlockSync());
}

}  // namespace

cudaError_t launch_decode_bf16(const DecodeArgs &a, cudaStream_t st) {
    const size_t smem_g1 = (size_t)a.chunk * sizeof(float);
    if (a.G == 1) {
        decode_bf16_kernel<1><<<dim3(a.S, a.H, a.B), 128, smem_g1, st>>>(a);
    } else {
        decode_bf16_kernel<2><<<dim3(a.S, a.H, a.B * (a.G / 2)), 128, 2 * smem_g1, st>>>(a);
    }
    return cudaGetLastError();
}

int decode_bf16_occupancy(int G, int chunk) {
    int n = 0;
    const size_t smem = (size_t)chunk * sizeof(float) * (G == 1 ? 1 : 2);
    cudaError_t e = G == 1 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_bf16_kernel<1>, 128, smem)
                           : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_bf16_kernel<2>, 128, smem);
    return (e == cudaSuccess && n > 0) ? n : 1;
}

cudaError_t launch_combine(const CombineArgs &a, cudaStream_t st) {
    combine_kernel<<<dim3(a.Hq, a.B), 128, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace rq
