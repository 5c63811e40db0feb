// combine.cuh -- merging split-KV partials (max m_s, sum l_s, unnormalised
// o_s, log2 domain) and BF16 tail tokens into one attention output row:
//   o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s
// with M = max_s m_s (kept as a running maximum over batches of splits),
// then the tail tokens folded in one by one by the same rule.
#pragma once

#include <math_constants.h>

#include "common.cuh"
#include "rq_internal.h"

namespace rq {

// The split partials of a row merged into (M, l, o) for element tid:
// kBatch splits per round of loads (one round for up to kBatch splits), the
// batch's maximum, the running sums rescaled to it, then the batch folded in
// (a split with no key has m = -inf: weight 0).  `part` points at slot 0 of
// the row's partials (stride kPartialStride); it is read with L1-bypassing
// loads because other CTAs wrote it.
__device__ __forceinline__ void merge_partials(const float *part, int S, int tid, float &M, float &l, float &o) {
    constexpr int kBatch = 16;
    M = -CUDART_INF_F;
    l = 0.f;
    o = 0.f;
    for (int s0 = 0; s0 < S; s0 += kBatch) {
        float m[kBatch], ls[kBatch], os[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; u++) {
            const bool in = s0 + u < S;
            const float *p = part + (size_t)(s0 + u) * kPartialStride;
            m[u] = in ? __ldcg(p + kHeadDim) : -CUDART_INF_F;
            ls[u] = in ? __ldcg(p + kHeadDim + 1) : 0.f;
            os[u] = in ? __ldcg(p + tid) : 0.f;
        }
        float Mn = M;
#pragma unroll
        for (int u = 0; u < kBatch; u++) Mn = fmaxf(Mn, m[u]);
        if (Mn == -CUDART_INF_F) continue;   // nothing attended yet
        const float c0 = exp2f(M - Mn);      // 0 while M = -inf
        l *= c0;
        o *= c0;
#pragma unroll
        for (int u = 0; u < kBatch; u++) {
            const float c = m[u] == -CUDART_INF_F ? 0.f : exp2f(m[u] - Mn);
            l = fmaf(ls[u], c, l);
            o = fmaf(os[u], c, o);
        }
        M = Mn;
    }
}

// Run by 128 threads (thread `tid` owns element tid of the row).  `sync` is a
// barrier over exactly those threads; `red` is 4 floats of shared memory.
template <typename Sync>
__device__ __forceinline__ void combine_row(const float *part, int S, const uint16_t *q_row, float scale_log2,
                                            const uint16_t *tail_k, const uint16_t *tail_v, size_t tail_stride,
                                            int n_tail, float *out_row, int tid, float *red, Sync sync) {
    const int lane = tid & 31, warp = tid >> 5;
    // q and the first tail token are fetched first, so that their latency
    // overlaps the partials' (L2 loads: the tail rows may have been written
    // during this kernel by another CTA)
    float q = 0.f, k0 = 0.f, v0 = 0.f;
    if (n_tail > 0) {
        q = bf16_to_f32(q_row[tid]) * scale_log2;
        k0 = bf16_to_f32(__ldcg(tail_k + tid));
        v0 = bf16_to_f32(__ldcg(tail_v + tid));
    }
    float M, l, o;
    merge_partials(part, S, tid, M, l, o);
    // tail tokens, folded in one by one with the running-max rule
    for (int j = 0; j < n_tail; j++) {
        const size_t row = (size_t)j * tail_stride;
        const float kj = j == 0 ? k0 : bf16_to_f32(__ldcg(tail_k + row + tid));
        const float vj = j == 0 ? v0 : bf16_to_f32(__ldcg(tail_v + row + tid));
        float z = q * kj;
        for (int m = 16; m >= 1; m >>= 1) z += __shfl_xor_sync(0xffffffffu, z, m);
        sync();
        if (lane == 0) red[warp] = z;
        sync();
        z = red[0] + red[1] + red[2] + red[3];
        const float nm = fmaxf(M, z);
        const float c0 = exp2f(M - nm), c1 = exp2f(z - nm);
        o = o * c0 + vj * c1;
        l = l * c0 + c1;
        M = nm;
    }
    out_row[tid] = (l > 0.f) ? o / l : 0.f;
}

}  // namespace rq
