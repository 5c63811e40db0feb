// combine.cuh -- merging split-KV partials (max m_s, sum l_s, unnormalised
// o_s, log2 domain) and BF16 tail tokens into one attention output row:
//   o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s
// with the tail tokens folded in one by one by the same rescaling rule.
#pragma once

#include <math_constants.h>

#include "common.cuh"
#include "rq_internal.h"

namespace rq {

// Run by 128 threads (thread `tid` owns element tid of the row).  `sync` is a
// barrier over exactly those threads; `red` is 4 floats of shared memory.
// `part` points at slot 0 of this row's partials (stride kPartialStride); it
// is read with L1-bypassing loads because other CTAs wrote it.
template <typename Sync>
__device__ __forceinline__ void combine_row(const float *part, int S, const uint16_t *q_row, float scale_log2,
                                            const uint16_t *tail_k, const uint16_t *tail_v, size_t tail_stride,
                                            int n_tail, float *out_row, int tid, float *red, Sync sync) {
    const int lane = tid & 31, warp = tid >> 5;
    float M = -CUDART_INF_F, l = 0.f, o = 0.f;
    for (int s = 0; s < S; s++) {
        const float *p = part + (size_t)s * kPartialStride;
        const float ms = __ldcg(p + kHeadDim), ls = __ldcg(p + kHeadDim + 1), os = __ldcg(p + tid);
        const float nm = fmaxf(M, ms);
        const float c0 = exp2f(M - nm), c1 = exp2f(ms - nm);
        o = o * c0 + os * c1;
        l = l * c0 + ls * c1;
        M = nm;
    }
    if (n_tail > 0) {
        const float q = bf16_to_f32(q_row[tid]) * scale_log2;
        for (int j = 0; j < n_tail; j++) {
            const size_t row = (size_t)j * tail_stride;
            float z = q * bf16_to_f32(tail_k[row + tid]);
            for (int m = 16; m >= 1; m >>= 1) z += __shfl_xor_sync(0xffffffffu, z, m);
            sync();
            if (lane == 0) red[warp] = z;
            sync();
            z = red[0] + red[1] + red[2] + red[3];
            const float nm = fmaxf(M, z);
            const float c0 = exp2f(M - nm), c1 = exp2f(z - nm);
            o = o * c0 + bf16_to_f32(tail_v[row + tid]) * c1;
            l = l * c0 + c1;
            M = nm;
        }
    }
    out_row[tid] = (l > 0.f) ? o / l : 0.f;
}

}  // namespace rq
