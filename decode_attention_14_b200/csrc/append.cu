// append.cu -- builds the compressed cache format for tokens whose final
// loop has finished (ResidualQuant, arXiv 2610.10381; ai4snews summary,
// paragraph 1: final-loop anchor, least-squares scaling, rotation applied
// to the residuals only, INT4 anchor / INT2 residuals; paragraph 2: group
// size 16 with FP8 scales and offsets, BF16 least-squares coefficients).
//
// One warp encodes one record (the anchor or one loop's residual) of one
// (K|V, sequence, token, kv head): lane l holds the four head_dim elements
// 4l..4l+3.  Every encoding decision (group min/max, the
// scale and minimum before their FP8 rounding, the code quotient, the
// least-squares coefficient before its BF16 rounding, the rotated residual)
// is computed in fp64, so the integer codes come out the same as from an
// fp64 statement of the method except where a value sits on a rounding
// boundary to within fp64 rounding.  The rotation is an in-register fast
// Walsh-Hadamard transform (2 in-lane stages + 5 shuffle stages).
#include "common.cuh"
#include "rq_internal.h"

namespace rq {
namespace {

constexpr double kInvSqrt128 = 0.08838834764831845;   // 1/sqrt(128), correctly rounded

// Grouped asymmetric quantizer on the 4 values of this lane; the group spans
// g/4 consecutive lanes.  Returns the packed codes of the 4 elements
// (element k at bits k*bits), the dequantized values, and the FP8 bytes.
__device__ __forceinline__ uint32_t quantize4(const double x[4], int bits, int g, int lane, double deq[4],
                                              uint32_t *s8_out, uint32_t *m8_out) {
    const int qmax = (1 << bits) - 1;
    double mn = fmin(fmin(x[0], x[1]), fmin(x[2], x[3]));
    double mx = fmax(fmax(x[0], x[1]), fmax(x[2], x[3]));
    for (int m = 1; m < g / 4; m <<= 1) {
        mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, m));
        mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, m));
    }
    const double sig = __ddiv_rn(__dsub_rn(mx, mn), (double)qmax);
    const uint32_t s8 = f64_to_e4m3(sig);
    const uint32_t m8 = f64_to_e4m3(mn == 0.0 ? 0.0 : mn);   // a zero minimum is stored as +0
    const double sv = e4m3_to_f64(s8), mv = e4m3_to_f64(m8);
    uint32_t packed = 0;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        int c = 0;
        if (sv != 0.0) {
            double u = rint(__ddiv_rn(__dsub_rn(x[k], mv), sv));
            u = fmin(fmax(u, 0.0), (double)qmax);
            c = (int)u;
        }
        deq[k] = __dadd_rn(mv, __dmul_rn((double)c, sv));   // exact
        packed |= (uint32_t)c << (k * bits);
    }
    *s8_out = s8;
    *m8_out = m8;
    return packed;
}

__device__ __forceinline__ void store_record(uint8_t *codes, uint8_t *meta, uint32_t packed, uint32_t s8,
                                             uint32_t m8, int bits, int g, int lane) {
    if (bits == 4)
        reinterpret_cast<uint16_t *>(codes)[lane] = (uint16_t)packed;   // elements 4l..4l+3 = bytes 2l, 2l+1
    else
        codes[lane] = (uint8_t)packed;                                   // elements 4l..4l+3 = byte l
    const int lanes_per_group = g / 4;
    if ((lane % lanes_per_group) == 0) {
        const int grp = lane / lanes_per_group;
        reinterpret_cast<uint16_t *>(meta)[grp] = (uint16_t)(s8 | (m8 << 8));
    }
}

// Raise the stream's largest V scale byte (FP8 E4M3 scales are never
// negative, and for non-negative E4M3 values the byte order is the value
// order) to the record's largest.
__device__ __forceinline__ void raise_vmax(int *slot, uint32_t s8, int lane) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, s8);
    if (lane == 0) atomicMax(slot, (int)m);
}

__device__ __forceinline__ void load4_bf16(const uint16_t *p, double x[4]) {
    const uint2 raw = *reinterpret_cast<const uint2 *>(p);
    x[0] = (double)bf16_to_f32((uint16_t)(raw.x & 0xFFFF));
    x[1] = (double)bf16_to_f32((uint16_t)(raw.x >> 16));
    x[2] = (double)bf16_to_f32((uint16_t)(raw.y & 0xFFFF));
    x[3] = (double)bf16_to_f32((uint16_t)(raw.y >> 16));
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, m));
    return v;
}

// The residual record j of one token-head against the reference ref (the
// dequantized anchor, or in the chained reference the previous loop's
// reconstruction): coefficient s (least squares <x, ref>/<ref, ref>, norm
// ratio |x|/|ref|, or 1; 0 when ref = 0 in the first two), stored in BF16;
// residual x - s_hat ref with the stored coefficient; y = R r =
// H (sigma . r) / sqrt(d); y quantized at resid_bits.  If next != nullptr it
// receives the reconstruction s_hat ref + R^T y_hat.
__device__ __forceinline__ void encode_residual(const AppendArgs &a, const double xl[4], const double ref[4],
                                                int j, int kv, int b, int h, size_t rec, int lane,
                                                double next[4]) {
    double rr = 0.0, xr = 0.0, xx = 0.0;
#pragma unroll
    for (int k = 0; k < 4; k++) {
        rr = __dadd_rn(rr, __dmul_rn(ref[k], ref[k]));
        xr = __dadd_rn(xr, __dmul_rn(xl[k], ref[k]));
        xx = __dadd_rn(xx, __dmul_rn(xl[k], xl[k]));
    }
    const double den = warp_sum(rr);
    const double num = warp_sum(xr);
    double s;
    if (a.scale_mode == 2) {
        s = 1.0;
    } else if (den == 0.0) {
        s = 0.0;
    } else if (a.scale_mode == 0) {
        s = __ddiv_rn(num, den);
    } else {
        s = __ddiv_rn(__dsqrt_rn(warp_sum(xx)), __dsqrt_rn(den));
    }
    const __nv_bfloat16 sb = __double2bfloat16(s);
    const double sh = (double)__bfloat162float(sb);
    double y[4];
#pragma unroll
    for (int k = 0; k < 4; k++) {
        double r = __dsub_rn(xl[k], __dmul_rn(sh, ref[k]));
        if (a.rotate && sigma_neg(a.sigma, lane * 4 + k)) r = -r;
        y[k] = r;
    }
    if (a.rotate) {
        wht128_warp<double>(y, lane);
#pragma unroll
        for (int k = 0; k < 4; k++) y[k] = __dmul_rn(y[k], kInvSqrt128);
    }
    double yhat[4];
    uint32_t s8, m8;
    const uint32_t rpack = quantize4(y, a.br, a.g, lane, yhat, &s8, &m8);
    const int meta_rec = 2 * (kHeadDim / a.g);
    uint8_t *rc = a.r_codes0 + j * a.resid_loop_stride + kv * a.resid_kv_stride + rec * (kHeadDim * a.br / 8);
    uint8_t *rm = a.r_meta0 + j * a.resid_loop_stride + kv * a.resid_kv_stride + rec * meta_rec;
    store_record(rc, rm, rpack, s8, m8, a.br, a.g, lane);
    if (kv == 1) raise_vmax(a.vmax + ((size_t)j * a.B + b) * a.H + h, s8, lane);
    if (lane == 0) {
        uint16_t *rf = reinterpret_cast<uint16_t *>(a.r_coef0 + j * a.resid_loop_stride + kv * a.resid_kv_stride);
        rf[rec] = __bfloat16_as_ushort(sb);
    }
    if (next) {
        // R^T y_hat = sigma . (H y_hat) / sqrt(d), then s_hat ref + that
        double back[4] = {yhat[0], yhat[1], yhat[2], yhat[3]};
        if (a.rotate) {
            wht128_warp<double>(back, lane);
#pragma unroll
            for (int k = 0; k < 4; k++) {
                back[k] = __dmul_rn(back[k], kInvSqrt128);
                if (sigma_neg(a.sigma, lane * 4 + k)) back[k] = -back[k];
            }
        }
#pragma unroll
        for (int k = 0; k < 4; k++) next[k] = __dadd_rn(__dmul_rn(sh, ref[k]), back[k]);
    }
}

// One warp per record: (K|V, sequence, token, kv head, j), j < nres the
// residual of loop j, j == nres the anchor.  Every warp re-derives the anchor
// (a few fp64 operations) so that the records of one token are encoded in
// parallel rather than one after another.
__global__ void __launch_bounds__(128) append_kernel(const AppendArgs a) {
    const int lane = threadIdx.x & 31;
    const long long wid = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
    const int nrec = a.nres + 1;
    const long long total = 2LL * a.B * a.n * a.H * nrec;
    if (wid >= total) return;   // uniform per warp
    const int j = (int)(wid % nrec);
    long long r = wid / nrec;
    const int h = (int)(r % a.H);
    r /= a.H;
    const int t = (int)(r % a.n);
    r /= a.n;
    const int b = (int)(r % a.B);
    const int kv = (int)(r / a.B);

    // anchor = last loop of the group, original basis (never rotated)
    double x[4], ahat[4];
    load4_bf16(a.x_anchor[kv] + (((size_t)b * a.n + t) * a.H + h) * kHeadDim + lane * 4, x);
    uint32_t s8, m8;
    const uint32_t apack = quantize4(x, a.ba, a.g, lane, ahat, &s8, &m8);
    const size_t rec = rec_row(a.pg, a.H, b, h, a.pos0.v[b] + t);
    const int meta_rec = 2 * (kHeadDim / a.g);
    if (j == a.nres) {
        uint8_t *ac = a.a_codes0 + kv * a.anchor_kv_stride + rec * (kHeadDim * a.ba / 8);
        uint8_t *am = a.a_meta0 + kv * a.anchor_kv_stride + rec * meta_rec;
        store_record(ac, am, apack, s8, m8, a.ba, a.g, lane);
        if (kv == 1) raise_vmax(a.vmax + ((size_t)a.nres * a.B + b) * a.H + h, s8, lane);
        return;
    }

    const uint16_t *tail = reinterpret_cast<const uint16_t *>(a.tail0 + j * a.tail_loop_stride +
                                                               kv * a.tail_kv_stride);
    double xl[4];
    load4_bf16(tail + (((size_t)b * a.tail_cap + t) * a.H + h) * kHeadDim + lane * 4, xl);
    encode_residual(a, xl, ahat, j, kv, b, h, rec, lane, nullptr);
}

// One token-head's records in the chained (previous-loop) reference: loop 0
// is quantized at anchor_bits into the anchor record; loop l >= 1 is encoded
// as a residual (record l - 1) against the reconstruction of loop l - 1,
// which then becomes the reference of loop l + 1.  One warp per (K|V,
// sequence, token, kv head): the chain is sequential.
__global__ void __launch_bounds__(128) append_chain_kernel(const AppendArgs a) {
    const int lane = threadIdx.x & 31;
    const long long wid = (long long)blockIdx.x * 4 + (threadIdx.x >> 5);
    const long long total = 2LL * a.B * a.n * a.H;
    if (wid >= total) return;   // uniform per warp
    long long r = wid;
    const int h = (int)(r % a.H);
    r /= a.H;
    const int t = (int)(r % a.n);
    r /= a.n;
    const int b = (int)(r % a.B);
    const int kv = (int)(r / a.B);
    const size_t rec = rec_row(a.pg, a.H, b, h, a.pos0.v[b] + t);
    const int meta_rec = 2 * (kHeadDim / a.g);
    // loop l's input: the tails hold loops 0 .. nres-1, the call's input the last loop
    auto load_loop = [&](int l, double v[4]) {
        if (l == a.nres) {
            load4_bf16(a.x_anchor[kv] + (((size_t)b * a.n + t) * a.H + h) * kHeadDim + lane * 4, v);
        } else {
            const uint16_t *tail =
                reinterpret_cast<const uint16_t *>(a.tail0 + l * a.tail_loop_stride + kv * a.tail_kv_stride);
            load4_bf16(tail + (((size_t)b * a.tail_cap + t) * a.H + h) * kHeadDim + lane * 4, v);
        }
    };
    double x[4], ref[4];
    load_loop(0, x);
    uint32_t s8, m8;
    const uint32_t apack = quantize4(x, a.ba, a.g, lane, ref, &s8, &m8);
    store_record(a.a_codes0 + kv * a.anchor_kv_stride + rec * (kHeadDim * a.ba / 8),
                 a.a_meta0 + kv * a.anchor_kv_stride + rec * meta_rec, apack, s8, m8, a.ba, a.g, lane);
    if (kv == 1) raise_vmax(a.vmax + ((size_t)a.nres * a.B + b) * a.H + h, s8, lane);
    for (int l = 1; l <= a.nres; l++) {
        load_loop(l, x);
        encode_residual(a, x, ref, l - 1, kv, b, h, rec, lane, ref);   // ref becomes x_hat_l
    }
}

__global__ void tail_copy_kernel(const TailArgs a) {
    // 16-byte vectors: 16 per 128-element row
    const long long per_side = (long long)a.B * a.n * a.H * (kHeadDim / 8);
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= 2 * per_side) return;
    const int kv = (int)(i / per_side);
    long long r = i % per_side;
    const int vec = (int)(r % (kHeadDim / 8));
    r /= (kHeadDim / 8);
    const int h = (int)(r % a.H);
    r /= a.H;
    const int t = (int)(r % a.n);
    const int b = (int)(r / a.n);
    const uint4 *src = reinterpret_cast<const uint4 *>(a.src[kv] + (((size_t)b * a.n + t) * a.H + h) * kHeadDim);
    uint4 *dst = reinterpret_cast<uint4 *>(a.dst[kv] + (((size_t)b * a.cap + a.pos0 + t) * a.H + h) * kHeadDim);
    dst[vec] = src[vec];
}

__global__ void bf16_store_kernel(const Bf16StoreArgs a) {
    const long long per_side = (long long)a.B * a.n * a.H * (kHeadDim / 8);
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= 2 * per_side) return;
    const int kv = (int)(i / per_side);
    long long r = i % per_side;
    const int vec = (int)(r % (kHeadDim / 8));
    r /= (kHeadDim / 8);
    const int h = (int)(r % a.H);
    r /= a.H;
    const int t = (int)(r % a.n);
    const int b = (int)(r / a.n);
    const uint4 *src = reinterpret_cast<const uint4 *>(a.src[kv] + (((size_t)b * a.n + t) * a.H + h) * kHeadDim);
    uint4 *dst = reinterpret_cast<uint4 *>(a.dst[kv] + (((size_t)b * a.H + h) * a.Tp + a.pos0.v[b] + t) * kHeadDim);
    dst[vec] = src[vec];
}

// Paged caches: block-table writes (CTA (0, 0)) and block copies (CTA
// (copy, group x array) copies one block of one record array).
__global__ void block_ops_kernel(const BlockOpsArgs a) {
    if (blockIdx.x == 0 && blockIdx.y == 0)
        for (int i = threadIdx.x; i < a.n_sets; i += blockDim.x) a.table[a.set_idx[i]] = a.set_val[i];
    const int ci = blockIdx.x;
    if (ci >= a.n_copies) return;
    const int g = blockIdx.y / a.n_arrays, arr = blockIdx.y % a.n_arrays;
    const size_t bytes = a.rows_per_block * a.arr_rec[arr];
    uint8_t *base = a.records + g * a.group_block + a.arr_off[arr];
    const uint4 *src = reinterpret_cast<const uint4 *>(base + (size_t)a.copy_src[ci] * bytes);
    uint4 *dst = reinterpret_cast<uint4 *>(base + (size_t)a.copy_dst[ci] * bytes);
    for (size_t i = threadIdx.x; i < bytes / 16; i += blockDim.x) dst[i] = src[i];
}

}  // namespace

cudaError_t launch_block_ops(const BlockOpsArgs &a, cudaStream_t st) {
    if (a.n_sets == 0 && a.n_copies == 0) return cudaSuccess;
    const dim3 grid(a.n_copies > 0 ? a.n_copies : 1, a.n_copies > 0 ? a.n_groups * a.n_arrays : 1);
    if (grid.y > 65535) return cudaErrorInvalidValue;
    block_ops_kernel<<<grid, 256, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_append(const AppendArgs &a, cudaStream_t st) {
    const long long warps = 2LL * a.B * a.n * a.H * (a.chained ? 1 : a.nres + 1);
    const long long blocks = (warps + 3) / 4;
    if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    if (a.chained)
        append_chain_kernel<<<(unsigned)blocks, 128, 0, st>>>(a);
    else
        append_kernel<<<(unsigned)blocks, 128, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_tail_copy(const TailArgs &a, cudaStream_t st) {
    const long long n = 2LL * a.B * a.n * a.H * (kHeadDim / 8);
    tail_copy_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_bf16_store(const Bf16StoreArgs &a, cudaStream_t st) {
    const long long n = 2LL * a.B * a.n * a.H * (kHeadDim / 8);
    bf16_store_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace rq
