// prefill.h -- launch interface of the multi-token (chunked-prefill) attention
// over the compressed cache.  Not part of the public ABI.
#pragma once

#include "rq_internal.h"

namespace rq {

constexpr int kPrefillTile = 32;   // committed tokens per step of a CTA

// Causal attention of the n most recent tokens of every sequence: query row
// (i, hq) of sequence b (i < n) sees the first T_b + n_tail - n + 1 + i tokens
// of [committed tokens of the group, then the loop's tail tokens].
struct PrefillArgs {
    // anchor streams (kv 0 = K, 1 = V); residual streams null for an anchor loop
    const uint8_t *a_codes[2], *a_meta[2];
    const uint8_t *r_codes[2], *r_meta[2];
    const uint16_t *r_coef[2];
    const uint16_t *q;                 // [B][n][Hq][d] bf16
    const uint16_t *tail_k, *tail_v;   // [B][tail_cap][H][d] bf16, or null
    float *partials;                   // [B][n][Hq][S][kPartialStride]
    float *out;                        // [B][n][Hq][d] fp32
    SeqLens seqT;                      // committed tokens of each sequence
    Pages pg;                          // token -> record row (contiguous: row bh * Tp + t)
    int B, H, Hq, G, n, n_tail, tail_cap, Tp, S;
    int nqb;                           // blocks of 64 query rows per kv head
    int g;                             // quantization group size
    float scale_log2;                  // softmax_scale * log2(e)
    int rotate;
    uint32_t sigma[4];
    int *err;                          // device error word (bounded waits that gave up)
    int *counters;                     // [B][H][nqb] split arrivals (zero between calls): the last
                                       // split of a row block merges the partials; null: the
                                       // combine kernel merges them
    int tail_in_kernel;                // the attention kernel (last split) takes the tail tokens
};

// Sets a->nqb and the split count a->S over the committed tokens (T
// = the longest sequence); a->B, H, G and n must be set.
void prefill_plan(PrefillArgs *a, int T, int ba, int br, int sms);
cudaError_t launch_prefill(const PrefillArgs &a, int ba, int br, cudaStream_t st);

}  // namespace rq
