// Internal declarations of the backward pass (backward.cu, backward_tc.cu) and its
// launches from the C ABI (hils_api.cu).
#pragma once

#include "hils_internal.cuh"

namespace hils {

struct BwdAttendArgs {
    View Q, K, V, O;
    const float *lse, *dO, *score;
    const int32_t *idx, *nsel;
    float *dQ, *dK, *dV, *dscore;
    int B, H, N, topk, W, G;
    float scale;
    long long wait_ns = kWaitLimitNs;  // work-wait limit of the tensor-core walk
};
// The tensor-core attend backward (bf16, d = 128; backward_tc.cu). A work item is a
// 64-key block of one (b, h) with at most kBwdItemQueries of the queries that attend it.
constexpr int kBwdItemQueries = 1024;
struct BwdTcArgs {
    BwdAttendArgs a;
    const float *Dv;      // [B*H*N] D_i = dO_i . o_i
    const int4 *recs;     // [B*H][N*K] per entry of the group's inverted index: {i*32+k or -1, w, D_i, i}
    const int4 *items;    // [B*Hk][max_items] chunk items {c, first entry, end entry, 0}
    const int *nitems;    // [B*Hk] chunk items listed
    int max_items;        // chunk item slots per (b, group)
    int nwin, nsegw;      // window items per (b, h) = key blocks * nsegw segments each
    int vec_ok;           // dQ 16-byte aligned: vector atomic adds
    uint32_t *status;     // bit 0: a bounded wait expired
};
hils_status launch_attend_bwd_tc(const BwdTcArgs &t, const void *Qc, const void *dOb, cudaStream_t s);
struct BwdSelectArgs {
    View Qcal, Ksum;
    const int32_t *idx, *nsel;
    const float *dscore;
    float *dQcal, *dKsum, *dBsum;
    int B, H, Lq, C, topk, G;
    float scale;
};
struct BwdSummarizeArgs {
    View K, LQ;
    const float *dKsum, *dBsum;
    float *dK, *dLQ;
    int B, H, N, C, G;
    float scale;
};
hils_status launch_attend_backward(hils_dtype dt, int d, const BwdAttendArgs &a, void *ws, cudaStream_t s);
size_t attend_backward_ws_bytes(hils_dtype dt, int d, int B, int H, int Hk, int N, int K);
hils_status launch_select_backward(hils_dtype dt, int d, const BwdSelectArgs &a, cudaStream_t s);
hils_status launch_summarize_backward(hils_dtype dt, int d, const BwdSummarizeArgs &a, cudaStream_t s);

}  // namespace hils
