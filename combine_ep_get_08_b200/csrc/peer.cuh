// peer.cuh -- launch interface of the peer-memory dispatch / combine kernels.
#pragma once

#include "ep_internal.cuh"

namespace ep {

struct PeerLaunch {
    const void *x;            // [T, H] bf16 (dispatch)
    void *const *base;        // device array [R]: each rank's row buffer, mapped here
    float *const *sbase;      // device array [R]: each rank's scale buffer (FP8 dispatch), else null
    const int32_t *row0;      // device array [R]: first row of this source's block there
    const int32_t *pos;       // [T, K] this rank's layout
    const int32_t *row_src;   // [cap]
    const int32_t *roff;      // [R+1]
    const float *w;           // [T, K] (combine)
    void *out;                // [T, H] bf16 (combine)
    int T, K, R, H;
    int64_t cap;
    bool zero_rows;           // expert_alignment > 1: padding rows are written as zeros
    bool prefetch_x;          // dispatch: x fits in half the L2; each CTA pulls its rows in first
};

cudaError_t launch_dispatch_peer(const PeerLaunch &l, int num_sms, cudaStream_t s);
cudaError_t launch_dispatch_fp8_peer(const PeerLaunch &l, int num_sms, cudaStream_t s);
cudaError_t launch_combine_peer(const PeerLaunch &l, int num_sms, cudaStream_t s);

// Bytes of dynamic shared memory the peer kernels take for R ranks.
inline size_t peer_smem_bytes(int R) { return 2 * sizeof(void *) * R + sizeof(int32_t) * (2 * R + 1); }

}  // namespace ep
