// Handle check: is a stored dispatch handle still the one for this routing?
//
// "How DeepEP Optimizes Handle Reuse ...", section "Performance Contract and
// Constraints": a handle may be reused only while topk_idx is unchanged.  This
// kernel recomputes, for every token, the set of ranks its experts live on
// (rank(e) = e / L over its valid ids) and compares it with the handle's
// is_token_in_rank row and with the membership send_head encodes (>= 0 exactly
// for the member ranks, and below that rank's receive count).  Any difference
// records EP_ERR_HANDLE_MISMATCH.  One thread per token; reads K*8 + R*5 bytes
// per token, no waits.

#include "common.cuh"
#include "check.h"
#include "kernels.h"

namespace ep {

namespace {

constexpr int kCheckThreads = 256;

template <int kMaxK>
__global__ void __launch_bounds__(kCheckThreads)
handle_check_kernel(const HandleCheckParams p) {
    const long long g = (long long)blockIdx.x * kCheckThreads + threadIdx.x;
    if (g >= p.G) return;
    int64_t ids[kMaxK];
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) ids[k] = k < p.K ? __ldg(p.topk_idx + g * p.K + k) : -1;
    uint32_t mask = 0;
#pragma unroll
    for (int k = 0; k < kMaxK; ++k)
        if (ids[k] >= 0 && ids[k] < p.E) mask |= 1u << ((uint32_t)ids[k] / (uint32_t)p.L);
    bool ok = true;
    for (int d = 0; d < p.R; ++d) {
        const bool member = (mask >> d) & 1u;
        const bool in_rank = __ldg(p.is_token_in_rank + g * p.R + d) != 0;
        const int h = __ldg(p.send_head + g * p.R + d);
        const long long n_d = p.recv_rank_offset[d + 1] - p.recv_rank_offset[d];
        ok &= in_rank == member && (h >= 0) == member && (h < 0 || h < n_d);
    }
    if (!ok) record_error(p.err, EP_ERR_HANDLE_MISMATCH);
}

}  // namespace

cudaError_t launch_handle_check(const HandleCheckParams& p, cudaStream_t stream) {
    if (p.G == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((p.G + kCheckThreads - 1) / kCheckThreads);
    if (p.K <= 8)
        handle_check_kernel<8><<<blocks, kCheckThreads, 0, stream>>>(p);
    else if (p.K <= 16)
        handle_check_kernel<16><<<blocks, kCheckThreads, 0, stream>>>(p);
    else
        handle_check_kernel<32><<<blocks, kCheckThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace ep
