// Dispatch layout kernel.
//
// "DeepEP Buffer Class API ...", section "Configuration and Layout Helpers":
// from topk_idx derive, before any data moves, how many tokens each rank
// receives and which ranks each token goes to; the per-expert counts are the
// receive counts of the "Code Examples" section.
//
// One thread per token, all its K ids loaded at once.  The rank-hit set of a
// token is a 32-bit mask (R <= 32);
// per-rank counts come from warp ballots + popc, per-expert counts from shared
// memory atomics, and each block adds its counts to the global histograms.
// The grid is (token blocks, source rank), so a block never straddles ranks; the
// sources are all R ranks, or those of one shard of a sharded exchange.
// Traffic: K*8 bytes read and R bytes written per token; latency-bound.

#include "common.cuh"
#include "kernels.h"

namespace ep {

namespace {

__device__ __forceinline__ uint32_t spread4(uint32_t m) {
    // bits 0..3 of m -> bytes 0..3 (each 0 or 1)
    return (m & 1u) | ((m & 2u) << 7) | ((m & 4u) << 14) | ((m & 8u) << 21);
}

template <int kMaxK>
__global__ void __launch_bounds__(kLayoutThreads)
layout_kernel(const LayoutParams p) {
    extern __shared__ int sh[];
    int* sh_rank = sh;        // [32]
    int* sh_expert = sh + 32; // [E]
    pdl_wait();               // (launched with programmatic serialization: reads nothing before this)
    for (int i = threadIdx.x; i < 32 + p.E; i += blockDim.x) sh[i] = 0;

    const int s = blockIdx.y;
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t g = (int64_t)s * p.T + t;
    int64_t ids[kMaxK];   // all of the token's ids in flight at once
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) ids[k] = (t < p.T && k < p.K) ? __ldg(p.topk_idx + g * p.K + k) : -1;
    __syncthreads();

    uint32_t mask = 0;
    bool bad = false;
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) {
        const int64_t e = ids[k];
        if (e == -1) continue;
        if (e < -1 || e >= p.E) {
            bad = true;
            continue;
        }
        mask |= 1u << ((uint32_t)e / (uint32_t)p.L);
        atomicAdd(&sh_expert[e], 1);
    }
    if (t < p.T) {
        if (bad) record_error(p.err, EP_ERR_BAD_TOPK);
        uint8_t* out = p.is_token_in_rank + g * p.R;
        if ((p.R & 3) == 0) {
            uint32_t* o4 = reinterpret_cast<uint32_t*>(out);
            for (int c = 0; c < p.R / 4; ++c) o4[c] = spread4(mask >> (4 * c));
        } else {
            for (int d = 0; d < p.R; ++d) out[d] = (mask >> d) & 1u;
        }
    }
    const int lane = threadIdx.x & 31;
    for (int d = 0; d < p.R; ++d) {
        const unsigned b = __ballot_sync(kFullMask, (mask >> d) & 1u);
        if (lane == 0 && b) atomicAdd(&sh_rank[d], __popc(b));
    }
    __syncthreads();
    for (int i = threadIdx.x; i < p.R; i += blockDim.x)
        if (sh_rank[i]) atomicAdd(p.num_tokens_per_rank + s * p.R + i, sh_rank[i]);
    for (int i = threadIdx.x; i < p.E; i += blockDim.x)
        if (sh_expert[i]) atomicAdd(p.num_tokens_per_expert + (int64_t)s * p.E + i, sh_expert[i]);
}

}  // namespace

cudaError_t launch_layout(const LayoutParams& p, cudaStream_t stream) {
    if (p.T == 0) return cudaSuccess;
    if (p.num_src == 0) return cudaSuccess;
    dim3 grid((p.T + kLayoutThreads - 1) / kLayoutThreads, p.num_src);
    const size_t smem = (32 + (size_t)p.E) * sizeof(int);
    if (p.K <= 8) return launch_pdl(layout_kernel<8>, grid, dim3(kLayoutThreads), smem, stream, p);
    if (p.K <= 16) return launch_pdl(layout_kernel<16>, grid, dim3(kLayoutThreads), smem, stream, p);
    return launch_pdl(layout_kernel<32>, grid, dim3(kLayoutThreads), smem, stream, p);
}

}  // namespace ep
