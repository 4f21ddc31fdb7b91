// Dispatch layout kernel.
//
// "DeepEP Buffer Class API ...", section "Configuration and Layout Helpers":
// from topk_idx derive, before any data moves, how many tokens each rank
// receives and which ranks each token goes to; the per-expert counts are the
// receive counts of the "Code Examples" section.
//
// One thread block cluster per source rank; its CTAs (up to 8) split the
// source's tokens, one thread per token with all its K ids loaded at once.
// The rank-hit set of a token is a 32-bit mask (R <= 32).  Each CTA counts in
// shared memory -- ranks by warp ballots + popc, experts by shared-memory
// atomics -- and after a cluster barrier the CTAs sum the cluster's histograms
// through distributed shared memory, each CTA a slice of the entries, and
// write them: no global atomics, and the outputs need no zeroing before the
// launch (measured on B200, DSv3 step: the two zeroing memsets of a global-
// atomic design alone cost ~4 us).  The sources are all R ranks, or those of
// one shard of a sharded exchange.
// Traffic: K*8 bytes read and R bytes written per token; latency-bound.

#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace ep {

namespace {

namespace cg = cooperative_groups;

constexpr int kLayoutMaxCluster = 8;   // portable cluster size

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
    cg::cluster_group cluster = cg::this_cluster();
    const int cs = (int)cluster.num_blocks();     // CTAs of this source (gridDim.x)
    const int cr = (int)cluster.block_rank();     // this CTA's place among them
    pdl_wait();               // (launched with programmatic serialization: reads nothing before this)
    for (int i = threadIdx.x; i < 32 + p.E; i += blockDim.x) sh[i] = 0;
    __syncthreads();

    const int s = blockIdx.y;
    const int per = (p.T + cs - 1) / cs;
    const int t_lo = cr * per, t_hi = min(p.T, t_lo + per);
    const int lane = threadIdx.x & 31;
    for (int t0 = t_lo; t0 < t_hi; t0 += kLayoutThreads) {   // block-uniform bounds
        const int t = t0 + threadIdx.x;
        const int64_t g = (int64_t)s * p.T + t;
        int64_t ids[kMaxK];   // all of the token's ids in flight at once
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) ids[k] = (t < t_hi && k < p.K) ? __ldg(p.topk_idx + g * p.K + k) : -1;

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
        if (t < t_hi) {
            if (bad) record_error(p.err, EP_ERR_BAD_TOPK);
            uint8_t* out = p.is_token_in_rank + g * p.R;
            if ((p.R & 3) == 0) {
                uint32_t* o4 = reinterpret_cast<uint32_t*>(out);
                for (int c = 0; c < p.R / 4; ++c) o4[c] = spread4(mask >> (4 * c));
            } else {
                for (int d = 0; d < p.R; ++d) out[d] = (mask >> d) & 1u;
            }
        }
        for (int d = 0; d < p.R; ++d) {
            const unsigned b = __ballot_sync(kFullMask, (mask >> d) & 1u);
            if (lane == 0 && b) atomicAdd(&sh_rank[d], __popc(b));
        }
    }
    cluster.sync();   // every CTA's counts are final and visible to the cluster

    // entries [0, R) are the rank counts (sh[i]), [R, R + E) the expert counts
    // (sh[32 + i - R]); CTA cr sums and writes its slice of them
    const int n = p.R + p.E;
    const int chunk = (n + cs - 1) / cs;
    const int i_hi = min(n, (cr + 1) * chunk);
    for (int i = cr * chunk + threadIdx.x; i < i_hi; i += kLayoutThreads) {
        const int idx = i < p.R ? i : 32 + (i - p.R);
        int sum = 0;
        for (int b = 0; b < cs; ++b) sum += *cluster.map_shared_rank(sh + idx, b);
        if (i < p.R)
            p.num_tokens_per_rank[s * p.R + i] = sum;
        else
            p.num_tokens_per_expert[(int64_t)s * p.E + (i - p.R)] = sum;
    }
    cluster.sync();   // no CTA leaves while another still reads its shared memory
}

template <int kMaxK>
cudaError_t launch_k(const LayoutParams& p, int cs, size_t smem, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cs, (unsigned)p.num_src);
    cfg.blockDim = dim3(kLayoutThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, layout_kernel<kMaxK>, p);
}

}  // namespace

cudaError_t launch_layout(const LayoutParams& p, cudaStream_t stream) {
    if (p.num_src == 0) return cudaSuccess;
    // CTAs per source: one per kLayoutThreads tokens, at most a portable cluster
    // (a CTA then walks several token blocks); T = 0 still writes zero counts
    const int cs = max(1, min(kLayoutMaxCluster, (p.T + kLayoutThreads - 1) / kLayoutThreads));
    const size_t smem = (32 + (size_t)p.E) * sizeof(int);
    if (p.K <= 8) return launch_k<8>(p, cs, smem, stream);
    if (p.K <= 16) return launch_k<16>(p, cs, smem, stream);
    return launch_k<32>(p, cs, smem, stream);
}

}  // namespace ep
