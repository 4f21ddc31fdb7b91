// Offsets of a sharded exchange: the R virtual ranks spread over W GPUs, GPU w
// hosting the ranks [w*R/W, (w+1)*R/W) and their receive buffers.
//
// The receive order stays the one of "DeepEP Buffer Class API ...", section
// "Dispatch Operation": the rows of destination d in (source rank, token)
// order, so a token's position in d's block is the same exclusive running
// count P(g)[d] as on one GPU.  A shard scans only its own sources, so its
// counts start at the tokens that earlier shards' sources send to d:
//   base[d]        = sum_{s < r0} num_tokens_per_rank[s][d]
// and d's block starts, inside the receive buffer of the GPU hosting d, after
// the blocks of that GPU's lower ranks:
//   N_d            = sum_s num_tokens_per_rank[s][d]
//   dst_offset[d]  = sum_{d' in shard(d), d' < d} N_{d'}
// The counts are the layouts of all shards, gathered (a few KB).  One block:
// a handful of loads per thread, latency-bound.

#include "common.cuh"
#include "kernels.h"

namespace ep {

namespace {

constexpr int kShardThreads = 256;

__global__ void __launch_bounds__(kShardThreads)
shard_offsets_kernel(const ShardOffsetsParams p) {
    __shared__ long long s_n[32];
    const int tid = threadIdx.x;
    const int R = p.R;
    if (tid < R) {
        long long n = 0;
        int before = 0;
        for (int s = 0; s < R; ++s) {
            const int v = p.num_tokens_per_rank_all[s * R + tid];
            n += v;
            if (s < p.r0) before += v;
        }
        s_n[tid] = n;
        p.base[tid] = before;
    }
    __syncthreads();
    if (tid < R) {
        const int first = tid / p.ranks_per_shard * p.ranks_per_shard;
        long long off = 0;
        for (int d = first; d < tid; ++d) off += s_n[d];
        p.dst_offset[tid] = off;
    }
    if (tid == 0 && p.num_recv_rows != nullptr) {
        long long rows = 0;
        for (int d = p.r0; d < p.r0 + p.ranks_per_shard; ++d) rows += s_n[d];
        *p.num_recv_rows = rows;
    }
    if (p.num_recv_tokens_per_expert != nullptr) {
        const int ne = p.ranks_per_shard * p.L;     // this shard's experts, from expert r0*L on
        for (int i = tid; i < ne; i += kShardThreads) {
            int sum = 0;
            for (int s = 0; s < R; ++s) sum += p.num_tokens_per_expert_all[(long long)s * p.E + p.r0 * p.L + i];
            p.num_recv_tokens_per_expert[i] = sum;
        }
    }
}

}  // namespace

cudaError_t launch_shard_offsets(const ShardOffsetsParams& p, cudaStream_t stream) {
    shard_offsets_kernel<<<1, kShardThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace ep
