// Load balance for redundant experts: weight prefetch and gradient reduction.
//
// "第 10 章 V2：EP 之外的 Buffer 与扩展能力", section 10.2: lb_prefetch_weights
// copies the weights of redundant expert replicas in before the expert compute,
// lb_reduce_grads folds the replicas' gradients back into the original experts,
// both keyed by redundancy_mapping (replica i -> original expert, -1 unused).
// With every expert's weights one block of W bf16 values:
//   prefetch: redundant[i] = expert_weights[mapping[i]]                (bit copy)
//   reduce:   expert_grads[e] = bf16(expert_grads[e] + sum_{i ascending,
//             mapping[i] = e} redundant_grads[i])           (fp32, one rounding)
// Both are HBM-bound streams of 16-byte vectors; each CTA moves a 32 KB chunk of
// one replica (prefetch) or one expert (reduce), so even a few large experts
// spread over the whole GPU.

#include "common.cuh"
#include "kernels.h"

namespace ep {

namespace {

constexpr int kLBThreads = 256;
constexpr int kLBVec = 8;                              // vectors per thread per CTA
constexpr long long kLBChunk = (long long)kLBThreads * kLBVec;   // 2048 vectors = 32 KB
constexpr int kLBMaxReplicas = 1024;                   // replicas of one expert
constexpr int kLBMaxExperts = 4096;

__global__ void __launch_bounds__(kLBThreads)
lb_prefetch_kernel(const LBParams p) {
    pdl_wait();   // (launched with programmatic serialization: reads nothing before this)
    const int i = blockIdx.y;
    const int e = p.mapping[i];
    if (e == -1) return;
    if (e < -1 || e >= p.E) {
        if (threadIdx.x == 0 && blockIdx.x == 0) record_error(p.err, EP_ERR_BAD_TOPK);
        return;
    }
    const uint4* src = reinterpret_cast<const uint4*>(p.expert) + (long long)e * p.Wv;
    uint4* dst = reinterpret_cast<uint4*>(p.redundant) + (long long)i * p.Wv;
    const long long base = (long long)blockIdx.x * kLBChunk + threadIdx.x;
    uint4 v[kLBVec];
#pragma unroll
    for (int u = 0; u < kLBVec; ++u) {
        const long long c = base + (long long)u * kLBThreads;
        if (c < p.Wv) v[u] = ld_nc_v4(src + c);
    }
#pragma unroll
    for (int u = 0; u < kLBVec; ++u) {
        const long long c = base + (long long)u * kLBThreads;
        if (c < p.Wv) st_stream_v4(dst + c, v[u]);
    }
}

__device__ __forceinline__ void add8(float* a, const uint4& v) {
    a[0] = __fadd_rn(a[0], bf16_lo(v.x)); a[1] = __fadd_rn(a[1], bf16_hi(v.x));
    a[2] = __fadd_rn(a[2], bf16_lo(v.y)); a[3] = __fadd_rn(a[3], bf16_hi(v.y));
    a[4] = __fadd_rn(a[4], bf16_lo(v.z)); a[5] = __fadd_rn(a[5], bf16_hi(v.z));
    a[6] = __fadd_rn(a[6], bf16_lo(v.w)); a[7] = __fadd_rn(a[7], bf16_hi(v.w));
}

// Grid row y handles the y-th expert (ascending id) that has at least one
// replica, so experts without replicas cost nothing.
__global__ void __launch_bounds__(kLBThreads)
lb_reduce_kernel(const LBParams p) {
    __shared__ uint32_t s_touched[kLBMaxExperts / 32];
    __shared__ int s_list[kLBMaxReplicas];
    __shared__ int s_warp[kLBThreads / 32];
    __shared__ int s_n, s_e;
    pdl_wait();   // (launched with programmatic serialization: reads nothing before this)
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int words = (p.E + 31) / 32;
    for (int i = tid; i < words; i += kLBThreads) s_touched[i] = 0;
    if (tid == 0) { s_n = 0; s_e = -1; }
    __syncthreads();
    for (int i = tid; i < p.N; i += kLBThreads) {
        const int m = p.mapping[i];
        if (m >= 0 && m < p.E) atomicOr(&s_touched[m >> 5], 1u << (m & 31));
        else if (m != -1 && blockIdx.x == 0 && blockIdx.y == 0) record_error(p.err, EP_ERR_BAD_TOPK);
    }
    __syncthreads();
    if (tid == 0) {   // the blockIdx.y-th touched expert
        int k = blockIdx.y;
        for (int w = 0; w < words; ++w) {
            const int c = __popc(s_touched[w]);
            if (k < c) {
                uint32_t bits = s_touched[w];
                for (int q = 0; q < k; ++q) bits &= bits - 1;
                s_e = w * 32 + __ffs(bits) - 1;
                break;
            }
            k -= c;
        }
    }
    __syncthreads();
    const int e = s_e;
    if (e < 0) return;
    // replicas of e in ascending order: ordered compaction, 256 entries per round
    for (int i0 = 0; i0 < p.N; i0 += kLBThreads) {
        const int i = i0 + tid;
        const int m = i < p.N ? p.mapping[i] : -1;
        const uint32_t b = __ballot_sync(kFullMask, m == e);
        if (lane == 0) s_warp[warp] = __popc(b);
        __syncthreads();
        int before = 0, total = 0;
        for (int w = 0; w < kLBThreads / 32; ++w) {
            before += w < warp ? s_warp[w] : 0;
            total += s_warp[w];
        }
        const int pos = s_n + before + __popc(b & lanemask_lt());
        if (m == e && pos < kLBMaxReplicas) s_list[pos] = i;
        __syncthreads();
        if (tid == 0) s_n += total;
        __syncthreads();
    }
    const int n = s_n;
    if (n > kLBMaxReplicas) {
        if (tid == 0 && blockIdx.x == 0) record_error(p.err, EP_ERR_CAPACITY);
        return;
    }
    uint4* __restrict__ g = reinterpret_cast<uint4*>(p.expert) + (long long)e * p.Wv;
    const uint4* __restrict__ red = reinterpret_cast<const uint4*>(p.redundant);
    const long long base = (long long)blockIdx.x * kLBChunk + tid;
    float acc[kLBVec][8];
    const long long chunk0 = (long long)blockIdx.x * kLBChunk;
    const uint32_t chunk_bytes = (uint32_t)(min(kLBChunk, p.Wv - chunk0) * 16);
    // The gradient chunk and the first replica's chunk are loaded together (measured
    // on B200, 32 DSv3-sized experts with 8 replicas: 336 -> 308 us against loading
    // the gradient chunk first); each later replica's chunk is pulled into L2 one
    // replica ahead of its loads.
    {
        uint4 gv[kLBVec], v0[kLBVec];
        const uint4* r0 = red + (long long)(n > 0 ? s_list[0] : 0) * p.Wv;
        if (tid == 0 && n > 1 && chunk0 < p.Wv) prefetch_l2(red + (long long)s_list[1] * p.Wv + chunk0, chunk_bytes);
#pragma unroll
        for (int u = 0; u < kLBVec; ++u) {
            const long long c = base + (long long)u * kLBThreads;
            gv[u] = c < p.Wv ? ld_stream_v4(g + c) : make_uint4(0, 0, 0, 0);
            if (n > 0 && c < p.Wv) v0[u] = ld_stream_v4(r0 + c);
        }
#pragma unroll
        for (int u = 0; u < kLBVec; ++u) {
            const uint4 g0 = gv[u];
            acc[u][0] = bf16_lo(g0.x); acc[u][1] = bf16_hi(g0.x); acc[u][2] = bf16_lo(g0.y); acc[u][3] = bf16_hi(g0.y);
            acc[u][4] = bf16_lo(g0.z); acc[u][5] = bf16_hi(g0.z); acc[u][6] = bf16_lo(g0.w); acc[u][7] = bf16_hi(g0.w);
            if (n > 0 && base + (long long)u * kLBThreads < p.Wv) add8(acc[u], v0[u]);
        }
    }
    for (int j = 1; j < n; ++j) {      // later replicas in ascending order; all loads of one replica in flight
        if (tid == 0 && j + 1 < n && chunk0 < p.Wv)
            prefetch_l2(red + (long long)s_list[j + 1] * p.Wv + chunk0, chunk_bytes);
        const uint4* r = red + (long long)s_list[j] * p.Wv;
        uint4 v[kLBVec];
#pragma unroll
        for (int u = 0; u < kLBVec; ++u) {
            const long long c = base + (long long)u * kLBThreads;
            if (c < p.Wv) v[u] = ld_stream_v4(r + c);
        }
#pragma unroll
        for (int u = 0; u < kLBVec; ++u)
            if (base + (long long)u * kLBThreads < p.Wv) add8(acc[u], v[u]);
    }
#pragma unroll
    for (int u = 0; u < kLBVec; ++u) {
        const long long c = base + (long long)u * kLBThreads;
        if (c >= p.Wv) continue;
        uint4 o;
        o.x = pack_bf16x2_rn(acc[u][0], acc[u][1]); o.y = pack_bf16x2_rn(acc[u][2], acc[u][3]);
        o.z = pack_bf16x2_rn(acc[u][4], acc[u][5]); o.w = pack_bf16x2_rn(acc[u][6], acc[u][7]);
        g[c] = o;
    }
}

}  // namespace

cudaError_t launch_lb_prefetch(const LBParams& p, cudaStream_t stream) {
    if (p.N == 0 || p.Wv == 0) return cudaSuccess;
    const dim3 grid((unsigned)((p.Wv + kLBChunk - 1) / kLBChunk), (unsigned)p.N);
    return launch_pdl(lb_prefetch_kernel, grid, dim3(kLBThreads), 0, stream, p);
}

cudaError_t launch_lb_reduce(const LBParams& p, cudaStream_t stream) {
    if (p.N == 0 || p.Wv == 0) return cudaSuccess;
    // at most min(E, N) experts have replicas; rows past the touched count exit at once
    const dim3 grid((unsigned)((p.Wv + kLBChunk - 1) / kLBChunk), (unsigned)(p.N < p.E ? p.N : p.E));
    return launch_pdl(lb_reduce_kernel, grid, dim3(kLBThreads), 0, stream, p);
}

}  // namespace ep
