// Low-latency (expert-major packed) dispatch bookkeeping and combine.
//
// "DeepEP Buffer Class API ...", sections "IB-GDA Kernels" and "Low-Latency
// Inference with FP8": the low-latency dispatch streams tokens into packed
// per-expert receive buffers bounded by num_max_dispatch_tokens_per_rank and
// returns per-expert counts plus a handle; the low-latency combine reduces the
// expert outputs back to token positions with topk_idx, the weights and the
// handle.
//
// Slot order: the tokens of expert e are packed in (source rank, token) order,
// so slot(s, t, e) = #{(s', t') < (s, t) naming e}.  ll_count_kernel computes
// it with one CTA per expert: the CTA sweeps all G tokens in order, a block
// scan of the membership flags gives each member its slot, and it writes
// src_info (token index per slot), layout_range (first slot and count per
// source rank), the count, and a [G][K] slot map for the copy kernel (the
// dispatch kernel's packed mode).  No atomics touch the order, so the packing
// is deterministic.
//
// ll_combine_kernel: one warp per token.  Lane k finds the slot of its expert
// by binary search in src_info inside layout_range[e][s] (ascending token
// ids), the valid slots are ranked by (expert id, k), and the rows are reduced
// with an fp32 fused multiply-add chain in that order.

#include "common.cuh"
#include "kernels.h"

namespace ep {

namespace {

constexpr int kCountThreads = 512;
constexpr int kCountWarps = kCountThreads / 32;
constexpr int kLLCombineThreads = 256;
constexpr int kLLCombineWarps = kLLCombineThreads / 32;
constexpr int kRowsPerGroup = 8;

__global__ void __launch_bounds__(kCountThreads)
ll_count_kernel(const LLCountParams p) {
    __shared__ int s_warp_total[kCountWarps];
    __shared__ int s_base;
    __shared__ int s_begin[33];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int e = blockIdx.x;
    const long long cap = p.ll_capacity;
    int* src_info = p.src_info + (long long)e * cap;
    if (tid == 0) s_base = 0;
    __syncthreads();

    for (long long c0 = 0; c0 < p.G; c0 += kCountThreads) {
        const long long g = c0 + tid;
        uint32_t kmask = 0;
        if (g < p.G) {
            const int64_t* row = p.topk_idx + g * p.K;
            for (int k = 0; k < p.K; ++k) {
                const int64_t v = __ldg(row + k);
                if (v == e) kmask |= 1u << k;
                if (e == 0 && (v < -1 || v >= p.E)) record_error(p.err, EP_ERR_BAD_TOPK);
            }
        }
        const bool member = kmask != 0;
        const uint32_t b = __ballot_sync(kFullMask, member);
        if (lane == 0) s_warp_total[warp] = __popc(b);
        __syncthreads();
        int warp_off = 0, block_total = 0;
        for (int w = 0; w < kCountWarps; ++w) {
            const int v = s_warp_total[w];
            warp_off += (w < warp) ? v : 0;
            block_total += v;
        }
        const int slot = s_base + warp_off + __popc(b & lanemask_lt());
        if (g < p.G) {
            const int t = (int)(g % p.T);
            if (t == 0) s_begin[g / p.T] = slot;   // slots before this rank's first token
            if (member) {
                if (slot < cap) {
                    src_info[slot] = t;
                    for (int k = 0; k < p.K; ++k)
                        if ((kmask >> k) & 1u) p.slot_map[g * p.K + k] = slot;
                } else {
                    record_error(p.err, EP_ERR_CAPACITY);
                }
            }
        }
        __syncthreads();
        if (tid == 0) s_base += block_total;
        __syncthreads();
    }
    if (tid == 0) s_begin[p.R] = s_base;
    __syncthreads();
    for (int s = tid; s < p.R; s += kCountThreads) {
        p.layout_range[((long long)e * p.R + s) * 2 + 0] = s_begin[s];
        p.layout_range[((long long)e * p.R + s) * 2 + 1] = s_begin[s + 1] - s_begin[s];
    }
    if (tid == 0) p.packed_recv_count[e] = s_base;
}

__device__ __forceinline__ void fma_bf16x8(float* acc, float w, const uint4& v) {
    acc[0] = __fmaf_rn(w, bf16_lo(v.x), acc[0]);
    acc[1] = __fmaf_rn(w, bf16_hi(v.x), acc[1]);
    acc[2] = __fmaf_rn(w, bf16_lo(v.y), acc[2]);
    acc[3] = __fmaf_rn(w, bf16_hi(v.y), acc[3]);
    acc[4] = __fmaf_rn(w, bf16_lo(v.z), acc[4]);
    acc[5] = __fmaf_rn(w, bf16_hi(v.z), acc[5]);
    acc[6] = __fmaf_rn(w, bf16_lo(v.w), acc[6]);
    acc[7] = __fmaf_rn(w, bf16_hi(v.w), acc[7]);
}

template <int U>
__global__ void __launch_bounds__(kLLCombineThreads)
ll_combine_kernel(const LLCombineParams p) {
    __shared__ long long s_rows[kLLCombineWarps][32];
    __shared__ float s_w[kLLCombineWarps][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nvec = p.H / 8;
    const long long cap = p.ll_capacity;

    const long long stride = (long long)gridDim.x * kLLCombineWarps;
    for (long long g = (long long)blockIdx.x * kLLCombineWarps + warp; g < p.G; g += stride) {
        const int s = (int)(g / p.T), t = (int)(g % p.T);
        long long e = -1;
        float w = 0.f;
        if (lane < p.K) {
            e = p.topk_idx[g * p.K + lane];
            w = p.topk_weights[g * p.K + lane];
        }
        bool valid = e >= 0 && e < p.E;
        long long row = -1;
        if (valid) {
            const int* range = p.layout_range + ((long long)e * p.R + s) * 2;
            int lo = max(range[0], 0);
            const int end = (int)min((long long)lo + max(range[1], 0), cap);
            const int* info = p.src_info + e * cap;
            int hi = end;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (info[mid] < t) lo = mid + 1; else hi = mid;
            }
            if (lo < end && info[lo] == t) {
                row = e * cap + lo;
            } else {
                record_error(p.err, EP_ERR_HANDLE_MISMATCH);
                valid = false;
            }
        }
        // rank among valid slots by (expert id, k)
        int rank = 0;
        for (int k = 0; k < p.K; ++k) {
            const long long ek = __shfl_sync(kFullMask, e, k);
            const bool vk = __shfl_sync(kFullMask, valid, k);
            if (vk && (ek < e || (ek == e && k < lane))) ++rank;
        }
        const int nv = __popc(__ballot_sync(kFullMask, valid));
        if (valid) {
            s_rows[warp][rank] = row;
            s_w[warp][rank] = w;
        }
        __syncwarp();

        uint4* out = reinterpret_cast<uint4*>(p.out_x + g * p.H);
        for (int c0 = 0; c0 < nvec; c0 += 32 * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
            for (int i0 = 0; i0 < nv; i0 += kRowsPerGroup) {
                uint4 v[kRowsPerGroup][U];
#pragma unroll
                for (int i = 0; i < kRowsPerGroup; ++i) {
                    if (i0 + i < nv) {
                        const uint4* src = reinterpret_cast<const uint4*>(p.y + s_rows[warp][i0 + i] * p.H);
#pragma unroll
                        for (int u = 0; u < U; ++u) {
                            const int c = c0 + lane + 32 * u;
                            if (c < nvec) v[i][u] = ld_stream_v4(src + c);
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < kRowsPerGroup; ++i) {
                    if (i0 + i < nv) {
                        const float wi = s_w[warp][i0 + i];
#pragma unroll
                        for (int u = 0; u < U; ++u)
                            if (c0 + lane + 32 * u < nvec) fma_bf16x8(acc[u], wi, v[i][u]);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + lane + 32 * u;
                if (c >= nvec) continue;
                uint4 o;
                o.x = pack_bf16x2_rn(acc[u][0], acc[u][1]);
                o.y = pack_bf16x2_rn(acc[u][2], acc[u][3]);
                o.z = pack_bf16x2_rn(acc[u][4], acc[u][5]);
                o.w = pack_bf16x2_rn(acc[u][6], acc[u][7]);
                st_stream_v4(out + c, o);
            }
        }
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_ll_count(const LLCountParams& p, cudaStream_t stream) {
    if (p.G == 0 || p.E == 0) return cudaSuccess;
    ll_count_kernel<<<p.E, kCountThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_ll_combine(const LLCombineParams& p, int num_sms, cudaStream_t stream) {
    if (p.G == 0) return cudaSuccess;
    constexpr int U = 2;
    long long blocks = (p.G + kLLCombineWarps - 1) / kLLCombineWarps;
    const long long cap = (long long)num_sms * 4;
    if (blocks > cap) blocks = cap;
    ll_combine_kernel<U><<<(int)blocks, kLLCombineThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace ep
