// Combine: fixed-order fp32 gather-reduce back to source order.
//
// "DeepEP Buffer Class API ...", section "Combine Operation": with the handle
// of the matching dispatch, the received rows are reduced by addition back to
// their source tokens, with optional bias terms; the "Code Examples" combine
// also returns the combined top-k weights.
//
//   out[g] = bf16_rn( ((0 + y[row_d0]) + y[row_d1]) + ... + bias0[g] + bias1[g] )
//
// over the token's destination ranks d0 < d1 < ... (row_d = recv_rank_offset[d]
// + send_head[g][d]), accumulated in fp32 in exactly that order, so the result
// does not depend on scheduling.
//
// One warp per token, or per column slice of its row when there are too few
// tokens to fill the GPU: lane d reads send_head[g][d], a ballot gives the
// destination set, and the rows are compacted in ascending rank order into
// shared memory.  Each lane then owns 16-byte columns of the hidden row; for
// every U-vector slab it issues the loads of a group of 4 rows at once
// (4 x 4 vectors; measured best on B200 for fan-ins of 3.6 and 5.2), then adds
// them in rank order, group after group.  Lane i also asks for the next column
// slab of row i ahead of time (a bulk L2 prefetch), so the slab's loads hit L2.
// Traffic per token: fan-out * H*2 bytes read (streaming), H*2 written.  The
// sharded form reads rank d's rows from the GPU hosting d (its own memory or a
// peer's, mapped into this process): the return exchange happens inside the
// reduction; it prefetches only the rows in this GPU's own memory.

#include "common.cuh"
#include "kernels.h"

namespace ep {

namespace {

constexpr int kCombineThreads = 256;
constexpr int kCombineWarps = kCombineThreads / 32;
constexpr int kRowsPerGroup = 4;   // rows whose loads are in flight together

__device__ __forceinline__ void add_bf16x8(float* acc, const uint4& v) {
    acc[0] = __fadd_rn(acc[0], bf16_lo(v.x));
    acc[1] = __fadd_rn(acc[1], bf16_hi(v.x));
    acc[2] = __fadd_rn(acc[2], bf16_lo(v.y));
    acc[3] = __fadd_rn(acc[3], bf16_hi(v.y));
    acc[4] = __fadd_rn(acc[4], bf16_lo(v.z));
    acc[5] = __fadd_rn(acc[5], bf16_hi(v.z));
    acc[6] = __fadd_rn(acc[6], bf16_lo(v.w));
    acc[7] = __fadd_rn(acc[7], bf16_hi(v.w));
}

template <int U, bool kSharded, int kGroup = kRowsPerGroup>
__global__ void __launch_bounds__(kCombineThreads, 2)
combine_kernel(const CombineParams p) {
    pdl_wait();   // (launched with programmatic serialization: reads nothing before this)
    __shared__ long long s_rows[kCombineWarps][32];             // row index, or (sharded) row address
    __shared__ long long s_wrow[kSharded ? kCombineWarps : 1][32];   // sharded: weight-row address
    __shared__ bool s_local[kSharded ? kCombineWarps : 1][32];       // sharded: row in this GPU's memory
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long wid = (long long)blockIdx.x * kCombineWarps + warp;
    const long long g = wid / p.splits;          // token
    const int part = (int)(wid % p.splits);      // column slice of its row
    if (g >= p.G) return;   // whole warp
    const int R = p.R;

    long long row = -1;
    if (lane < R) {
        const int h = p.send_head[g * R + lane];
        if (h >= 0) {
            row = (kSharded ? p.dst_offset[lane] : p.recv_rank_offset[lane]) + h;
            if (row >= p.y_rows) {
                record_error(p.err, EP_ERR_CAPACITY);
                row = -1;
            }
        }
    }
    const uint32_t m = __ballot_sync(kFullMask, row >= 0);
    const int f = __popc(m);
    if (row >= 0) {
        const int at = __popc(m & lanemask_lt());
        if constexpr (kSharded) {   // rank d's rows are in shard d / ranks_per_shard (own or peer memory)
            const int shard = lane / p.ranks_per_shard;
            s_rows[warp][at] = (long long)reinterpret_cast<uintptr_t>(p.shard_y[shard] + row * p.H);
            s_local[warp][at] = shard == p.self_shard;
            s_wrow[warp][at] =
                p.shard_w[shard] ? (long long)reinterpret_cast<uintptr_t>(p.shard_w[shard] + row * p.K) : 0;
        } else {
            s_rows[warp][at] = row;
        }
    }
    __syncwarp();

    const uint4* b0 = p.bias0 ? reinterpret_cast<const uint4*>(p.bias0 + g * p.H) : nullptr;
    const uint4* b1 = p.bias1 ? reinterpret_cast<const uint4*>(p.bias1 + g * p.H) : nullptr;
    uint4* out = reinterpret_cast<uint4*>(p.out_x + g * p.H);

    // this warp's column slice: whole 32-vector strides
    const int nvec = p.H / 8;
    const int per = ((nvec + p.splits - 1) / p.splits + 31) / 32 * 32;
    const int lo = part * per, hi = min(nvec, lo + per);
    // rows' next column slab into L2 ahead of its loads (lane i: row i of the token);
    // in the sharded form only rows in this GPU's own memory (never a peer's)
    const uint4* pf_row = nullptr;
    if (lane < f) {
        if constexpr (kSharded) {
            if (s_local[warp][lane]) pf_row = reinterpret_cast<const uint4*>(static_cast<uintptr_t>(s_rows[warp][lane]));
        } else {
            pf_row = reinterpret_cast<const uint4*>(p.y + s_rows[warp][lane] * p.H);
        }
    }
    if (pf_row != nullptr && lo < hi) prefetch_l2(pf_row + lo, (uint32_t)min(32 * U, hi - lo) * 16u);
    for (int c0 = lo; c0 < hi; c0 += 32 * U) {
        const int nxt = c0 + 32 * U;
        if (pf_row != nullptr && nxt < hi) prefetch_l2(pf_row + nxt, (uint32_t)min(32 * U, hi - nxt) * 16u);
        float acc[U][8];
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;

        for (int i0 = 0; i0 < f; i0 += kGroup) {
            uint4 v[kGroup][U];
#pragma unroll
            for (int i = 0; i < kGroup; ++i) {
                if (i0 + i < f) {
                    const uint4* src =
                        kSharded ? reinterpret_cast<const uint4*>(static_cast<uintptr_t>(s_rows[warp][i0 + i]))
                                 : reinterpret_cast<const uint4*>(p.y + s_rows[warp][i0 + i] * p.H);
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const int c = c0 + lane + 32 * u;
                        if (c < hi) v[i][u] = ld_stream_v4(src + c);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < kGroup; ++i) {
                if (i0 + i < f) {
#pragma unroll
                    for (int u = 0; u < U; ++u)
                        if (c0 + lane + 32 * u < hi) add_bf16x8(acc[u], v[i][u]);
                }
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + lane + 32 * u;
            if (c >= hi) continue;
            if (b0 != nullptr) add_bf16x8(acc[u], ld_nc_v4(b0 + c));
            if (b1 != nullptr) add_bf16x8(acc[u], ld_nc_v4(b1 + c));
            uint4 o;
            o.x = pack_bf16x2_rn(acc[u][0], acc[u][1]);
            o.y = pack_bf16x2_rn(acc[u][2], acc[u][3]);
            o.z = pack_bf16x2_rn(acc[u][4], acc[u][5]);
            o.w = pack_bf16x2_rn(acc[u][6], acc[u][7]);
            st_stream_v4(out + c, o);
        }
    }

    if constexpr (kSharded) {
        // weight rows are given for every shard whenever out_topk_weights is asked for
        if (part == 0 && p.out_topk_weights != nullptr && lane < p.K) {
            float w = 0.f;
            for (int i = 0; i < f; ++i)
                w = __fadd_rn(w, reinterpret_cast<const float*>(static_cast<uintptr_t>(s_wrow[warp][i]))[lane]);
            p.out_topk_weights[g * p.K + lane] = w;
        }
    } else if (part == 0 && p.recv_topk_weights != nullptr && p.out_topk_weights != nullptr && lane < p.K) {
        float w = 0.f;
        for (int i = 0; i < f; ++i) w = __fadd_rn(w, p.recv_topk_weights[s_rows[warp][i] * p.K + lane]);
        p.out_topk_weights[g * p.K + lane] = w;
    }
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, int num_sms, cudaStream_t stream) {
    if (p.G == 0) return cudaSuccess;
    constexpr int U = 4;   // 4 x 16-byte vectors per lane per row: 16 loads in flight per group
    // one warp per token (or column slice): the block scheduler balances the work
    (void)num_sms;
    const long long blocks = (p.G * p.splits + kCombineWarps - 1) / kCombineWarps;
    if (p.sharded) return launch_pdl(combine_kernel<U, true>, dim3((unsigned)blocks), dim3(kCombineThreads), 0, stream, p);
    return launch_pdl(combine_kernel<U, false>, dim3((unsigned)blocks), dim3(kCombineThreads), 0, stream, p);
}

}  // namespace ep
