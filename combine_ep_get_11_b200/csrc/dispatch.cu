// Dispatch row scatter (normal, cached and low-latency packed).
//
// "DeepEP Buffer Class API ...", section "Dispatch Operation": each token row
// goes, with its top-k ids and weights, to every rank that owns one of its
// experts.  "How DeepEP Optimizes Handle Reuse ...", section "Fast Path
// Dispatch with Handle Reuse": the cached form moves rows only.  Section
// "IB-GDA Kernels": the low-latency form packs rows expert-major.
//
// On one GPU every destination is a row of device memory, so the kernel is a
// fan-out copy: read each source row from HBM once, write it to all of its
// destinations.  The traffic is write-dominated (fan-out ~5 on the
// DeepSeek-V3 shape), and on B200 plain 16-byte stores from many resident
// warps write HBM faster than TMA bulk stores (measured: 6.8 vs 6.1-6.4 TB/s
// write-only; 6.5 vs 5.7 TB/s for this kernel), so:
//   * one warp per source token (or per column slice of its row when there
//     are too few tokens to fill the GPU), a grid of blocks of 8 warps: the
//     block scheduler balances the work (no persistent loop, no tail of long
//     CTAs), and the work is split by source token, so a skewed destination
//     histogram costs nothing extra;
//   * each lane loads its share of the row as up to kVecPerLane 16-byte
//     vectors at once (a 7168-wide bf16 row is 28 vectors per lane: one
//     round trip of loads in flight per warp), then stores the vectors to
//     every destination row (streaming stores, coalesced 512 B per warp
//     instruction);
//   * lane d (destination rank), or lane k (top-k slot) in the packed form,
//     resolves its destination row; a ballot compacts the rows in lane order;
//   * in the normal form the destination lanes also write the receive
//     metadata: local top-k ids, weights, and recv_src_idx.
// Per token the HBM traffic is H*2 bytes read + fan-out * H*2 bytes written.

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace ep {

namespace {

constexpr int kDispatchThreads = 256;
constexpr int kDispatchWarps = kDispatchThreads / 32;
constexpr int kVecPerLane = 28;   // 16-byte vectors held per lane per pass

template <int kMode, int kVec = kVecPerLane>
__global__ void __launch_bounds__(kDispatchThreads, 2)
dispatch_kernel(const DispatchParams p) {
    __shared__ long long s_rows[kDispatchWarps][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long wid = (long long)blockIdx.x * kDispatchWarps + warp;
    const long long g = wid / p.splits;          // token
    const int part = (int)(wid % p.splits);      // column slice of its row
    if (g >= p.G) return;   // whole warp

    long long row = -1;
    if (kMode == kModeLowLatency) {
        long long e = -1;
        if (lane < p.K) e = p.topk_idx[g * p.K + lane];
        bool valid = e >= 0 && e < p.E;
        for (int k = 0; k < p.K; ++k) {   // a repeated expert is sent once
            const long long ek = __shfl_sync(kFullMask, e, k);
            if (k < lane && ek == e) valid = false;
        }
        if (valid) {
            const int slot = p.slot_map[g * p.K + lane];
            if (slot >= 0 && slot < p.ll_capacity)
                row = e * p.ll_capacity + slot;
            else
                record_error(p.err, EP_ERR_CAPACITY);
        }
    } else if (lane < p.R) {
        const int h = p.send_head[g * p.R + lane];
        if (h >= 0) {
            row = p.recv_rank_offset[lane] + h;
            if (row >= p.recv_capacity) {
                record_error(p.err, EP_ERR_CAPACITY);
                row = -1;
            }
        }
    }

    if (kMode == kModeNormal && part == 0) {
        long long e = -1;
        float w = 0.f;
        if (lane < p.K) {
            e = p.topk_idx[g * p.K + lane];
            if (p.topk_weights != nullptr) w = p.topk_weights[g * p.K + lane];
        }
        if (row >= 0 && p.recv_src_idx != nullptr) p.recv_src_idx[row] = (int)(g % p.T);
        for (int k = 0; k < p.K; ++k) {
            const long long ek = __shfl_sync(kFullMask, e, k);
            const float wk = __shfl_sync(kFullMask, w, k);
            if (row >= 0) {
                const bool here = ek >= 0 && ek < p.E && (int)ek / p.L == lane;
                if (p.recv_topk_idx != nullptr)
                    p.recv_topk_idx[row * p.K + k] = here ? (long long)((int)ek % p.L) : -1LL;
                if (p.recv_topk_weights != nullptr)
                    p.recv_topk_weights[row * p.K + k] = here ? wk : 0.f;
            }
        }
    }
    if (kMode == kModeNormal && p.recv_x == nullptr) return;   // metadata only

    const uint32_t m = __ballot_sync(kFullMask, row >= 0);
    const int f = __popc(m);
    if (row >= 0) s_rows[warp][__popc(m & lanemask_lt())] = row;
    __syncwarp();

    // this warp's column slice: whole 32-vector strides
    const int nvec = p.H / 8;
    const int per = ((nvec + p.splits - 1) / p.splits + 31) / 32 * 32;
    const int lo = part * per, hi = min(nvec, lo + per);
    const uint4* src = reinterpret_cast<const uint4*>(p.x + g * p.H);
    for (int c0 = lo; c0 < hi; c0 += 32 * kVec) {
        uint4 v[kVec];
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
            const int c = c0 + lane + 32 * u;
            if (c < hi) v[u] = ld_nc_v4(src + c);
        }
        for (int i = 0; i < f; ++i) {
            uint4* dst = reinterpret_cast<uint4*>(p.recv_x + s_rows[warp][i] * p.H);
#pragma unroll
            for (int u = 0; u < kVec; ++u) {
                const int c = c0 + lane + 32 * u;
                if (c < hi) st_stream_v4(dst + c, v[u]);
            }
        }
    }
}

template <int kMode>
cudaError_t launch_mode(const DispatchParams& p, cudaStream_t stream) {
    const long long blocks = (p.G * p.splits + kDispatchWarps - 1) / kDispatchWarps;
    dispatch_kernel<kMode><<<(unsigned)blocks, kDispatchThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dispatch(int mode, const DispatchParams& p, cudaStream_t stream) {
    if (p.G == 0) return cudaSuccess;
    switch (mode) {
        case kModeNormal: return launch_mode<kModeNormal>(p, stream);
        case kModeCached: return launch_mode<kModeCached>(p, stream);
        case kModeLowLatency: return launch_mode<kModeLowLatency>(p, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ep
