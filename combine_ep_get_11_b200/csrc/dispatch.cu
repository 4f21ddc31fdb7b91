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
// destinations.  Design (persistent grid, work split by source token so a
// skewed destination histogram costs nothing extra):
//   * each CTA owns a contiguous range of global tokens; its warps take every
//     nwarps-th token of that range;
//   * each warp runs its own S-stage ring in shared memory.  Lane 0 brings a
//     row in with one TMA bulk copy (cp.async.bulk global->shared, completion
//     on an mbarrier), and each destination lane (lane d = destination rank,
//     or lane k = top-k slot in the packed form) writes it out with its own
//     bulk copy shared->global.  The row never passes through registers;
//   * a stage is refilled one iteration later, after the stores that read it
//     have finished reading (cp.async.bulk.wait_group.read), so S-1 row loads
//     and all issued stores stay in flight per warp;
//   * in the normal form the destination lanes also write the receive
//     metadata: local top-k ids, weights, and recv_src_idx.
// Per token the HBM traffic is H*2 bytes read + fan-out * H*2 bytes written.

#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace ep {

namespace {

constexpr int kDispatchMaxThreads = 256;
constexpr size_t kStageBudgetBytes = 200 * 1024;

__host__ __device__ __forceinline__ size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

template <int kMode>
__global__ void __launch_bounds__(kDispatchMaxThreads)
dispatch_kernel(const DispatchParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    const int S = p.stages;
    const uint32_t row_bytes = (uint32_t)p.H * 2u;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem) + warp * S;
    uint8_t* buf = smem + align_up((size_t)nwarps * S * 8, 128) + (size_t)warp * S * row_bytes;

    if (lane == 0) {
        for (int i = 0; i < S; ++i) mbar_init(bars + i, 1);
        fence_mbar_init();
    }
    __syncwarp();

    const long long cta_begin = p.G * blockIdx.x / gridDim.x;
    const long long cta_end = p.G * (blockIdx.x + 1) / gridDim.x;
    const long long first = cta_begin + warp;
    const int n = first < cta_end ? (int)((cta_end - first + nwarps - 1) / nwarps) : 0;

    long long off = 0;
    if (kMode != kModeLowLatency && lane < p.R) off = p.recv_rank_offset[lane];

    auto issue = [&](int j) {
        const int st = j % S;
        mbar_arrive_expect_tx(bars + st, row_bytes);
        bulk_g2s(buf + (size_t)st * row_bytes, p.x + (first + (long long)j * nwarps) * p.H, row_bytes,
                 bars + st);
    };
    // The normal form may be asked for the receive metadata only (recv_x null).
    const bool rows = p.recv_x != nullptr;
    if (rows && lane == 0)
        for (int j = 0; j < min(S, n); ++j) issue(j);

    bool ok = true;
    int j = 0;
    for (; j < n; ++j) {
        const long long g = first + (long long)j * nwarps;
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
                row = off + h;
                if (row >= p.recv_capacity) {
                    record_error(p.err, EP_ERR_CAPACITY);
                    row = -1;
                }
            }
        }
        if (kMode == kModeNormal) {
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
        if (!rows) continue;
        const int st = j % S;
        ok = __all_sync(kFullMask, mbar_wait_bounded(bars + st, (uint32_t)(j / S) & 1u));
        if (!ok) {
            record_error(p.err, EP_ERR_TIMEOUT);
            break;
        }
        if (row >= 0) bulk_s2g(p.recv_x + row * p.H, buf + (size_t)st * row_bytes, row_bytes);
        bulk_commit();
        if (j >= 1 && j - 1 + S < n) {
            bulk_wait_read<1>();
            __syncwarp();
            if (lane == 0) issue(j - 1 + S);
        }
    }
    bulk_wait<0>();
    if (!ok && lane == 0) {
        // Loads for tokens j+1 .. j+S-2 may still be landing in this warp's
        // stages; wait (bounded) before the shared memory is released.
        const int last = min(n - 1, max(min(S, n) - 1, j + S - 2));
        for (int jj = j + 1; jj <= last; ++jj) mbar_wait_bounded(bars + jj % S, (uint32_t)(jj / S) & 1u);
    }
    __syncwarp();
}

template <int kMode>
cudaError_t launch_mode(const DispatchParams& p, const DispatchGeometry& geo, cudaStream_t stream) {
    DispatchParams q = p;
    q.warps_per_cta = geo.warps_per_cta;
    q.stages = geo.stages;
    dispatch_kernel<kMode><<<geo.ctas, geo.warps_per_cta * 32, geo.smem_bytes, stream>>>(q);
    return cudaGetLastError();
}

}  // namespace

DispatchGeometry dispatch_geometry(int H, long long G, int num_sms) {
    DispatchGeometry geo{};
    const size_t row = (size_t)H * 2;
    geo.stages = row <= 4096 ? 4 : 3;
    size_t warps = kStageBudgetBytes / (geo.stages * row);
    if (warps < 1) {
        geo.stages = 2;
        warps = 1;
    }
    geo.warps_per_cta = (int)std::min<size_t>(warps, kDispatchMaxThreads / 32);
    geo.smem_bytes = align_up((size_t)geo.warps_per_cta * geo.stages * 8, 128) +
                     (size_t)geo.warps_per_cta * geo.stages * row;
    // CTAs resident per SM, limited by shared memory (228 KB per SM, 1 KB reserved per CTA)
    int per_sm = (int)std::max<size_t>(1, (228 * 1024) / (geo.smem_bytes + 1024));
    per_sm = std::min(per_sm, 2048 / (geo.warps_per_cta * 32));
    const long long need = (G + geo.warps_per_cta - 1) / geo.warps_per_cta;
    geo.ctas = (int)std::max<long long>(1, std::min<long long>((long long)num_sms * per_sm, need));
    return geo;
}

cudaError_t dispatch_prepare() {
    // Opt in to the full 227 KB of dynamic shared memory (per device).
    const int bytes = 227 * 1024;
    cudaError_t e = cudaFuncSetAttribute(dispatch_kernel<kModeNormal>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(dispatch_kernel<kModeCached>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(dispatch_kernel<kModeLowLatency>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    return e;
}

cudaError_t launch_dispatch(int mode, const DispatchParams& p, const DispatchGeometry& geo,
                            cudaStream_t stream) {
    if (p.G == 0) return cudaSuccess;
    switch (mode) {
        case kModeNormal: return launch_mode<kModeNormal>(p, geo, stream);
        case kModeCached: return launch_mode<kModeCached>(p, geo, stream);
        case kModeLowLatency: return launch_mode<kModeLowLatency>(p, geo, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ep
