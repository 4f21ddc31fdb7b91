// Dispatch row scatter (normal, cached, low-latency packed, and its FP8 form).
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
//     metadata: local top-k ids, weights, and recv_src_idx;
//   * the sharded form is the normal form for virtual ranks spread over
//     several GPUs: destination d's rows and metadata go straight into the
//     receive buffers of the GPU hosting d (its own memory, or a peer's mapped
//     into this process), so the exchange happens inside the copy.
// Per token the HBM traffic is H*2 bytes read + fan-out * H*2 bytes written
// (fan-out * (H + H/32) bytes in the FP8 packed form, ll_fp8_copy_kernel below).

#include <algorithm>

#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace ep {

namespace {

constexpr int kDispatchThreads = 256;
constexpr int kVecPerLane = 28;   // 16-byte vectors held per lane per pass

// Packed (low-latency) destination of lane k's top-k slot of token g: the row
// of its expert's list, or -1 (unused slot, a repeated expert after its first
// slot, a masked source or destination rank, or a slot past the capacity,
// which is recorded).  Waits (programmatic dependent launch) for the kernel
// before it -- the slot scan, or the direct-slot ranking -- before reading what
// that kernel writes; topk_idx and the rank mask are inputs of the call.
//
// Slot scan: the slot is the scan's slot map entry.  Direct slots (sources of
// at most kLLDirectMaxT tokens): slot = the tokens of earlier sources naming
// the expert (a sum over the ranking's per-source counts) + the token's rank
// among its own source's tokens naming it (the ranking's within); the warp of
// column slice 0 writes the slot map (a hint for the low-latency combine) and
// src_info.
__device__ __forceinline__ long long packed_row(const DispatchParams& p, long long g, int lane, int part) {
    const int L = p.E / p.R;
    const int s = (int)(g / p.T), t = (int)(g % p.T);
    long long e = -1;
    if (lane < p.K) e = p.topk_idx[g * p.K + lane];
    // slots from or to a masked rank are not sent
    const bool live = e >= 0 && e < p.E && p.rank_mask[s] == 0 && p.rank_mask[(int)e / L] == 0;
    bool first = live;
    for (int k = 0; k < p.K; ++k) {   // a repeated expert is sent once
        const long long ek = __shfl_sync(kFullMask, e, k);
        if (k < lane && ek == e) first = false;
    }
    pdl_wait();
    int slot = -1;
    if (live) {
        if (p.ll_cnt != nullptr) {
            slot = p.ll_within[g * p.K + lane];
            const int* col = p.ll_cnt + e;
            int base = 0;
#pragma unroll 4
            for (int s2 = 0; s2 < s; ++s2) base += col[(long long)s2 * p.E];
            slot += base;
            if (part == 0 && slot >= 0 && slot < p.ll_capacity) {
                p.slot_map[g * p.K + lane] = slot;
                if (first) p.ll_src_info[e * p.ll_capacity + slot] = t;
            }
        } else if (first) {
            slot = p.slot_map[g * p.K + lane];
        }
    }
    long long row = -1;
    if (first) {
        if (slot >= 0 && slot < p.ll_capacity)
            row = e * p.ll_capacity + slot;
        else
            record_error(p.err, EP_ERR_CAPACITY);
    }
    return row;
}

// Direct slots: the per-expert tables of the packed lists from the ranking's
// per-source counts -- layout_range[e][s] = (tokens of earlier sources, tokens
// of s) and the list length -- one expert per warp (an exclusive scan over the
// lanes, lane s holding source s), spread over all the copy's warps.
__device__ __forceinline__ void ll_direct_tables(const DispatchParams& p, long long wid, int lane) {
    const long long nwarps = p.G * p.splits;
    for (long long e = wid; e < p.E; e += nwarps) {
        const int c = lane < p.R ? p.ll_cnt[(long long)lane * p.E + e] : 0;
        int incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(kFullMask, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane < p.R) {
            p.ll_layout_range[(e * p.R + lane) * 2 + 0] = incl - c;
            p.ll_layout_range[(e * p.R + lane) * 2 + 1] = c;
        }
        if (lane == p.R - 1) p.ll_count[e] = incl;
    }
}

#ifndef EP_LL_COPY_VEC
#define EP_LL_COPY_VEC 28
#endif
#ifndef EP_LL_COPY_MINB
#define EP_LL_COPY_MINB 2
#endif
// The packed (low-latency) copy runs one-warp blocks: with few tokens its 2 x G
// warps fill 1.7 waves of the GPU, and single-warp blocks let the scheduler hand
// out the second wave warp by warp (measured on B200, LL shape: step 90.3 vs
// 91.2 us for 8-warp blocks; 2- and 4-warp blocks 91.2).
// The bf16 packed copy writes with the default (write-back) policy, the others
// with streaming (evict-first) stores: the packed rows are read again right
// away (by the experts; in the benchmark's step by the low-latency combine),
// and those still in L2 are read from there (measured on B200, LL shape: step
// 84.9 vs 88.3 us, combine 41.5 vs 45.9 us; for the FP8 copy the default
// policy measured 0.5 us slower, its codes not being read by the combine).
#ifndef EP_LL_STORE_STREAM
#define EP_LL_STORE_STREAM 0
#endif
#ifndef EP_LL_COPY_THREADS
#define EP_LL_COPY_THREADS 32
#endif

template <int kMode, int kVec = kVecPerLane, int kMinBlocks = 2, int kThreads = kDispatchThreads>
__global__ void __launch_bounds__(kThreads, kMinBlocks)
dispatch_kernel(const DispatchParams p) {
    constexpr int kWarps = kThreads / 32;
    __shared__ long long s_rows[kWarps][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long wid = (long long)blockIdx.x * kWarps + warp;
    const long long g = wid / p.splits;          // token
    const int part = (int)(wid % p.splits);      // column slice of its row
    if (g >= p.G) return;   // whole warp

    // this warp's column slice: whole 32-vector strides
    const int nvec = p.H / 8;
    const int per = ((nvec + p.splits - 1) / p.splits + 31) / 32 * 32;
    const int lo = part * per, hi = min(nvec, lo + per);
    const uint4* src = reinterpret_cast<const uint4*>(p.x + g * p.H);
    uint4 v[kVec];
    // The sharded form loads the first pass of its slice at once, before it reads
    // the handle (measured faster).  The normal and packed forms are launched
    // right behind the handle / slot kernel and may start before it ends: they
    // pull the slice (an input of the call, never written by that kernel) into L2
    // meanwhile and wait for that kernel (the packed form inside packed_row);
    // holding the slice in registers across the wait measured slower on B200
    // (DSv3 dispatch 459 vs 452 us).
    constexpr bool kPreload = kMode == kModeSharded;
    if constexpr (kPreload) {
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
            const int c = lo + lane + 32 * u;
            if (c < hi) v[u] = ld_nc_v4(src + c);
        }
    }
    if constexpr (kMode == kModeNormal || kMode == kModeLowLatency) {
        if (lane == 0 && lo < hi) prefetch_l2(src + lo, (uint32_t)(hi - lo) * 16u);
    }
    if constexpr (kMode == kModeNormal) pdl_wait();

    constexpr bool kPacked = kMode == kModeLowLatency;
    long long row = -1;
    if (kPacked) {
        row = packed_row(p, g, lane, part);
        if (p.ll_cnt != nullptr) ll_direct_tables(p, wid, lane);
    } else if (lane < p.R) {
        const int h = p.send_head[g * p.R + lane];
        if (h >= 0) {
            row = (kMode == kModeSharded ? p.dst_offset[lane] : p.recv_rank_offset[lane]) + h;
            if (row >= p.recv_capacity) {
                record_error(p.err, EP_ERR_CAPACITY);
                row = -1;
            }
        }
    }
    // sharded: lane d's destination buffers are those of shard d / ranks_per_shard
    const int shard = (kMode == kModeSharded && row >= 0) ? lane / p.ranks_per_shard : 0;

    if ((kMode == kModeNormal || kMode == kModeSharded) && part == 0) {
        int* r_src = p.recv_src_idx;
        int64_t* r_idx = p.recv_topk_idx;
        float* r_w = p.recv_topk_weights;
        if (kMode == kModeSharded) {
            r_src = p.shard_src[shard];
            r_idx = p.shard_idx[shard];
            r_w = p.shard_w[shard];
        }
        long long e = -1;
        float w = 0.f;
        if (lane < p.K) {
            e = p.topk_idx[g * p.K + lane];
            if (p.topk_weights != nullptr) w = p.topk_weights[g * p.K + lane];
        }
        if (row >= 0 && r_src != nullptr) r_src[row] = (int)(g % p.T);
        for (int k = 0; k < p.K; ++k) {
            const long long ek = __shfl_sync(kFullMask, e, k);
            const float wk = __shfl_sync(kFullMask, w, k);
            if (row >= 0) {
                const bool here = ek >= 0 && ek < p.E && (int)ek / p.L == lane;
                if (r_idx != nullptr) r_idx[row * p.K + k] = here ? (long long)((int)ek % p.L) : -1LL;
                if (r_w != nullptr) r_w[row * p.K + k] = here ? wk : 0.f;
            }
        }
    }
    if (kMode == kModeNormal && p.recv_x == nullptr) return;   // metadata only (the loaded row unused)
    if (kMode == kModeSharded && row >= 0)                     // keep the row's address
        row = (long long)reinterpret_cast<uintptr_t>(p.shard_rows[shard] + row * p.H);

    const uint32_t m = __ballot_sync(kFullMask, row >= 0);
    const int f = __popc(m);
    if (row >= 0) s_rows[warp][__popc(m & lanemask_lt())] = row;
    __syncwarp();

    for (int c0 = lo; c0 < hi; c0 += 32 * kVec) {
        if (!kPreload || c0 != lo) {
#pragma unroll
            for (int u = 0; u < kVec; ++u) {
                const int c = c0 + lane + 32 * u;
                if (c < hi) v[u] = ld_nc_v4(src + c);
            }
        }
        for (int i = 0; i < f; ++i) {
            uint4* dst = kMode == kModeSharded
                             ? reinterpret_cast<uint4*>(static_cast<uintptr_t>(s_rows[warp][i]))
                             : reinterpret_cast<uint4*>(p.recv_x + s_rows[warp][i] * p.H);
#pragma unroll
            for (int u = 0; u < kVec; ++u) {
                const int c = c0 + lane + 32 * u;
                if (c < hi) {
                    if (kMode == kModeLowLatency && !EP_LL_STORE_STREAM)
                        st_v4(dst + c, v[u]);
                    else
                        st_stream_v4(dst + c, v[u]);
                }
            }
        }
    }
    // sharded: rows and metadata may sit in other GPUs' memory; make them
    // visible system-wide before the kernel ends (a peer reads them after the
    // caller's cross-GPU barrier)
    if (kMode == kModeSharded) __threadfence_system();
}

// ---------------------------------------------------------------- FP8 form
//
// "DeepEP Buffer Class API ...", "Low-Latency Inference with FP8": the packed
// low-latency rows as OCP E4M3 codes with one fp32 scale per token per 128
// hidden channels (scale = amax / 448, code = E4M3(x * (448 / amax)), each an
// fp32 operation rounded to nearest even; E4M3 nearest even, saturating; an
// all-zero block has scale 1 and zero codes).
//
// The row is cut into 512-channel steps and each warp (a one-warp block) takes
// a slice of kFp8Steps steps -- seven warps per 7168-wide row -- and loads all
// of it at once.  In a step lane l holds channels [16 l, 16 l + 16) (one 32-byte
// load), so the 8 lanes of an aligned group hold one 128-channel block.  A
// block's amax is a max over bf16 magnitudes, whose bit patterns order like the
// values: a packed bf16x2 max-of-magnitudes over the lane's 8 words, then three
// xor shuffles.  Lane j takes the amax of block j of the slice and computes its
// scale and 448 / amax (one division pair per block); each step's lanes fetch
// their block's multiplier back with a shuffle.  A lane turns its 16 values into
// 16 code bytes (one 16-byte store per destination row and step, 512 B per warp
// instruction), and lane j stores block j's scale, so a destination row gets
// the slice's scales from one coalesced store.  The slice is loaded and
// converted before the warp waits for the slots (the row is an input of the
// call).  Traffic per token: H*2 bytes read, fan-out * (H + H/32) bytes written.
//
// Measured on B200 (16 ranks, H 7168, top-8): 28.8 us at 128 tokens/rank
// against 29.4 for warps walking whole rows in two-step passes, 51.8 against
// 61.0 at 256 tokens/rank; one-step slices 34.1 us, seven-step slices 33.3 us,
// two-step slices in 4-warp blocks 29.1 us.
constexpr int kFp8Steps = 2;                        // 512-channel steps per warp
constexpr int kFp8LanesPerBlock = kFp8Block / 16;   // 8 lanes x 16 channels
constexpr int kFp8MinBlocks = 32;                   // one-warp blocks per SM (64 registers)
static_assert(kFp8LanesPerBlock == 8, "a block is 8 lanes of 16 channels");
static_assert(kFp8Steps * 4 <= 32, "one lane per block of the slice");

// largest magnitude of each bf16 half of x and y (the result's sign bits are
// not meaningful); a NaN half yields the other operand's half
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t x, uint32_t y) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(x), "r"(y));
    return d;
}

// E4M3 codes of the 4 channels of bf16 pairs w0, w1, each multiplied by inv in
// fp32 (rounded to nearest even) first
__device__ __forceinline__ uint32_t e4m3x4_scaled(uint32_t w0, uint32_t w1, float inv) {
    const float x0 = __fmul_rn(bf16_lo(w0), inv), x1 = __fmul_rn(bf16_hi(w0), inv);
    const float x2 = __fmul_rn(bf16_lo(w1), inv), x3 = __fmul_rn(bf16_hi(w1), inv);
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(x0, x1), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(x2, x3), __NV_SATFINITE, __NV_E4M3);
    return (uint32_t)lo | ((uint32_t)hi << 16);
}

__global__ void __launch_bounds__(32, kFp8MinBlocks)
ll_fp8_copy_kernel(const DispatchParams p) {
    __shared__ long long s_rows[32];
    const int lane = threadIdx.x;
    const long long wid = blockIdx.x;
    const long long g = wid / p.splits;          // token
    const int part = (int)(wid % p.splits);      // slice of its row (whole steps)
    if (g >= p.G) return;

    const int nvec = p.H / 8;                    // 16-byte vectors (8 channels) per row
    const int nstep = (nvec + 63) / 64;
    const int per = (nstep + p.splits - 1) / p.splits;   // <= kFp8Steps (launch_ll_copy_fp8)
    const int s_lo = part * per, s_hi = min(nstep, s_lo + per);
    const uint4* src = reinterpret_cast<const uint4*>(p.x + g * p.H);
    uint4 a[kFp8Steps], b[kFp8Steps];
#pragma unroll
    for (int k = 0; k < kFp8Steps; ++k) {
        const int c = (s_lo + k) * 64 + 2 * lane;
        if (s_lo + k < s_hi && c < nvec) ld_nc_v8(src + c, a[k], b[k]);
    }
    // block amax as a bf16 bit pattern; a half that is all NaN counts as 0, as a
    // float max that skips NaN would have it
    uint32_t amax_bits[kFp8Steps];
#pragma unroll
    for (int k = 0; k < kFp8Steps; ++k) {
        uint32_t m = 0;
        if (s_lo + k < s_hi && (s_lo + k) * 64 + 2 * lane < nvec) {
            m = absmax_bf16x2(a[k].x, a[k].y);
            m = absmax_bf16x2(m, a[k].z);
            m = absmax_bf16x2(m, a[k].w);
            m = absmax_bf16x2(m, b[k].x);
            m = absmax_bf16x2(m, b[k].y);
            m = absmax_bf16x2(m, b[k].z);
            m = absmax_bf16x2(m, b[k].w);
        }
        uint32_t lo = m & 0x7fffu, hi = (m >> 16) & 0x7fffu;
        lo = lo > 0x7f80u ? 0u : lo;
        hi = hi > 0x7f80u ? 0u : hi;
        uint32_t v = max(lo, hi);
        v = max(v, __shfl_xor_sync(kFullMask, v, 1));
        v = max(v, __shfl_xor_sync(kFullMask, v, 2));
        v = max(v, __shfl_xor_sync(kFullMask, v, 4));
        amax_bits[k] = v;
    }
    // lane j: block j of the slice (step j / 4, block j % 4 of the step)
    uint32_t mine = 0;
#pragma unroll
    for (int k = 0; k < kFp8Steps; ++k) {
        const uint32_t v = __shfl_sync(kFullMask, amax_bits[k], (lane & 3) * kFp8LanesPerBlock);
        if ((lane >> 2) == k) mine = v;
    }
    const float amax = __uint_as_float(mine << 16);
    const float my_scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
    const float my_inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 0.f;
    uint4 codes[kFp8Steps];
#pragma unroll
    for (int k = 0; k < kFp8Steps; ++k) {
        const float inv = __shfl_sync(kFullMask, my_inv, k * 4 + lane / kFp8LanesPerBlock);
        codes[k] = make_uint4(e4m3x4_scaled(a[k].x, a[k].y, inv), e4m3x4_scaled(a[k].z, a[k].w, inv),
                              e4m3x4_scaled(b[k].x, b[k].y, inv), e4m3x4_scaled(b[k].z, b[k].w, inv));
    }

    const long long row = packed_row(p, g, lane, part);
    if (p.ll_cnt != nullptr) ll_direct_tables(p, wid, lane);
    const uint32_t m = __ballot_sync(kFullMask, row >= 0);
    const int f = __popc(m);
    if (row >= 0) s_rows[__popc(m & lanemask_lt())] = row;
    __syncwarp();

    const int nblk = p.H / kFp8Block;
    const int nb = min((s_hi - s_lo) * 4, nblk - s_lo * 4);   // blocks of the slice
    for (int i = 0; i < f; ++i) {
        const long long r = s_rows[i];
        uint8_t* dst = p.recv_fp8 + r * p.H;
#pragma unroll
        for (int k = 0; k < kFp8Steps; ++k) {
            const int c = (s_lo + k) * 64 + 2 * lane;
            if (s_lo + k < s_hi && c < nvec) st_stream_v4(reinterpret_cast<uint4*>(dst + (long long)c * 8), codes[k]);
        }
        if (lane < nb) __stcs(p.recv_scales + r * nblk + s_lo * 4 + lane, my_scale);
    }
}

cudaError_t launch_ll_copy_fp8(DispatchParams p, cudaStream_t stream, bool after_scan) {
    const int nstep = (p.H / 8 + 63) / 64;
    // slices of at most kFp8Steps steps; more (down to one step) when there are
    // too few rows to give the GPU ~8 warps per SM
    const long long want = (long long)p.num_sms * 8;
    p.splits = (int)min((long long)nstep,
                        max((long long)(nstep + kFp8Steps - 1) / kFp8Steps, (want + p.G - 1) / p.G));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.G * p.splits));
    cfg.blockDim = dim3(32);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_scan ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, ll_fp8_copy_kernel, p);
}

template <int kMode>
cudaError_t launch_mode(const DispatchParams& p, cudaStream_t stream, bool after_scan) {
    constexpr int kThreads = kMode == kModeLowLatency ? EP_LL_COPY_THREADS : kDispatchThreads;
    // the sharded form holds its first pass across its handle reads: 14 vectors per
    // lane (one pass of a 7168-wide row in two column slices) keep that within the
    // register budget
    constexpr int kVec = kMode == kModeLowLatency ? EP_LL_COPY_VEC : (kMode == kModeSharded ? 14 : kVecPerLane);
    constexpr int kMinB = kMode == kModeLowLatency ? EP_LL_COPY_MINB * (kDispatchThreads / kThreads) : 2;
    const long long blocks = (p.G * p.splits + kThreads / 32 - 1) / (kThreads / 32);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = after_scan ? 1 : 0;   // may overlap the scan's tail (see pdl_wait above)
    return cudaLaunchKernelEx(&cfg, dispatch_kernel<kMode, kVec, kMinB, kThreads>, p);
}

}  // namespace

cudaError_t launch_dispatch(int mode, const DispatchParams& p, cudaStream_t stream, bool after_scan) {
    if (p.G == 0) return cudaSuccess;
    switch (mode) {
        case kModeNormal: return launch_mode<kModeNormal>(p, stream, after_scan);
        case kModeCached: return launch_mode<kModeCached>(p, stream, false);
        case kModeLowLatency: return launch_mode<kModeLowLatency>(p, stream, after_scan);
        case kModeLowLatencyFp8: return launch_ll_copy_fp8(p, stream, after_scan);
        case kModeSharded: return launch_mode<kModeSharded>(p, stream, false);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ep
