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
// so slot(s, t, e) = #{(s', t') < (s, t) naming e}: an exclusive running count
// over the G tokens, one column per expert.  ll_scan_kernel computes all E
// columns in one decoupled-lookback pass and writes src_info (token index per
// slot), layout_range (first slot and count per source rank), the counts and a
// [G][K] slot map for the copy kernel (the dispatch kernel's packed mode).  No
// atomic decides an order, so the packing is deterministic.
//
// ll_combine_kernel: one warp per token.  Lane k finds the slot of its expert
// by binary search in src_info inside layout_range[e][s] (ascending token
// ids), the valid slots are ranked by (expert id, k), and the rows are reduced
// with an fp32 fused multiply-add chain in that order.

#include "common.cuh"
#include "kernels.h"

namespace ep {

namespace {

constexpr int kLLCombineThreads = 256;
constexpr int kLLCombineWarps = kLLCombineThreads / 32;
constexpr int kLLRowsPerGroup = 8;
constexpr int kLLWords = kLLTile / 32;
constexpr int kLLStride = kLLWords + 1;   // odd row stride: no shared-memory bank conflicts
constexpr unsigned long long kLLFlagAggregate = 1ull << 62;
constexpr unsigned long long kLLFlagInclusive = 2ull << 62;

__host__ __device__ inline size_t ll_scan_smem(int E) {
    return (size_t)E * kLLStride * sizeof(uint32_t) + (size_t)E * sizeof(int);
}

// One 256-token tile per block (ticket order).  Each thread owns one token:
// its experts set one bit each in the tile's [E][8]-word membership bitmap (a
// token naming an expert twice sets the same bit).  Thread e then publishes
// expert e's tile count and looks back over earlier tiles for the exclusive
// prefix (bounded wait); a member's slot is that prefix plus the members of the
// expert earlier in the tile.  Samples of the running counts at each source
// rank's first token go to `boundary`; the last tile to finish turns them into
// layout_range and the per-expert counts.
template <int kMaxK>
__global__ void __launch_bounds__(kLLTile)
ll_scan_kernel(const LLCountParams p) {
    extern __shared__ uint32_t ll_smem[];
    uint32_t* bits = ll_smem;                                       // [E][kLLStride]
    int* s_excl = reinterpret_cast<int*>(ll_smem + (size_t)p.E * kLLStride);  // [E]
    __shared__ int s_tile, s_last;
    const int tid = threadIdx.x;
    const int E = p.E;
    if (tid == 0) s_tile = atomicAdd(p.ticket, 1);
    for (int i = tid; i < E * kLLStride; i += kLLTile) bits[i] = 0;
    __syncthreads();
    const int tile = s_tile;
    const long long g0 = (long long)tile * kLLTile;
    const long long g = g0 + tid;
    const int w = tid >> 5, b = tid & 31;

    int64_t ids[kMaxK];
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) ids[k] = (g < p.G && k < p.K) ? __ldg(p.topk_idx + g * p.K + k) : -1;
    // a slot from or to a masked rank is not part of the exchange
    const int L = E / p.R;
    const bool src_masked = g < p.G && p.rank_mask[g / p.T] != 0;
    bool bad = false;
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) {
        const int64_t e = ids[k];
        if (e < -1 || e >= E) { bad = true; ids[k] = -1; continue; }
        if (e >= 0 && (src_masked || p.rank_mask[e / L] != 0)) ids[k] = -1;
        if (ids[k] >= 0) atomicOr(&bits[e * kLLStride + w], 1u << b);
    }
    if (bad) record_error(p.err, EP_ERR_BAD_TOPK);
    __syncthreads();

    for (int e = tid; e < E; e += kLLTile) {
        int agg = 0;
#pragma unroll
        for (int q = 0; q < kLLWords; ++q) agg += __popc(bits[e * kLLStride + q]);
        unsigned long long* mine = p.status + (size_t)tile * E + e;
        int excl = 0;
        if (tile == 0) {
            st_relaxed_u64(mine, kLLFlagInclusive | (unsigned)agg);
        } else {
            st_relaxed_u64(mine, kLLFlagAggregate | (unsigned)agg);
            int j = tile - 1;
            uint64_t t0 = 0;
            uint32_t spins = 0;
            while (j >= 0) {
                const unsigned long long v = ld_relaxed_u64(p.status + (size_t)j * E + e);
                const unsigned long long flag = v & (3ull << 62);
                if (flag == 0) {
                    if (spins == 0) t0 = globaltimer_ns();
                    ++spins;
                    if (spins > kWaitLimitIters ||
                        ((spins & 63u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs)) {
                        record_error(p.err, EP_ERR_TIMEOUT);
                        break;
                    }
                    continue;
                }
                excl += (int)(uint32_t)v;
                if (flag == kLLFlagInclusive) break;
                --j;
            }
            st_relaxed_u64(mine, kLLFlagInclusive | (unsigned)(excl + agg));
        }
        s_excl[e] = excl;
    }
    __syncthreads();

    const long long cap = p.ll_capacity;
    if (g < p.G) {
        const int t = (int)(g % p.T);
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) {
            const int64_t e = ids[k];
            if (e < 0) continue;
            const uint32_t* be = bits + e * kLLStride;
            int slot = s_excl[e] + __popc(be[w] & ((1u << b) - 1u));
            for (int q = 0; q < w; ++q) slot += __popc(be[q]);
            if (slot < cap) {
                p.slot_map[g * p.K + k] = slot;
                p.src_info[e * cap + slot] = t;
            } else {
                record_error(p.err, EP_ERR_CAPACITY);
            }
        }
    }

    // running counts at source starts s*T (s = 0..R; s*T == G belongs to the last tile)
    const bool last_tile = tile == p.num_tiles - 1;
    const int s_lo = (int)((g0 + p.T - 1) / p.T);
    const int s_hi = (int)min((long long)p.R, (g0 + kLLTile) / p.T);
    for (int s = s_lo; s <= s_hi; ++s) {
        const long long gb = (long long)s * p.T;
        const bool mine = (gb >= g0 && gb < g0 + kLLTile && gb < p.G) || (gb == p.G && last_tile);
        if (!mine) continue;
        const int rel = (int)(gb - g0);    // 0..256
        for (int e = tid; e < E; e += kLLTile) {
            const uint32_t* be = bits + e * kLLStride;
            int cnt = 0;
            for (int q = 0; q < (rel >> 5); ++q) cnt += __popc(be[q]);
            if ((rel >> 5) < kLLWords) cnt += __popc(be[rel >> 5] & ((1u << (rel & 31)) - 1u));
            p.boundary[(long long)s * E + e] = s_excl[e] + cnt;
        }
    }

    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(p.done, 1) == p.num_tiles - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // loads of each batch before its stores, so the L2 round trips overlap
    constexpr int kBatch = 8;
    const int nr = E * p.R;
    for (int i0 = 0; i0 < nr; i0 += kLLTile * kBatch) {
        int vb[kBatch], vn[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u * kLLTile + tid;   // i = e*R + s
            if (i < nr) {
                const int e = i / p.R, s = i % p.R;
                vb[u] = __ldcg(p.boundary + (long long)s * E + e);
                vn[u] = __ldcg(p.boundary + (long long)(s + 1) * E + e);
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u * kLLTile + tid;
            if (i < nr) {
                p.layout_range[(long long)i * 2 + 0] = vb[u];
                p.layout_range[(long long)i * 2 + 1] = vn[u] - vb[u];
            }
        }
    }
    for (int e = tid; e < E; e += kLLTile) p.packed_recv_count[e] = __ldcg(p.boundary + (long long)p.R * E + e);
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

template <int U, int kGroup = kLLRowsPerGroup>
__global__ void __launch_bounds__(kLLCombineThreads)
ll_combine_kernel(const LLCombineParams p) {
    __shared__ long long s_rows[kLLCombineWarps][32];
    __shared__ float s_w[kLLCombineWarps][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nvec = p.H / 8;
    const long long cap = p.ll_capacity;

    const long long wid = (long long)blockIdx.x * kLLCombineWarps + warp;
    const long long g = wid / p.splits;          // token
    const int part = (int)(wid % p.splits);      // column slice of its row
    if (g >= p.G) return;   // whole warp
    {
        const int s = (int)(g / p.T), t = (int)(g % p.T);
        const bool src_masked = p.rank_mask[s] != 0;   // warp-uniform: the token took no part
        long long e = -1;
        float w = 0.f;
        if (lane < p.K && !src_masked) {
            e = p.topk_idx[g * p.K + lane];
            w = p.topk_weights[g * p.K + lane];
        }
        bool valid = e >= 0 && e < p.E && p.rank_mask[(int)e / (p.E / p.R)] == 0;
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
        const int per = ((nvec + p.splits - 1) / p.splits + 31) / 32 * 32;
        const int clo = part * per, chi = min(nvec, clo + per);
        for (int c0 = clo; c0 < chi; c0 += 32 * U) {
            float acc[U][8];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[u][i] = 0.f;
            for (int i0 = 0; i0 < nv; i0 += kGroup) {
                uint4 v[kGroup][U];
#pragma unroll
                for (int i = 0; i < kGroup; ++i) {
                    if (i0 + i < nv) {
                        const uint4* src = reinterpret_cast<const uint4*>(p.y + s_rows[warp][i0 + i] * p.H);
#pragma unroll
                        for (int u = 0; u < U; ++u) {
                            const int c = c0 + lane + 32 * u;
                            if (c < chi) v[i][u] = ld_stream_v4(src + c);
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < kGroup; ++i) {
                    if (i0 + i < nv) {
                        const float wi = s_w[warp][i0 + i];
#pragma unroll
                        for (int u = 0; u < U; ++u)
                            if (c0 + lane + 32 * u < chi) fma_bf16x8(acc[u], wi, v[i][u]);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + lane + 32 * u;
                if (c >= chi) continue;
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

__global__ void set_mask_kernel(int* rank_mask, int rank, int value) { rank_mask[rank] = value; }

cudaError_t launch_set_mask(int* rank_mask, int rank, int value, cudaStream_t stream) {
    set_mask_kernel<<<1, 1, 0, stream>>>(rank_mask, rank, value);
    return cudaGetLastError();
}

cudaError_t ll_prepare(int E) {
    // opt in to large dynamic shared memory when E needs it
    const size_t smem = ll_scan_smem(E);
    if (smem <= 48 * 1024) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(ll_scan_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ll_scan_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ll_scan_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    return e;
}

cudaError_t launch_ll_count(const LLCountParams& p, cudaStream_t stream) {
    if (p.G == 0 || p.E == 0) return cudaSuccess;
    const size_t smem = ll_scan_smem(p.E);
    if (p.K <= 8)
        ll_scan_kernel<8><<<p.num_tiles, kLLTile, smem, stream>>>(p);
    else if (p.K <= 16)
        ll_scan_kernel<16><<<p.num_tiles, kLLTile, smem, stream>>>(p);
    else
        ll_scan_kernel<32><<<p.num_tiles, kLLTile, smem, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_ll_combine(const LLCombineParams& p, int num_sms, cudaStream_t stream) {
    if (p.G == 0) return cudaSuccess;
    (void)num_sms;
    const long long blocks = (p.G * p.splits + kLLCombineWarps - 1) / kLLCombineWarps;
    // 4 x 16-byte vectors per lane per row, groups of 4 rows (measured best on B200)
    ll_combine_kernel<4, 4><<<(unsigned)blocks, kLLCombineThreads, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace ep
