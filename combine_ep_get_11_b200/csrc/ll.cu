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
// over the G tokens, one column per expert.  ll_slot_kernel computes all E
// columns in one decoupled-lookback pass over tiles of at most 256 tokens of
// one source rank each, and writes src_info (token index per slot),
// layout_range (first slot and count per source rank), the counts and a [G][K]
// slot map for the copy kernel (the dispatch kernel's packed mode).  No atomic
// decides an order, so the packing is deterministic.
//
// ll_combine_kernel: one warp per token.  Lane k finds the slot of its expert:
// the slot the last low-latency dispatch on the context gave (token, k), if the
// handle confirms it (inside layout_range[e][s] and holding the token), else by
// binary search in src_info inside layout_range[e][s] (ascending token ids), the valid slots are ranked by (expert id, k), and the rows are reduced
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
constexpr int kLLWindow = 16;             // predecessor tiles read at once in the lookback
// Tile status word: count in bits 0-31, flag in bits 32-33, call epoch in bits 34-63.
constexpr unsigned long long kLLFlagAggregate = 1ull << 32;
constexpr unsigned long long kLLFlagInclusive = 2ull << 32;
constexpr unsigned long long kLLFlagMask = 3ull << 32;
constexpr unsigned long long kLLTagMask = ~0ull << 34;
constexpr int kLLEpochShift = 34;

__host__ __device__ inline size_t ll_slot_smem(int E) {
    return (size_t)E * kLLStride * sizeof(uint32_t)   // membership bitmap
           + (size_t)E * sizeof(int)                  // exclusive prefix per expert
           + (size_t)E * kLLWords                     // members before each word (<= 224)
           + (size_t)E;                               // expert on a masked rank
}

__device__ __forceinline__ bool ll_published(unsigned long long v, unsigned long long tag) {
    return (v & kLLTagMask) == tag && (v & kLLFlagMask) != 0;
}

// Tiles: source rank s is cut into m = ceil(T/256) tiles of at most 256 of its
// tokens, numbered s*m + j in token order.  Blocks take tickets from one 64-bit
// counter that is never reset: ticket = call * num_tiles + tile, so a tile
// only waits on tiles that already started, and the call number tags every
// status word (words left by an earlier call never match; nothing is cleared
// between calls).  Each thread owns one token: its experts set one bit each in
// the tile's [E][8]-word membership bitmap (a token naming an expert twice
// sets the same bit).  Thread e then publishes expert e's tile count and looks
// back over earlier tiles, 16 status words loaded at once per round and summed
// up to the first inclusive prefix (while a word before it is unpublished, the
// window is re-read, with a bounded wait).  A member's slot is that prefix
// plus the members of the expert earlier in the tile.  The first tile of a
// source writes layout_range's start; its last tile the count (reading the
// start from a tagged word when the source spans several tiles); the last tile
// of all the per-expert totals.
template <int kMaxK>
__global__ void __launch_bounds__(kLLTile, 1)
ll_slot_kernel(const LLCountParams p) {
    extern __shared__ uint32_t ll_smem[];
    const int E = p.E;
    uint32_t* bits = ll_smem;                                                 // [E][kLLStride]
    int* s_excl = reinterpret_cast<int*>(bits + (size_t)E * kLLStride);       // [E]
    uint8_t* s_wpref = reinterpret_cast<uint8_t*>(s_excl + E);                // [E][kLLWords]
    uint8_t* s_dead = s_wpref + (size_t)E * kLLWords;                         // [E]
    __shared__ int s_tile;
    __shared__ unsigned long long s_tag;
    const int tid = threadIdx.x;
    pdl_wait();                // everything before this kernel has completed ...
    pdl_launch_dependents();   // ... so the packed copy may start prefetching its rows
    if (tid == 0) {
        const unsigned long long tk = atomicAdd(p.ticket, 1ull);
        s_tile = (int)(tk % (unsigned long long)p.num_tiles);
        s_tag = (tk / (unsigned long long)p.num_tiles + 1) << kLLEpochShift;   // never 0
    }
    const int lane = tid & 31;   // masked ranks (R <= 32): one load per lane, in every warp
    const uint32_t mbits = __ballot_sync(kFullMask, lane < p.R && p.rank_mask[lane] != 0);
    const int L = E / p.R;
    for (int e = tid; e < E; e += kLLTile) {
#pragma unroll
        for (int q = 0; q < kLLStride; ++q) bits[e * kLLStride + q] = 0;
        s_dead[e] = (uint8_t)((mbits >> (e / L)) & 1u);
    }
    __syncthreads();
    const int tile = s_tile;
    const unsigned long long tag = s_tag;
    const int m = p.tiles_per_src;
    const int s = tile / m, j = tile - s * m;
    const int t = j * kLLTile + tid;                        // token of this thread in source s
    const int n = min(kLLTile, p.T - j * kLLTile);          // tokens in the tile
    const long long g = (long long)s * p.T + t;
    const bool src_live = ((mbits >> s) & 1u) == 0;        // a masked rank sends nothing
    const int w = tid >> 5, b = tid & 31;

    int ids[kMaxK];
    bool bad = false;
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) {
        const int64_t e = (tid < n && k < p.K) ? __ldg(p.topk_idx + g * p.K + k) : -1;
        bad |= e < -1 || e >= E;
        ids[k] = (e >= 0 && e < E && src_live && !s_dead[(int)e]) ? (int)e : -1;
    }
    if (bad) record_error(p.err, EP_ERR_BAD_TOPK);
#pragma unroll
    for (int k = 0; k < kMaxK; ++k)
        if (ids[k] >= 0) atomicOr(&bits[ids[k] * kLLStride + w], 1u << b);
    __syncthreads();

    const bool last_of_src = j == m - 1, last_tile = tile == p.num_tiles - 1;
    for (int e = tid; e < E; e += kLLTile) {
        int agg = 0;
#pragma unroll
        for (int q = 0; q < kLLWords; ++q) {
            s_wpref[e * kLLWords + q] = (uint8_t)agg;
            agg += __popc(bits[e * kLLStride + q]);
        }
        unsigned long long* mine = p.status + (size_t)tile * E + e;
        long long excl = 0;
        if (tile == 0) {
            st_relaxed_u64(mine, tag | kLLFlagInclusive | (unsigned)agg);
        } else {
            st_relaxed_u64(mine, tag | kLLFlagAggregate | (unsigned)agg);
            int top = tile - 1;             // newest tile of the current window
            bool found = false;
            uint64_t t0 = 0;
            uint32_t spins = 0;
            while (top >= 0 && !found) {
                const int cnt = min(kLLWindow, top + 1);
                unsigned long long v[kLLWindow];
                bool ok = false;
                int take = 0;
                for (;;) {
#pragma unroll
                    for (int u = 0; u < kLLWindow; ++u)
                        v[u] = u < cnt ? ld_relaxed_u64(p.status + (size_t)(top - u) * E + e) : 0ull;
                    // words are needed only up to the first inclusive one
                    ok = true;
                    found = false;
                    take = cnt;
#pragma unroll
                    for (int u = 0; u < kLLWindow; ++u) {
                        if (u < take) {
                            if (!ll_published(v[u], tag)) {
                                ok = false;
                                take = u;
                            } else if ((v[u] & kLLFlagMask) == kLLFlagInclusive) {
                                found = true;
                                take = u + 1;
                            }
                        }
                    }
                    if (ok) break;
                    if (spins == 0) t0 = globaltimer_ns();
                    ++spins;
                    if (spins > kWaitLimitIters ||
                        ((spins & 63u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs)) {
                        record_error(p.err, EP_ERR_TIMEOUT);
                        break;
                    }
                }
                if (!ok) break;
#pragma unroll
                for (int u = 0; u < kLLWindow; ++u)
                    if (u < take) excl += (uint32_t)v[u];
                top -= cnt;
            }
            st_relaxed_u64(mine, tag | kLLFlagInclusive | (unsigned)(excl + agg));
        }
        s_excl[e] = (int)excl;

        // layout_range[e][s] = (first slot of source s, its count); the per-expert totals
        int* lr = p.layout_range + ((long long)e * p.R + s) * 2;
        long long begin = excl;
        if (j == 0) {
            lr[0] = (int)excl;
            if (m > 1) st_relaxed_u64(p.src_begin + (size_t)s * E + e, tag | kLLFlagInclusive | (unsigned)excl);
        } else if (last_of_src) {   // the source's first tile started earlier: bounded wait for its start
            unsigned long long v = ld_relaxed_u64(p.src_begin + (size_t)s * E + e);
            uint32_t sp = 0;
            uint64_t ts = 0;
            while (!ll_published(v, tag)) {
                if (sp == 0) ts = globaltimer_ns();
                ++sp;
                if (sp > kWaitLimitIters || ((sp & 63u) == 0 && globaltimer_ns() - ts > kWaitLimitNs)) {
                    record_error(p.err, EP_ERR_TIMEOUT);
                    break;
                }
                v = ld_relaxed_u64(p.src_begin + (size_t)s * E + e);
            }
            begin = (uint32_t)v;
        }
        if (last_of_src) lr[1] = (int)(excl + agg - begin);
        if (last_tile) p.packed_recv_count[e] = (int)(excl + agg);
    }
    __syncthreads();

    if (tid < n) {
        const long long cap = p.ll_capacity;
        const uint32_t below = (1u << b) - 1u;
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) {
            const int e = ids[k];
            if (e < 0) continue;
            const int slot = s_excl[e] + s_wpref[e * kLLWords + w] + __popc(bits[e * kLLStride + w] & below);
            if (slot < cap) {
                p.slot_map[g * p.K + k] = slot;
                p.src_info[e * cap + slot] = t;
            } else {
                record_error(p.err, EP_ERR_CAPACITY);
            }
        }
    }
}

// Direct slots, ranking part: block s holds the tokens of source s, one per
// thread.  Each token sets one bit per expert it names in a [E][8]-word
// membership bitmap (a token naming an expert twice sets the same bit; tokens
// of a masked source and experts of a masked rank set nothing).  Thread e then
// stores expert e's count for the source, and each token's within for slot k is
// the members of its expert before it: the bitmap words before its own plus the
// bits below it in its word.  No block waits on another; the copy kernel adds
// the earlier sources' counts.
template <int kMaxK>
__global__ void __launch_bounds__(kLLTile)
ll_rank_kernel(const LLRankParams p) {
    extern __shared__ uint32_t rk_smem[];
    const int E = p.E;
    uint32_t* bits = rk_smem;                                                 // [E][kLLStride]
    uint8_t* s_wpref = reinterpret_cast<uint8_t*>(bits + (size_t)E * kLLStride);   // [E][kLLWords]
    pdl_wait();                      // everything before this kernel has completed ...
    pdl_launch_dependents();         // ... so the copy may start reading its rows
    const int s = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const int L = E / p.R;
    const int w = tid >> 5, b = lane;
    const long long g = (long long)s * p.T + tid;
    // the token's ids and the rank mask are independent loads: issue both before using either
    int64_t raw[kMaxK];
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) raw[k] = (tid < p.T && k < p.K) ? __ldg(p.topk_idx + g * p.K + k) : -1;
    const int mask_lane = lane < p.R ? p.rank_mask[lane] : 0;
    for (int e = tid; e < E; e += kLLTile) {
#pragma unroll
        for (int q = 0; q < kLLStride; ++q) bits[e * kLLStride + q] = 0;
    }
    const uint32_t mbits = __ballot_sync(kFullMask, mask_lane != 0);
    const bool src_live = ((mbits >> s) & 1u) == 0;
    int ids[kMaxK];
    bool bad = false;
#pragma unroll
    for (int k = 0; k < kMaxK; ++k) {
        const int64_t e = raw[k];
        bad |= e < -1 || e >= E;
        ids[k] = (e >= 0 && e < E && src_live && ((mbits >> ((int)e / L)) & 1u) == 0) ? (int)e : -1;
    }
    __syncthreads();   // the bitmap is clear
    if (bad) record_error(p.err, EP_ERR_BAD_TOPK);
#pragma unroll
    for (int k = 0; k < kMaxK; ++k)
        if (ids[k] >= 0) atomicOr(&bits[ids[k] * kLLStride + w], 1u << b);
    __syncthreads();
    for (int e = tid; e < E; e += kLLTile) {
        int agg = 0;
#pragma unroll
        for (int q = 0; q < kLLWords; ++q) {
            s_wpref[e * kLLWords + q] = (uint8_t)agg;
            agg += __popc(bits[e * kLLStride + q]);
        }
        p.cnt[(size_t)s * E + e] = agg;
    }
    __syncthreads();
    if (tid < p.T) {
        const uint32_t below = (1u << b) - 1u;
#pragma unroll
        for (int k = 0; k < kMaxK; ++k) {
            if (k >= p.K) break;
            const int e = ids[k];
            p.within[g * p.K + k] =
                e >= 0 ? (int)s_wpref[e * kLLWords + w] + __popc(bits[e * kLLStride + w] & below) : -1;
        }
    }
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
    pdl_wait();   // (launched with programmatic serialization: reads nothing before this)
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
        int hint = -1;
        if (lane < p.K && !src_masked) {
            e = p.topk_idx[g * p.K + lane];
            w = p.topk_weights[g * p.K + lane];
            if (p.slot_hint != nullptr) hint = p.slot_hint[g * p.K + lane];
        }
        bool valid = e >= 0 && e < p.E && p.rank_mask[(int)e / (p.E / p.R)] == 0;
        long long row = -1;
        if (valid) {
            const int* range = p.layout_range + ((long long)e * p.R + s) * 2;
            const int* info = p.src_info + e * cap;
            // the slot the last dispatch gave (token, k), if it is this token's
            // slot under this handle: inside source s's range and holding t (a
            // token appears once per list, so that slot is the one)
            const int hint_t = (hint >= 0 && hint < cap) ? info[hint] : -1;
            int lo = max(range[0], 0);
            const int end = (int)min((long long)lo + max(range[1], 0), cap);
            int slot = -1;
            if (hint >= lo && hint < end && hint_t == t) {
                slot = hint;
            } else {   // binary search of t in the source's ascending token ids
                int hi = end;
                while (lo < hi) {
                    const int mid = (lo + hi) >> 1;
                    if (info[mid] < t) lo = mid + 1; else hi = mid;
                }
                if (lo < end && info[lo] == t) slot = lo;
            }
            if (slot >= 0) {
                row = e * cap + slot;
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

__host__ __device__ inline size_t ll_rank_smem(int E) {
    return (size_t)E * kLLStride * sizeof(uint32_t) + (size_t)E * kLLWords;
}

cudaError_t launch_ll_rank(const LLRankParams& p, cudaStream_t stream) {
    if (p.R == 0 || p.E == 0) return cudaSuccess;
    const size_t smem = ll_rank_smem(p.E);
    if (p.K <= 8) return launch_pdl(ll_rank_kernel<8>, dim3(p.R), dim3(kLLTile), smem, stream, p);
    if (p.K <= 16) return launch_pdl(ll_rank_kernel<16>, dim3(p.R), dim3(kLLTile), smem, stream, p);
    return launch_pdl(ll_rank_kernel<32>, dim3(p.R), dim3(kLLTile), smem, stream, p);
}

cudaError_t ll_prepare(int E) {
    // opt in to large dynamic shared memory when E needs it
    const size_t smem = ll_slot_smem(E);
    if (smem <= 48 * 1024) return cudaSuccess;
    cudaError_t e = cudaFuncSetAttribute(ll_slot_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ll_slot_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ll_slot_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int rsmem = (int)ll_rank_smem(E);
    if (e == cudaSuccess && rsmem > 48 * 1024)
        e = cudaFuncSetAttribute(ll_rank_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, rsmem);
    if (e == cudaSuccess && rsmem > 48 * 1024)
        e = cudaFuncSetAttribute(ll_rank_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, rsmem);
    if (e == cudaSuccess && rsmem > 48 * 1024)
        e = cudaFuncSetAttribute(ll_rank_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, rsmem);
    return e;
}

cudaError_t launch_ll_count(const LLCountParams& p, cudaStream_t stream) {
    if (p.G == 0 || p.E == 0) return cudaSuccess;
    const size_t smem = ll_slot_smem(p.E);
    if (p.K <= 8) return launch_pdl(ll_slot_kernel<8>, dim3(p.num_tiles), dim3(kLLTile), smem, stream, p);
    if (p.K <= 16) return launch_pdl(ll_slot_kernel<16>, dim3(p.num_tiles), dim3(kLLTile), smem, stream, p);
    return launch_pdl(ll_slot_kernel<32>, dim3(p.num_tiles), dim3(kLLTile), smem, stream, p);
}

cudaError_t launch_ll_combine(const LLCombineParams& p, int num_sms, cudaStream_t stream) {
    if (p.G == 0) return cudaSuccess;
    (void)num_sms;
    const long long blocks = (p.G * p.splits + kLLCombineWarps - 1) / kLLCombineWarps;
    // 4 x 16-byte vectors per lane per row, groups of 4 rows (measured best on B200)
    return launch_pdl(ll_combine_kernel<4, 4>, dim3((unsigned)blocks), dim3(kLLCombineThreads), 0, stream, p);
}

}  // namespace ep
