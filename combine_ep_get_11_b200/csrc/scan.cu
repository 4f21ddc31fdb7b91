// Dispatch handle: single-pass decoupled-lookback prefix scan.
//
// "How DeepEP Optimizes Handle Reuse ...", section "What the Handle Contains"
// lists rank_prefix_matrix, channel_prefix_matrix, recv_channel_prefix_matrix,
// recv_src_idx, is_token_in_rank and send_head.  With receive rows ordered by
// (source rank, token), every one of them is a sample of one function: the
// exclusive running count P(g)[d] of tokens g' < g (global id g = s*T + t)
// that go to rank d.  So the whole handle is one scan over G tokens of R
// columns at once:
//   send_head[g][d]               = P(g)[d]                 if g goes to d, else -1
//   recv_channel_prefix[d][s][c]  = P(s*T + start(c))[d]
//   channel_prefix[s][d][c]       = P(s*T + start(c+1))[d] - P(s*T)[d]
//   rank_prefix[s][d]             = P((s+1)*T)[d]
//   N_d                           = P(G)[d]
// (start(c) = min(c*q, T), q = ceil(T/C)).
//
// Each 256-token tile turns its tokens' membership into per-column bit words
// (warp ballots), publishes its column counts, and finds its exclusive prefix
// by looking back over earlier tiles (flags: aggregate / inclusive), one lane
// per column, 16 earlier tiles' words loaded at once per round and consumed
// up to the first inclusive one.  A status word holds a tile's count, its flag
// and the call's tag, so relaxed (not acquire/release) accesses suffice and
// nothing is cleared between calls.  Tiles are numbered by a 64-bit ticket
// that is only ever incremented (ticket = call * num_tiles + tile), so a tile
// only ever waits on tiles that are already running and the call number tags
// the words; every wait is bounded (EP_ERR_TIMEOUT).
// The tile then writes send_head and every handle entry whose sample point
// falls in it: the channel starts (recv_channel_prefix), the channel ends
// relative to the rank's start (channel_prefix; the rank start P(s*T) comes
// from a call-tagged word that the tile holding s*T publishes) and the rank
// ends (rank_prefix).  The last tile holds P(G): it writes the receive offsets
// and the per-expert receive counts.  No tile waits for all the others.
// recv_src_idx needs the final offsets and is written by the dispatch kernel.

#include "common.cuh"
#include "kernels.h"

namespace ep {

namespace {

// Status word: count in bits 0-31, flag in bits 32-33, call tag in bits 34-63.
constexpr unsigned long long kFlagAggregate = 1ull << 32;
constexpr unsigned long long kFlagInclusive = 2ull << 32;
constexpr unsigned long long kFlagMask = 3ull << 32;
constexpr unsigned long long kTagMask = ~0ull << 34;
constexpr int kTagShift = 34;
constexpr int kWindow = 16;
constexpr int kWordsPerTile = kScanTile / 32;

__device__ __forceinline__ bool published(unsigned long long v, unsigned long long tag) {
    return (v & kTagMask) == tag && (v & kFlagMask) != 0;
}

__global__ void __launch_bounds__(kScanTile)
scan_kernel(const ScanParams p) {
    __shared__ int s_tile;
    __shared__ unsigned long long s_tag;
    __shared__ uint32_t s_bits[32][kWordsPerTile];   // [column][word] membership
    __shared__ int s_wpref[32][kWordsPerTile + 1];   // exclusive popc prefix over words
    __shared__ int s_excl[32];                        // tile's exclusive prefix per column

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int R = p.R;
    pdl_wait();                // everything before this kernel has completed ...
    pdl_launch_dependents();   // ... so the dispatch kernel may start prefetching its rows
    if (tid == 0) {
        const unsigned long long tk = atomicAdd(p.ticket, 1ull);
        s_tile = (int)(tk % (unsigned long long)p.num_tiles);
        s_tag = (tk / (unsigned long long)p.num_tiles + 1) << kTagShift;   // never 0
    }
    __syncthreads();
    const int tile = s_tile;
    const unsigned long long tag = s_tag;
    const long long g0 = (long long)tile * kScanTile;
    const long long g = g0 + tid;

    // membership mask of this thread's token
    uint32_t mask = 0;
    if (g < p.G) {
        const uint8_t* row = p.is_token_in_rank + g * R;
        if ((R & 3) == 0) {
            const uint32_t* r4 = reinterpret_cast<const uint32_t*>(row);
            for (int c = 0; c < R / 4; ++c) {
                const uint32_t w = __ldg(r4 + c);
                mask |= (uint32_t)((w & 0xffu) != 0) << (4 * c);
                mask |= (uint32_t)((w & 0xff00u) != 0) << (4 * c + 1);
                mask |= (uint32_t)((w & 0xff0000u) != 0) << (4 * c + 2);
                mask |= (uint32_t)((w & 0xff000000u) != 0) << (4 * c + 3);
            }
        } else {
            for (int d = 0; d < R; ++d) mask |= (uint32_t)(__ldg(row + d) != 0) << d;
        }
    }
    for (int d = 0; d < R; ++d) {
        const uint32_t b = __ballot_sync(kFullMask, (mask >> d) & 1u);
        if (lane == 0) s_bits[d][warp] = b;
    }
    __syncthreads();

    if (warp == 0 && lane < R) {
        int agg = 0;
        for (int w = 0; w < kWordsPerTile; ++w) {
            s_wpref[lane][w] = agg;
            agg += __popc(s_bits[lane][w]);
        }
        s_wpref[lane][kWordsPerTile] = agg;
        unsigned long long* mine = p.status + (size_t)tile * R + lane;
        int excl = 0;
        if (tile == 0) {
            st_relaxed_u64(mine, tag | kFlagInclusive | (unsigned)agg);
        } else {
            st_relaxed_u64(mine, tag | kFlagAggregate | (unsigned)agg);
            int top = tile - 1;          // newest tile of the current window
            bool found = false;
            uint64_t t0 = 0;
            uint32_t spins = 0;
            while (top >= 0 && !found) {
                const int cnt = min(kWindow, top + 1);
                unsigned long long v[kWindow];
                bool ok = false;
                int take = 0;
                for (;;) {
#pragma unroll
                    for (int u = 0; u < kWindow; ++u)
                        v[u] = u < cnt ? ld_relaxed_u64(p.status + (size_t)(top - u) * R + lane) : 0ull;
                    // words are needed only up to the first inclusive one
                    ok = true;
                    found = false;
                    take = cnt;
#pragma unroll
                    for (int u = 0; u < kWindow; ++u) {
                        if (u < take) {
                            if (!published(v[u], tag)) {
                                ok = false;
                                take = u;
                            } else if ((v[u] & kFlagMask) == kFlagInclusive) {
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
                for (int u = 0; u < kWindow; ++u)
                    if (u < take) excl += (int)(uint32_t)v[u];
                top -= cnt;
            }
            st_relaxed_u64(mine, tag | kFlagInclusive | (unsigned)(excl + agg));
        }
        s_excl[lane] = excl + (p.base != nullptr ? p.base[lane] : 0);
    }
    __syncthreads();

    // send_head for the tile, written [token][column] in order (coalesced)
    const int G = (int)p.G;                       // G * R < 2^31
    const int gt = (int)g0;
    const int ntok = min(kScanTile, G - gt);
    for (int i = tid; i < ntok * R; i += kScanTile) {
        const int tok = i / R, d = i - tok * R;
        const int w = tok >> 5, b = tok & 31;
        const uint32_t bits = s_bits[d][w];
        int v = -1;
        if ((bits >> b) & 1u) v = s_excl[d] + s_wpref[d][w] + __popc(bits & ((1u << b) - 1u));
        p.send_head[(long long)gt * R + i] = v;
    }

    // sample points gb = s*T + start(c), c in [0, C], that fall in this tile
    // (gb == G belongs to the last tile); P(gb)[d] = s_excl[d] + members before gb
    const bool last_tile = tile == p.num_tiles - 1;
    const int T = p.T, C = p.C;
    if (p.recv_channel_prefix_matrix != nullptr) {
        const int s_lo = max(0, gt / T - 1);
        const int s_hi = min(R - 1, (gt + kScanTile) / T);
        const int per_src = (C + 1) * R;
        const int nb = (s_hi - s_lo + 1) * per_src;
        for (int i = tid; i < nb; i += kScanTile) {
            const int s = s_lo + i / per_src;
            const int rem = i - (i / per_src) * per_src;
            const int c = rem / R, d = rem - (rem / R) * R;
            const int gb = s * T + min(c * p.q, T);
            const bool here = (gb >= gt && gb < gt + kScanTile && gb < G) || (gb == G && last_tile);
            if (!here) continue;
            const int rel = gb - gt;   // 0..256
            const int w = rel >> 5, b = rel & 31;
            const int pv = s_excl[d] + ((w < kWordsPerTile) ? s_wpref[d][w] + __popc(s_bits[d][w] & ((1u << b) - 1u))
                                                             : s_wpref[d][kWordsPerTile]);
            if (c == 0 && s > 0) st_relaxed_u64(p.rank_start + (size_t)s * R + d, tag | kFlagInclusive | (unsigned)pv);
            if (c < C) p.recv_channel_prefix_matrix[((long long)d * R + s) * C + c] = pv;
            if (c == C) p.rank_prefix_matrix[s * R + d] = pv;
            if (c > 0) {
                // the rank's start P(s*T)[d]: in this tile, or published by an earlier one
                int start = 0;
                const int gs = s * T;
                if (s == 0) {
                    start = 0;
                } else if (gs >= gt) {
                    const int rs = gs - gt, ws = rs >> 5, bs = rs & 31;
                    start = s_excl[d] + s_wpref[d][ws] + __popc(s_bits[d][ws] & ((1u << bs) - 1u));
                } else {
                    unsigned long long v = ld_relaxed_u64(p.rank_start + (size_t)s * R + d);
                    uint64_t t0 = 0;
                    uint32_t spins = 0;
                    while (!published(v, tag)) {
                        if (spins == 0) t0 = globaltimer_ns();
                        ++spins;
                        if (spins > kWaitLimitIters ||
                            ((spins & 63u) == 0 && globaltimer_ns() - t0 > kWaitLimitNs)) {
                            record_error(p.err, EP_ERR_TIMEOUT);
                            break;
                        }
                        v = ld_relaxed_u64(p.rank_start + (size_t)s * R + d);
                    }
                    start = (int)(uint32_t)v;
                }
                p.channel_prefix_matrix[((long long)s * R + d) * C + (c - 1)] = pv - start;
            }
        }
    }

    if (!last_tile || p.recv_rank_offset == nullptr) return;
    // P(G)[d] = N_d: receive offsets; per-expert receive counts from the layout
    __shared__ long long s_total[32];
    if (tid < R) s_total[tid] = s_excl[tid] + s_wpref[tid][kWordsPerTile];
    __syncthreads();
    if (tid == 0) {
        long long off = 0;
        for (int d = 0; d < R; ++d) {
            p.recv_rank_offset[d] = off;
            off += s_total[d];
        }
        p.recv_rank_offset[R] = off;
    }
    constexpr int kBatch = 8;
    for (int i = tid; i < p.E; i += kScanTile) {
        // i = d*L + j: sum over sources, 8 independent loads per round
        int part[kBatch] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int s0 = 0; s0 < R; s0 += kBatch) {
#pragma unroll
            for (int u = 0; u < kBatch; ++u)
                if (s0 + u < R) part[u] += __ldcg(p.num_tokens_per_expert + (long long)(s0 + u) * p.E + i);
        }
        int sum = 0;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) sum += part[u];
        p.num_recv_tokens_per_expert[i] = sum;
    }
}

}  // namespace

cudaError_t launch_scan(const ScanParams& p, cudaStream_t stream) {
    if (p.num_tiles == 0) return cudaSuccess;
    return launch_pdl(scan_kernel, dim3(p.num_tiles), dim3(kScanTile), 0, stream, p);
}

}  // namespace ep
