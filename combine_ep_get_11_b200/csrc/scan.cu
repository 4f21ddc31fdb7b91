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
// per column.  A flag and its count share one 64-bit word, and nothing else is
// read on the strength of a flag, so relaxed (not acquire/release) accesses
// suffice; the finishing tile's reads of the boundary samples are ordered by
// a fence and the finish counter.  Tiles are numbered by an atomic ticket in start order, so a
// tile only ever waits on tiles that are already running; every wait is
// bounded (EP_ERR_TIMEOUT).  The tile then writes send_head and the channel
// boundary samples; the last tile to finish (atomic counter) assembles the
// matrices, the receive offsets and the per-expert receive counts.
// recv_src_idx needs the final offsets and is written by the dispatch kernel.

#include "common.cuh"
#include "kernels.h"

namespace ep {

namespace {

constexpr unsigned long long kFlagAggregate = 1ull << 62;
constexpr unsigned long long kFlagInclusive = 2ull << 62;
constexpr int kWordsPerTile = kScanTile / 32;

__global__ void __launch_bounds__(kScanTile)
scan_kernel(const ScanParams p) {
    __shared__ int s_tile;
    __shared__ int s_last;
    __shared__ uint32_t s_bits[32][kWordsPerTile];   // [column][word] membership
    __shared__ int s_wpref[32][kWordsPerTile + 1];   // exclusive popc prefix over words
    __shared__ int s_excl[32];                        // tile's exclusive prefix per column

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int R = p.R;
    if (tid == 0) s_tile = atomicAdd(p.ticket, 1);
    __syncthreads();
    const int tile = s_tile;
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
            st_relaxed_u64(mine, kFlagInclusive | (unsigned)agg);
        } else {
            st_relaxed_u64(mine, kFlagAggregate | (unsigned)agg);
            int j = tile - 1;
            uint64_t t0 = 0;
            uint32_t spins = 0;
            while (j >= 0) {
                const unsigned long long v = ld_relaxed_u64(p.status + (size_t)j * R + lane);
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
                if (flag == kFlagInclusive) break;
                --j;
            }
            st_relaxed_u64(mine, kFlagInclusive | (unsigned)(excl + agg));
        }
        s_excl[lane] = excl;
    }
    __syncthreads();

    // send_head for the tile, written [token][column] in order (coalesced)
    const int ntok = (int)min((long long)kScanTile, p.G - g0);
    for (int i = tid; i < ntok * R; i += kScanTile) {
        const int tok = i / R, d = i - tok * R;
        const int w = tok >> 5, b = tok & 31;
        const uint32_t bits = s_bits[d][w];
        int v = -1;
        if ((bits >> b) & 1u) v = s_excl[d] + s_wpref[d][w] + __popc(bits & ((1u << b) - 1u));
        p.send_head[g0 * R + i] = v;
    }

    // channel boundaries gb = s*T + start(c), c in [0, C], that fall in this tile
    // (gb == G belongs to the last tile)
    const bool last_tile = tile == p.num_tiles - 1;
    const long long s_lo = max(0LL, g0 / p.T - 1);
    const long long s_hi = min((long long)R - 1, (g0 + kScanTile) / p.T);
    const int per_src = (p.C + 1) * R;
    const long long nb = (s_hi - s_lo + 1) * per_src;
    for (long long i = tid; i < nb; i += kScanTile) {
        const int s = (int)(s_lo + i / per_src);
        const int rem = (int)(i % per_src);
        const int c = rem / R, d = rem - (rem / R) * R;
        const long long gb = (long long)s * p.T + min((long long)c * p.q, (long long)p.T);
        const bool mine = (gb >= g0 && gb < g0 + kScanTile && gb < p.G) || (gb == p.G && last_tile);
        if (!mine) continue;
        const int rel = (int)(gb - g0);   // 0..256
        const int w = rel >> 5, b = rel & 31;
        const int cnt = (w < kWordsPerTile)
                            ? s_wpref[d][w] + __popc(s_bits[d][w] & ((1u << b) - 1u))
                            : s_wpref[d][kWordsPerTile];
        p.boundary[((long long)s * (p.C + 1) + c) * R + d] = s_excl[d] + cnt;
    }

    // the last tile to finish assembles the matrices
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(p.done, 1) == p.num_tiles - 1;
    __syncthreads();
    if (!s_last) return;
    __threadfence();

    // Loads of each batch are issued before its stores (independent L2 round
    // trips overlap; a store between loads would serialise them).
    const int C = p.C;
    const int* bp = p.boundary;
    auto B = [&](int s, int c, int d) { return __ldcg(bp + ((long long)s * (C + 1) + c) * R + d); };
    constexpr int kBatch = 8;
    const int nm = R * R * C;
    for (int i0 = 0; i0 < nm; i0 += kScanTile * kBatch) {
        int vc[kBatch], vn[kBatch], v0[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u * kScanTile + tid;   // i enumerates [d][s][c]
            if (i < nm) {
                const int c = i % C, s = (i / C) % R, d = i / (C * R);
                vc[u] = B(s, c, d);
                vn[u] = B(s, c + 1, d);
                v0[u] = B(s, 0, d);
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int i = i0 + u * kScanTile + tid;
            if (i < nm) {
                const int c = i % C, s = (i / C) % R, d = i / (C * R);
                p.recv_channel_prefix_matrix[i] = vc[u];
                p.channel_prefix_matrix[((long long)s * R + d) * C + c] = vn[u] - v0[u];
            }
        }
    }
    for (int i = tid; i < R * R; i += kScanTile) {
        const int s = i / R, d = i % R;
        p.rank_prefix_matrix[i] = B(s, C, d);
    }
    __shared__ long long s_total[32];
    if (tid < R) s_total[tid] = B(R - 1, C, tid);
    __syncthreads();
    if (tid == 0) {
        long long off = 0;
        for (int d = 0; d < R; ++d) {
            p.recv_rank_offset[d] = off;
            off += s_total[d];
        }
        p.recv_rank_offset[R] = off;
    }
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
    scan_kernel<<<p.num_tiles, kScanTile, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace ep
