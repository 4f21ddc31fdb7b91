// Reference oracle for MoE expert-parallel dispatch / combine on virtual ranks.
//
// TEST INFRASTRUCTURE ONLY.  This file is a plain, slow, single-threaded CPU
// statement of what the dispatch/combine hot path computes.  Only the tests,
// the smoke check and the benchmark's CPU-baseline leg may load it.  It shares
// no code, header, table or helper with the CUDA library, and the library never
// calls it.
//
// Sources (web pages about DeepSeek's DeepEP `Buffer`):
//   [API]    "DeepEP Buffer Class API for Expert Parallel Communication:
//             Architecture and Usage" -- sections "Configuration and Layout
//             Helpers", "Dispatch Operation", "Combine Operation",
//             "IB-GDA Kernels", "Code Examples".
//   [REUSE]  "How DeepEP Optimizes Handle Reuse for Repeated Dispatches" --
//             sections "What the Handle Contains", "Performance Contract and
//             Constraints".
//   [ARCH]   "Architecture" (DeepEP-Lib) -- section "Configuration System".
//   [CORE]   "Core-Implementation" (DeepEP C++ runtime) -- section "Memory
//             Alignment and Validation".
//
// The pages name the outputs but leave their exact meaning open; the readings
// taken here (expert->rank map, receive order, matrix orientation, channel
// partition, LL slot order, summation order) are listed in the design notes
// and restated next to each function below.
//
// Notation: R ranks, E experts, L = E / R local experts per rank, T tokens per
// rank, K top-k slots, H hidden size, C channels.  Rank s owns tokens
// x[s][0..T).  A global token id is g = s * T + t.  rank(e) = e / L,
// loc(e) = e mod L, an expert id of -1 marks an unused slot.
//
// Floating point: every reduction is stated twice.
//   * The fixed-order fp32 definition (oracle_combine_fp32,
//     oracle_ll_combine_fp32, oracle_lb_reduce_grads_fp32): an fp32
//     accumulator starting at +0 (or at the original gradient), one IEEE
//     binary32 operation per term in the stated order (round to nearest even;
//     the low-latency combine uses a fused multiply-add, one rounding per
//     term), then one rounding to bf16.  This is the result the method
//     computes, bit for bit, so the CUDA path must match it exactly.
//   * The exact sum (oracle_combine, oracle_ll_combine, oracle_lb_reduce_grads):
//     accumulated in double (exact for these term counts and magnitudes up to
//     the last bits) and rounded once to bf16.  It is the reference for the
//     "within one bf16 ulp" accuracy statement.
// bf16 values are passed as their raw 16-bit patterns.  Built with
// -ffp-contract=off so no multiply and add is fused unless written as fma.
//
// Parity status: every function here is pinned by tests/test_oracle_pins.py
// (brute force with an independent sort-based formulation, closed forms,
// invariants, special cases and hand-worked fixtures; the summation order and
// the fused multiply-add of the fp32 reductions by hand-worked cancellation
// cases in tests/golden/fp32_order.txt), and tests/test_oracle_mutations.py
// checks that planted mistakes fail those pins.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <algorithm>

namespace {

enum {
    ORACLE_OK = 0,
    ORACLE_BAD_ARG = 1,
    ORACLE_BAD_TOPK = 2,
    ORACLE_CAPACITY = 3,
    ORACLE_NOT_FOUND = 4,
};

double bf16_bits_to_double(uint16_t b) {
    uint32_t u = static_cast<uint32_t>(b) << 16;
    float f;
    std::memcpy(&f, &u, sizeof f);
    return static_cast<double>(f);
}

// Round a finite double to the nearest bf16 value, ties to even, in one step
// (no intermediate rounding to fp32).  bf16 keeps 8 significant bits; the
// smallest normal exponent is -126 and subnormals step by 2^-133.
uint16_t double_to_bf16_bits(double v) {
    if (std::isnan(v)) return 0x7fc0;
    const bool neg = std::signbit(v);
    double a = std::fabs(v);
    if (a == 0.0) return neg ? 0x8000 : 0x0000;
    int e;
    std::frexp(a, &e);                 // a = m * 2^e, m in [0.5, 1)
    int quantum_exp = e - 8;           // weight of the lowest kept bit
    if (quantum_exp < -133) quantum_exp = -133;
    const double scaled = std::ldexp(a, -quantum_exp);   // exact
    double r = std::nearbyint(scaled);                   // default mode: ties to even
    double q = std::ldexp(r, quantum_exp);               // exact
    if (q >= std::ldexp(1.0, 128)) {                     // overflow to infinity
        return neg ? 0xff80 : 0x7f80;
    }
    float f = static_cast<float>(q);                     // exact: q is a bf16 value
    uint32_t u;
    std::memcpy(&u, &f, sizeof u);
    uint16_t b = static_cast<uint16_t>(u >> 16);
    return neg ? static_cast<uint16_t>(b | 0x8000) : b;
}

// bf16 bits -> float (exact: bf16 is the upper half of a binary32 pattern).
float bf16_bits_to_float(uint16_t b) {
    uint32_t u = static_cast<uint32_t>(b) << 16;
    float f;
    std::memcpy(&f, &u, sizeof f);
    return f;
}

// float -> bf16 bits, nearest even.  A float is exactly a double, so the
// one-step double rounding above rounds the float itself.
uint16_t float_to_bf16_bits(float f) { return double_to_bf16_bits(static_cast<double>(f)); }

bool shape_ok(int32_t R, int32_t E, int32_t T, int32_t K) {
    return R >= 1 && E >= 1 && E % R == 0 && T >= 0 && K >= 1;
}

}  // namespace

extern "C" {

// Exposed so the tests can pin the rounding step on its own.
void oracle_round_bf16(const double* in, uint16_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16_bits(in[i]);
}

// Dispatch layout.  [API] "Configuration and Layout Helpers": from topk_idx,
// derive how many tokens go to each rank and, per token, whether it goes to a
// rank; the per-expert token counts are the receive counts of [API] "Code
// Examples" (`recv_counts`).
//
//   is_token_in_rank[s][t][d] = 1 iff some slot k has a valid expert e with
//                               rank(e) = d                       (u8, [R][T][R])
//   num_tokens_per_rank[s][d] = sum_t is_token_in_rank[s][t][d]     (i32, [R][R])
//   num_tokens_per_expert[s][e] = #{(t, k) : topk_idx[s][t][k] = e} (i32, [R][E])
//
// Expert ids outside [-1, E) are an error.
int oracle_layout(int32_t R, int32_t E, int32_t T, int32_t K, const int64_t* topk_idx,
                  int32_t* num_tokens_per_rank, int32_t* num_tokens_per_expert,
                  uint8_t* is_token_in_rank) {
    if (!shape_ok(R, E, T, K)) return ORACLE_BAD_ARG;
    const int32_t L = E / R;
    for (int64_t i = 0; i < (int64_t)R * R; ++i) num_tokens_per_rank[i] = 0;
    for (int64_t i = 0; i < (int64_t)R * E; ++i) num_tokens_per_expert[i] = 0;
    for (int32_t s = 0; s < R; ++s) {
        for (int32_t t = 0; t < T; ++t) {
            const int64_t g = (int64_t)s * T + t;
            uint8_t* in_row = is_token_in_rank + g * R;
            for (int32_t d = 0; d < R; ++d) in_row[d] = 0;
            for (int32_t k = 0; k < K; ++k) {
                const int64_t e = topk_idx[g * K + k];
                if (e == -1) continue;
                if (e < -1 || e >= E) return ORACLE_BAD_TOPK;
                in_row[e / L] = 1;
                num_tokens_per_expert[(int64_t)s * E + e] += 1;
            }
            for (int32_t d = 0; d < R; ++d) num_tokens_per_rank[(int64_t)s * R + d] += in_row[d];
        }
    }
    return ORACLE_OK;
}

// Dispatch handle.  [REUSE] "What the Handle Contains" lists rank_prefix_matrix,
// channel_prefix_matrix, recv_channel_prefix_matrix, recv_src_idx,
// is_token_in_rank and send_head; [API] "Dispatch Operation" says they map
// received rows back to their source tokens.  Readings:
//   * receive order of destination d: every (s, t) with is_token_in_rank = 1,
//     source rank ascending, then token ascending;
//   * send_head[s][t][d] = position of (s, t) in that order, or -1;
//   * destination blocks are concatenated: rows of d start at
//     recv_rank_offset[d] = sum_{d' < d} N_d';  recv_rank_offset[R] = N;
//   * recv_src_idx[recv_rank_offset[d] + p] = t of the p-th received token;
//   * rank_prefix_matrix[i][d] = sum_{s <= i} num_tokens_per_rank[s][d];
//   * channel c of a rank covers tokens [start(c), start(c+1)) with
//     start(c) = min(c * ceil(T / C), T) ([ARCH] "Configuration System" sizes
//     work in channels but gives no partition; contiguous ranges are taken);
//     channel_prefix_matrix[s][d][c] = tokens of s for d in channels 0..c;
//   * recv_channel_prefix_matrix[d][s][c] = first position in d's order that
//     belongs to channel c of source s
//     = rank_prefix[s-1][d] (or 0) + channel_prefix[s][d][c-1] (or 0);
//   * num_recv_tokens_per_expert[d][j] = sum_s num_tokens_per_expert[s][d*L+j].
// recv_src_idx may be null (only the matrices are produced).
int oracle_dispatch_handle(int32_t R, int32_t E, int32_t T, int32_t C,
                           const uint8_t* is_token_in_rank, const int32_t* num_tokens_per_expert,
                           int32_t* rank_prefix_matrix, int32_t* channel_prefix_matrix,
                           int32_t* recv_channel_prefix_matrix, int32_t* send_head,
                           int64_t* recv_rank_offset, int32_t* num_recv_tokens_per_expert,
                           int32_t* recv_src_idx, int64_t recv_capacity) {
    if (R < 1 || E < 1 || E % R != 0 || T < 0 || C < 1) return ORACLE_BAD_ARG;
    const int32_t L = E / R;

    // Receive order per destination; positions become send_head.
    std::vector<int64_t> N(R, 0);
    for (int32_t d = 0; d < R; ++d) {
        int64_t p = 0;
        for (int32_t s = 0; s < R; ++s) {
            for (int32_t t = 0; t < T; ++t) {
                const int64_t g = (int64_t)s * T + t;
                if (is_token_in_rank[g * R + d]) {
                    send_head[g * R + d] = (int32_t)p;
                    ++p;
                } else {
                    send_head[g * R + d] = -1;
                }
            }
        }
        N[d] = p;
    }
    recv_rank_offset[0] = 0;
    for (int32_t d = 0; d < R; ++d) recv_rank_offset[d + 1] = recv_rank_offset[d] + N[d];

    if (recv_src_idx != nullptr) {
        if (recv_rank_offset[R] > recv_capacity) return ORACLE_CAPACITY;
        for (int32_t s = 0; s < R; ++s)
            for (int32_t t = 0; t < T; ++t)
                for (int32_t d = 0; d < R; ++d) {
                    const int64_t g = (int64_t)s * T + t;
                    const int32_t h = send_head[g * R + d];
                    if (h >= 0) recv_src_idx[recv_rank_offset[d] + h] = t;
                }
    }

    // rank_prefix_matrix[i][d]: inclusive over source ranks.
    for (int32_t d = 0; d < R; ++d) {
        int64_t running = 0;
        for (int32_t i = 0; i < R; ++i) {
            for (int32_t t = 0; t < T; ++t)
                running += is_token_in_rank[((int64_t)i * T + t) * R + d];
            rank_prefix_matrix[(int64_t)i * R + d] = (int32_t)running;
        }
    }

    // Channels: contiguous token ranges of ceil(T / C) tokens.
    const int64_t q = (T + (int64_t)C - 1) / C;
    auto start = [&](int64_t c) -> int64_t { return std::min<int64_t>(c * q, T); };
    for (int32_t s = 0; s < R; ++s)
        for (int32_t d = 0; d < R; ++d) {
            int64_t running = 0;
            for (int32_t c = 0; c < C; ++c) {
                for (int64_t t = start(c); t < start(c + 1); ++t)
                    running += is_token_in_rank[((int64_t)s * T + t) * R + d];
                channel_prefix_matrix[((int64_t)s * R + d) * C + c] = (int32_t)running;
            }
        }
    for (int32_t d = 0; d < R; ++d)
        for (int32_t s = 0; s < R; ++s)
            for (int32_t c = 0; c < C; ++c) {
                const int64_t before_rank = s > 0 ? rank_prefix_matrix[(int64_t)(s - 1) * R + d] : 0;
                const int64_t before_chan = c > 0 ? channel_prefix_matrix[((int64_t)s * R + d) * C + (c - 1)] : 0;
                recv_channel_prefix_matrix[((int64_t)d * R + s) * C + c] = (int32_t)(before_rank + before_chan);
            }

    for (int32_t d = 0; d < R; ++d)
        for (int32_t j = 0; j < L; ++j) {
            int64_t sum = 0;
            for (int32_t s = 0; s < R; ++s) sum += num_tokens_per_expert[(int64_t)s * E + (int64_t)d * L + j];
            num_recv_tokens_per_expert[(int64_t)d * L + j] = (int32_t)sum;
        }
    return ORACLE_OK;
}

// Dispatch rows.  [API] "Dispatch Operation": every token is sent, with its
// top-k indices and weights, to each rank that owns one of its experts.
//   recv_x[off_d + p] = x[s][t]                       (bit copy, H bf16)
//   recv_topk_idx[off_d + p][k] = loc(e) if e valid and rank(e) = d, else -1
//   recv_topk_weights[off_d + p][k] = w[s][t][k] under the same test, else 0
// where p = send_head[s][t][d].  Any output pointer may be null (skipped);
// topk_weights may be null when recv_topk_weights is null.
int oracle_dispatch_rows(int32_t R, int32_t E, int32_t T, int32_t K, int32_t H,
                         const uint16_t* x, const int64_t* topk_idx, const float* topk_weights,
                         const int32_t* send_head, const int64_t* recv_rank_offset,
                         uint16_t* recv_x, int64_t* recv_topk_idx, float* recv_topk_weights) {
    if (!shape_ok(R, E, T, K) || H < 1) return ORACLE_BAD_ARG;
    const int32_t L = E / R;
    for (int32_t d = 0; d < R; ++d) {
        for (int32_t s = 0; s < R; ++s) {
            for (int32_t t = 0; t < T; ++t) {
                const int64_t g = (int64_t)s * T + t;
                const int32_t p = send_head[g * R + d];
                if (p < 0) continue;
                const int64_t row = recv_rank_offset[d] + p;
                if (recv_x != nullptr)
                    for (int32_t i = 0; i < H; ++i) recv_x[row * H + i] = x[g * H + i];
                for (int32_t k = 0; k < K; ++k) {
                    const int64_t e = topk_idx[g * K + k];
                    const bool here = e >= 0 && e < E && e / L == d;
                    if (recv_topk_idx != nullptr) recv_topk_idx[row * K + k] = here ? e % L : -1;
                    if (recv_topk_weights != nullptr)
                        recv_topk_weights[row * K + k] = here ? topk_weights[g * K + k] : 0.0f;
                }
            }
        }
    }
    return ORACLE_OK;
}

// Combine.  [API] "Combine Operation": the handle maps received rows back to
// their source tokens and the rows are reduced by addition, with optional bias
// terms; in the usage example the call takes the received rows, the handle and
// the received weights and gives back combined rows and combined weights.
// Readings: the hidden rows are summed
// unweighted over destination ranks in ascending order, then bias0 and bias1
// ([R][T][H] each, optional) are added; the combined weights are the sum over
// destinations of the received weight rows.
//   out_x[s][t][i] = bf16( sum_{d : h = send_head[s][t][d] >= 0} y[off_d + h][i]
//                          + bias0[s][t][i] + bias1[s][t][i] )     (fp64 sum)
//   out_topk_weights[s][t][k] = sum_d recv_topk_weights[off_d + h][k]
// A token with no destination gets bf16(bias terms), i.e. +0 without bias.
// `tokens` (optional) restricts the work to a list of global token ids; the
// outputs then hold one row per listed token, in list order.
int oracle_combine(int32_t R, int32_t T, int32_t K, int32_t H,
                   const uint16_t* y, int64_t y_rows, const int32_t* send_head,
                   const int64_t* recv_rank_offset, const float* recv_topk_weights,
                   const uint16_t* bias0, const uint16_t* bias1,
                   uint16_t* out_x, float* out_topk_weights,
                   const int64_t* tokens, int64_t n_tokens) {
    if (R < 1 || T < 0 || K < 1 || H < 1) return ORACLE_BAD_ARG;
    const int64_t G = (int64_t)R * T;
    const int64_t n = tokens != nullptr ? n_tokens : G;
    std::vector<double> acc(H);
    for (int64_t i = 0; i < n; ++i) {
        const int64_t g = tokens != nullptr ? tokens[i] : i;
        if (g < 0 || g >= G) return ORACLE_BAD_ARG;
        std::fill(acc.begin(), acc.end(), 0.0);
        for (int32_t d = 0; d < R; ++d) {
            const int32_t h = send_head[g * R + d];
            if (h < 0) continue;
            const int64_t row = recv_rank_offset[d] + h;
            if (row >= y_rows) return ORACLE_CAPACITY;
            for (int32_t c = 0; c < H; ++c) acc[c] += bf16_bits_to_double(y[row * H + c]);
        }
        if (bias0 != nullptr)
            for (int32_t c = 0; c < H; ++c) acc[c] += bf16_bits_to_double(bias0[g * H + c]);
        if (bias1 != nullptr)
            for (int32_t c = 0; c < H; ++c) acc[c] += bf16_bits_to_double(bias1[g * H + c]);
        if (out_x != nullptr)
            for (int32_t c = 0; c < H; ++c) out_x[i * H + c] = double_to_bf16_bits(acc[c]);
        if (out_topk_weights != nullptr && recv_topk_weights != nullptr) {
            for (int32_t k = 0; k < K; ++k) {
                double w = 0.0;
                for (int32_t d = 0; d < R; ++d) {
                    const int32_t h = send_head[g * R + d];
                    if (h < 0) continue;
                    w += (double)recv_topk_weights[(recv_rank_offset[d] + h) * K + k];
                }
                out_topk_weights[i * K + k] = (float)w;
            }
        }
    }
    return ORACLE_OK;
}

// Combine, fixed-order fp32 definition (same arguments as oracle_combine).
// The reduction of [API] "Combine Operation" taken as the method computes it:
// an fp32 accumulator starting at +0 adds, one binary32 addition each (round
// to nearest even), the token's received rows in ascending destination rank,
// then bias0, then bias1, and is rounded once to bf16:
//   acc = +0;  for d = 0, 1, ..., R-1 with h = send_head[s][t][d] >= 0:
//                  acc = acc + y[off_d + h][i]
//   acc = acc + bias0[s][t][i];  acc = acc + bias1[s][t][i];  out = bf16(acc)
// The combined weights take the same ascending-rank fp32 sum of the received
// weight rows.
int oracle_combine_fp32(int32_t R, int32_t T, int32_t K, int32_t H,
                        const uint16_t* y, int64_t y_rows, const int32_t* send_head,
                        const int64_t* recv_rank_offset, const float* recv_topk_weights,
                        const uint16_t* bias0, const uint16_t* bias1,
                        uint16_t* out_x, float* out_topk_weights,
                        const int64_t* tokens, int64_t n_tokens) {
    if (R < 1 || T < 0 || K < 1 || H < 1) return ORACLE_BAD_ARG;
    const int64_t G = (int64_t)R * T;
    const int64_t n = tokens != nullptr ? n_tokens : G;
    std::vector<float> sum32(H);
    for (int64_t i = 0; i < n; ++i) {
        const int64_t g = tokens != nullptr ? tokens[i] : i;
        if (g < 0 || g >= G) return ORACLE_BAD_ARG;
        std::fill(sum32.begin(), sum32.end(), 0.0f);
        for (int32_t dst = 0; dst < R; ++dst) {          // ascending destination rank
            const int32_t h = send_head[g * R + dst];
            if (h < 0) continue;
            const int64_t row = recv_rank_offset[dst] + h;
            if (row >= y_rows) return ORACLE_CAPACITY;
            for (int32_t c = 0; c < H; ++c) sum32[c] = sum32[c] + bf16_bits_to_float(y[row * H + c]);
        }
        if (bias0 != nullptr)
            for (int32_t c = 0; c < H; ++c) sum32[c] = sum32[c] + bf16_bits_to_float(bias0[g * H + c]);
        if (bias1 != nullptr)
            for (int32_t c = 0; c < H; ++c) sum32[c] = sum32[c] + bf16_bits_to_float(bias1[g * H + c]);
        if (out_x != nullptr)
            for (int32_t c = 0; c < H; ++c) out_x[i * H + c] = float_to_bf16_bits(sum32[c]);
        if (out_topk_weights != nullptr && recv_topk_weights != nullptr) {
            for (int32_t k = 0; k < K; ++k) {
                float w32 = 0.0f;
                for (int32_t dst = 0; dst < R; ++dst) {
                    const int32_t h = send_head[g * R + dst];
                    if (h < 0) continue;
                    w32 = w32 + recv_topk_weights[(recv_rank_offset[dst] + h) * K + k];
                }
                out_topk_weights[i * K + k] = w32;
            }
        }
    }
    return ORACLE_OK;
}

// Low-latency dispatch.  [API] "IB-GDA Kernels" and "Low-Latency Inference
// with FP8": tokens are streamed into per-expert packed receive buffers bounded
// by num_max_dispatch_tokens_per_rank (Tmax); the call returns the packed rows,
// per-expert counts and a handle for the combine.  Readings:
//   * the list of expert e = d*L + j holds every (s, t) with some slot k
//     naming e (a token counts once per expert), in (s, t) ascending order;
//   * the slot of (s, t) is its position in that list, capacity R * Tmax;
//   * packed_recv_x[d][j][slot] = x[s][t];  src_info[d][j][slot] = t;
//   * layout_range[d][j][s] = {first slot of source s, its number of slots};
//   * packed_recv_count[d][j] = list length.
// Slots at or past the count are not written.  packed_recv_x may be null
// (handle only).
// [API] "Dynamic Rank Masking": masked ranks are left out of the exchange
// without tearing it down.  Reading: rank_mask[r] != 0 (nullable) removes rank
// r both as a source (its tokens are not sent) and as a destination (its
// experts receive nothing).
int oracle_ll_dispatch(int32_t R, int32_t E, int32_t T, int32_t K, int32_t H, int32_t Tmax,
                       const uint16_t* x, const int64_t* topk_idx, uint16_t* packed_recv_x,
                       int32_t* packed_recv_count, int32_t* src_info, int32_t* layout_range,
                       const int32_t* rank_mask) {
    if (!shape_ok(R, E, T, K) || H < 1 || Tmax < T) return ORACLE_BAD_ARG;
    const int32_t L = E / R;
    const int64_t cap = (int64_t)R * Tmax;
    for (int64_t i = 0; i < (int64_t)R * T * K; ++i)
        if (topk_idx[i] < -1 || topk_idx[i] >= E) return ORACLE_BAD_TOPK;
    for (int32_t e = 0; e < E; ++e) {
        const int32_t d = e / L, j = e % L;
        const int64_t list = (int64_t)d * L + j;
        int64_t slot = 0;
        for (int32_t s = 0; s < R; ++s) {
            const int64_t begin = slot;
            for (int32_t t = 0; t < T; ++t) {
                const int64_t g = (int64_t)s * T + t;
                bool member = false;
                for (int32_t k = 0; k < K; ++k) member = member || topk_idx[g * K + k] == e;
                const bool masked = rank_mask != nullptr && (rank_mask[s] != 0 || rank_mask[d] != 0);
                if (!member || masked) continue;
                if (slot >= cap) return ORACLE_CAPACITY;
                src_info[list * cap + slot] = t;
                if (packed_recv_x != nullptr)
                    for (int32_t i = 0; i < H; ++i)
                        packed_recv_x[(list * cap + slot) * H + i] = x[g * H + i];
                ++slot;
            }
            layout_range[(list * R + s) * 2 + 0] = (int32_t)begin;
            layout_range[(list * R + s) * 2 + 1] = (int32_t)(slot - begin);
        }
        packed_recv_count[list] = (int32_t)slot;
    }
    return ORACLE_OK;
}

// Low-latency combine.  [API] "IB-GDA Kernels" and "Low-Latency Inference
// with FP8": expert outputs are reduced back to their token positions using
// topk_idx, the top-k weights and the dispatch handle.  Reading: the weighted
// sum over the token's valid slots, visited in ascending (expert id, slot k):
//   out[s][t][i] = bf16( sum_k w[s][t][k] * y[d][j][slot(s, t, e)][i] )   (fp64)
// where e = topk_idx[s][t][k] = d*L + j and slot(s, t, e) is the position of t
// inside layout_range[d][j][s] (found through src_info).  `tokens` as in
// oracle_combine.  With a rank mask (see oracle_ll_dispatch), slots whose
// expert lives on a masked rank contribute nothing, and the tokens of a masked
// source rank get +0 (the rank took no part).
int oracle_ll_combine(int32_t R, int32_t E, int32_t T, int32_t K, int32_t H, int32_t Tmax,
                      const uint16_t* y, const int64_t* topk_idx, const float* topk_weights,
                      const int32_t* src_info, const int32_t* layout_range, uint16_t* out,
                      const int64_t* tokens, int64_t n_tokens, const int32_t* rank_mask) {
    if (!shape_ok(R, E, T, K) || H < 1 || Tmax < T) return ORACLE_BAD_ARG;
    const int32_t L = E / R;
    const int64_t cap = (int64_t)R * Tmax;
    const int64_t G = (int64_t)R * T;
    const int64_t n = tokens != nullptr ? n_tokens : G;
    std::vector<double> acc(H);
    std::vector<std::pair<int64_t, int32_t>> order;
    for (int64_t i = 0; i < n; ++i) {
        const int64_t g = tokens != nullptr ? tokens[i] : i;
        if (g < 0 || g >= G) return ORACLE_BAD_ARG;
        const int32_t s = (int32_t)(g / T), t = (int32_t)(g % T);
        order.clear();
        for (int32_t k = 0; k < K; ++k) {
            const int64_t e = topk_idx[g * K + k];
            if (e == -1) continue;
            if (e < -1 || e >= E) return ORACLE_BAD_TOPK;
            if (rank_mask != nullptr && (rank_mask[s] != 0 || rank_mask[e / L] != 0)) continue;
            order.emplace_back(e, k);
        }
        std::sort(order.begin(), order.end());
        std::fill(acc.begin(), acc.end(), 0.0);
        for (const auto& ek : order) {
            const int64_t e = ek.first;
            const int32_t k = ek.second;
            const int64_t list = e;   // = (e / L) * L + e % L
            const int32_t begin = layout_range[(list * R + s) * 2 + 0];
            const int32_t count = layout_range[(list * R + s) * 2 + 1];
            int64_t slot = -1;
            for (int32_t p = begin; p < begin + count; ++p)
                if (src_info[list * cap + p] == t) { slot = p; break; }
            if (slot < 0) return ORACLE_NOT_FOUND;
            const double w = (double)topk_weights[g * K + k];
            const uint16_t* row = y + (list * cap + slot) * H;
            for (int32_t c = 0; c < H; ++c) acc[c] += w * bf16_bits_to_double(row[c]);
        }
        for (int32_t c = 0; c < H; ++c) out[i * H + c] = double_to_bf16_bits(acc[c]);
    }
    return ORACLE_OK;
}

// Low-latency combine, fixed-order fp32 definition (same arguments as
// oracle_ll_combine).  The weighted reduction of [API] "IB-GDA Kernels" taken
// as the method computes it: the token's valid slots are visited in ascending
// (expert id, slot k), and each adds w * y with one fused multiply-add
// (binary32, one rounding of the exact w * y + acc), starting from +0; the
// result is rounded once to bf16:
//   acc = +0;  for (e, k) ascending:  acc = fma(w[s][t][k], y[e][slot][i], acc)
//   out = bf16(acc)
int oracle_ll_combine_fp32(int32_t R, int32_t E, int32_t T, int32_t K, int32_t H, int32_t Tmax,
                           const uint16_t* y, const int64_t* topk_idx, const float* topk_weights,
                           const int32_t* src_info, const int32_t* layout_range, uint16_t* out,
                           const int64_t* tokens, int64_t n_tokens, const int32_t* rank_mask) {
    if (!shape_ok(R, E, T, K) || H < 1 || Tmax < T) return ORACLE_BAD_ARG;
    const int32_t L = E / R;
    const int64_t cap = (int64_t)R * Tmax;
    const int64_t G = (int64_t)R * T;
    const int64_t n = tokens != nullptr ? n_tokens : G;
    std::vector<float> chain(H);
    std::vector<std::pair<int64_t, int32_t>> visit;   // (expert id, k), sorted
    for (int64_t i = 0; i < n; ++i) {
        const int64_t g = tokens != nullptr ? tokens[i] : i;
        if (g < 0 || g >= G) return ORACLE_BAD_ARG;
        const int32_t s = (int32_t)(g / T), t = (int32_t)(g % T);
        visit.clear();
        for (int32_t k = 0; k < K; ++k) {
            const int64_t e = topk_idx[g * K + k];
            if (e == -1) continue;
            if (e < -1 || e >= E) return ORACLE_BAD_TOPK;
            if (rank_mask != nullptr && (rank_mask[s] != 0 || rank_mask[e / L] != 0)) continue;
            visit.emplace_back(e, k);
        }
        std::sort(visit.begin(), visit.end());
        std::fill(chain.begin(), chain.end(), 0.0f);
        for (const auto& slot_of : visit) {
            const int64_t e = slot_of.first;
            const int32_t k = slot_of.second;
            const int32_t first = layout_range[(e * R + s) * 2 + 0];
            const int32_t count = layout_range[(e * R + s) * 2 + 1];
            int64_t slot = -1;
            for (int32_t p = first; p < first + count; ++p)
                if (src_info[e * cap + p] == t) { slot = p; break; }
            if (slot < 0) return ORACLE_NOT_FOUND;
            const float w32 = topk_weights[g * K + k];
            const uint16_t* yrow = y + (e * cap + slot) * H;
            for (int32_t c = 0; c < H; ++c) chain[c] = std::fma(w32, bf16_bits_to_float(yrow[c]), chain[c]);
        }
        for (int32_t c = 0; c < H; ++c) out[i * H + c] = float_to_bf16_bits(chain[c]);
    }
    return ORACLE_OK;
}

// ---------------------------------------------------------------- FP8 (LL)
//
// [API] "IB-GDA Kernels" / "Low-Latency Inference with FP8": the low-latency
// path can quantise to FP8 (use_fp8), and the packed result becomes a tuple
// (the example indexes packed_x[0]).  The pages give no format; the reading
// taken: OCP FP8 E4M3 (bias 7, 3 mantissa bits, largest finite 448, no
// infinities), one fp32 scale per token per block of 128 hidden channels,
//   scale = amax(|x| over the block) / 448       (fp32 division, nearest even)
//   code  = e4m3(x * (448 / amax))                (fp32 division and product,
//                                                  each nearest even; then E4M3
//                                                  nearest even, saturating)
// with scale = 1 and all codes 0 for an all-zero block; x ~= value(code) * scale.

// E4M3 code of a finite value, round to nearest even, saturating at +-448.
static uint8_t e4m3_encode(double v) {
    const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
    double a = std::fabs(v);
    if (a == 0.0) return sign;
    // spacing of E4M3 values at a: 2^(e-3) for a in [2^e, 2^(e+1)), e >= -6;
    // subnormals (a < 2^-6) step by 2^-9
    int e;
    std::frexp(a, &e);                   // a = m * 2^e, m in [0.5, 1): leading bit 2^(e-1)
    int qexp = (e - 1) - 3;
    if (qexp < -9) qexp = -9;
    double r = std::ldexp(std::nearbyint(std::ldexp(a, -qexp)), qexp);
    if (r > 448.0) r = 448.0;            // saturate to the largest finite value
    if (r == 0.0) return sign;
    if (r < std::ldexp(1.0, -6)) {       // subnormal: exponent field 0
        const int m = (int)std::ldexp(r, 9);
        return (uint8_t)(sign | m);
    }
    int re;
    std::frexp(r, &re);                  // r in [2^(re-1), 2^re)
    const int E = (re - 1) + 7;
    const int m = (int)(std::ldexp(r, -(re - 1)) * 8.0) - 8;
    return (uint8_t)(sign | (E << 3) | m);
}

void oracle_fp8_e4m3_encode(const double* in, uint8_t* out, int64_t n) {
    for (int64_t i = 0; i < n; ++i) out[i] = e4m3_encode(in[i]);
}

// Quantise n bf16 rows of H channels in blocks of `block` channels:
//   codes[r][c] (u8), scales[r][c / block] (f32).
int oracle_quantize_e4m3_blocks(const uint16_t* rows, int64_t n, int32_t H, int32_t block,
                                uint8_t* codes, float* scales) {
    if (H < 1 || block < 1 || H % block != 0) return ORACLE_BAD_ARG;
    const int32_t nb = H / block;
    for (int64_t r = 0; r < n; ++r) {
        for (int32_t b = 0; b < nb; ++b) {
            float amax = 0.0f;
            for (int32_t i = 0; i < block; ++i)
                amax = std::max(amax, (float)std::fabs(bf16_bits_to_double(rows[r * H + b * block + i])));
            const float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
            const float inv = amax > 0.0f ? 448.0f / amax : 0.0f;
            scales[r * nb + b] = scale;
            for (int32_t i = 0; i < block; ++i) {
                const float x = (float)bf16_bits_to_double(rows[r * H + b * block + i]);
                const float q = x * inv;
                codes[r * H + b * block + i] = e4m3_encode((double)q);
            }
        }
    }
    return ORACLE_OK;
}

// ------------------------------------------------- load balance (redundant experts)
//
// [V2] "10.2 与 EP 的关联能力": lb_prefetch_weights moves the weights of
// redundant expert replicas in before the expert compute, and lb_reduce_grads
// folds the replicas' gradients back into the original experts in the backward
// pass, both keyed by redundancy_mapping.  The page gives no shapes; readings:
//   * every expert's weights (or gradients) are one block of W bf16 values:
//     expert_weights [E][W], redundant weights/grads [N][W];
//   * redundancy_mapping[i] is the original expert of replica i, -1 = unused;
//   * prefetch: redundant[i] = expert_weights[mapping[i]] (bit copy);
//   * reduce:   expert_grads[e] = bf16( expert_grads[e] + sum over replicas i
//               of e, ascending i, of redundant_grads[i] )  (fp64 here).
int oracle_lb_prefetch_weights(const uint16_t* expert_weights, int32_t E, int64_t W,
                               const int32_t* mapping, int32_t N, uint16_t* redundant_weights) {
    if (E < 1 || W < 1 || N < 0) return ORACLE_BAD_ARG;
    for (int32_t i = 0; i < N; ++i) {
        const int32_t e = mapping[i];
        if (e == -1) continue;
        if (e < -1 || e >= E) return ORACLE_BAD_TOPK;
        for (int64_t c = 0; c < W; ++c) redundant_weights[(int64_t)i * W + c] = expert_weights[(int64_t)e * W + c];
    }
    return ORACLE_OK;
}

int oracle_lb_reduce_grads(const uint16_t* redundant_grads, const int32_t* mapping, int32_t N,
                           uint16_t* expert_grads, int32_t E, int64_t W) {
    if (E < 1 || W < 1 || N < 0) return ORACLE_BAD_ARG;
    for (int32_t i = 0; i < N; ++i)
        if (mapping[i] < -1 || mapping[i] >= E) return ORACLE_BAD_TOPK;
    for (int32_t e = 0; e < E; ++e) {
        bool any = false;
        for (int32_t i = 0; i < N; ++i) any = any || mapping[i] == e;
        if (!any) continue;   // untouched
        for (int64_t c = 0; c < W; ++c) {
            double acc = bf16_bits_to_double(expert_grads[(int64_t)e * W + c]);
            for (int32_t i = 0; i < N; ++i)
                if (mapping[i] == e) acc += bf16_bits_to_double(redundant_grads[(int64_t)i * W + c]);
            expert_grads[(int64_t)e * W + c] = double_to_bf16_bits(acc);
        }
    }
    return ORACLE_OK;
}

// Gradient reduction, fixed-order fp32 definition (same arguments as
// oracle_lb_reduce_grads): an fp32 accumulator starts at the original
// gradient and adds, one binary32 addition each, the replicas' gradients in
// ascending replica index; one rounding to bf16 at the end.
int oracle_lb_reduce_grads_fp32(const uint16_t* redundant_grads, const int32_t* mapping, int32_t N,
                                uint16_t* expert_grads, int32_t E, int64_t W) {
    if (E < 1 || W < 1 || N < 0) return ORACLE_BAD_ARG;
    for (int32_t i = 0; i < N; ++i)
        if (mapping[i] < -1 || mapping[i] >= E) return ORACLE_BAD_TOPK;
    std::vector<int32_t> replicas;
    for (int32_t e = 0; e < E; ++e) {
        replicas.clear();
        for (int32_t i = 0; i < N; ++i)
            if (mapping[i] == e) replicas.push_back(i);     // ascending replica index
        if (replicas.empty()) continue;                     // untouched
        for (int64_t c = 0; c < W; ++c) {
            float g32 = bf16_bits_to_float(expert_grads[(int64_t)e * W + c]);
            for (const int32_t i : replicas) g32 = g32 + bf16_bits_to_float(redundant_grads[(int64_t)i * W + c]);
            expert_grads[(int64_t)e * W + c] = float_to_bf16_bits(g32);
        }
    }
    return ORACLE_OK;
}

}  // extern "C"
