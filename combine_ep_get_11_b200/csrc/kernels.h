// Internal launch interface between the C ABI (abi.cu) and the kernels.
// Plain structs of device pointers and sizes; one launcher per kernel.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace ep {

// Warps per token for the row kernels: a token's row may be cut into column
// slices (whole 512-byte warp strides) handled by separate warps.  Measured on
// B200: the fan-out copy gains ~2% from two warps per row (more stores in
// flight per row); the gather-reduce kernels do best with one.
inline int dispatch_splits(int H) { return (H / 8) >= 64 ? 2 : 1; }
inline int combine_splits(int) { return 1; }

// ------------------------------------------------------------------ layout
struct LayoutParams {
    const int64_t* topk_idx;   // [S][T][K]   (S source ranks in this launch)
    uint8_t* is_token_in_rank; // [S][T][R]
    int* num_tokens_per_rank;  // [S][R], zeroed before launch
    int* num_tokens_per_expert;// [S][E], zeroed before launch
    int* err;
    int R, E, L, T, K;
    int num_src;               // S: R, or the ranks of one shard
};
constexpr int kLayoutThreads = 512;
cudaError_t launch_layout(const LayoutParams& p, cudaStream_t stream);

// -------------------------------------------------------------------- scan
// Decoupled-lookback scan over the G = R*T tokens in (rank, token) order of
// the R membership columns of is_token_in_rank.  Writes send_head and samples
// the running counts at every channel boundary; the last tile to finish turns
// the samples into the handle matrices.
struct ScanParams {
    const uint8_t* is_token_in_rank;   // [G][R]
    const int* num_tokens_per_expert;  // [R][E]
    unsigned long long* status;        // [num_tiles][R] call-tagged words (zero words never match)
    unsigned long long* ticket;        // block ticket: only incremented (or zeroed with status)
    unsigned long long* rank_start;    // [R][R] call-tagged P(s*T)[d] (zeroed with the ticket if at all)
    const int* base;                   // [R] or null: added to every P value (tokens of earlier shards)
    int* send_head;                    // [G][R]
    int* rank_prefix_matrix;           // [R][R]
    int* channel_prefix_matrix;        // [R][R][C]
    int* recv_channel_prefix_matrix;   // [R][R][C]
    long long* recv_rank_offset;       // [R+1]
    int* num_recv_tokens_per_expert;   // [R][L]
    int* err;
    long long G;
    int R, E, L, T, C, q, num_tiles;
};
// The handle matrices, recv_rank_offset and num_recv_tokens_per_expert may be
// null (a sharded exchange takes its offsets from launch_shard_offsets).
constexpr int kScanTile = 256;   // tokens per tile == threads per block
cudaError_t launch_scan(const ScanParams& p, cudaStream_t stream);

// ---------------------------------------------------- dispatch (row copies)
enum DispatchMode { kModeNormal = 0, kModeCached = 1, kModeLowLatency = 2, kModeLowLatencyFp8 = 3,
                    kModeSharded = 4 };
constexpr int kMaxShards = 32;   // GPUs of a sharded exchange (each hosts >= 1 virtual rank)
constexpr int kFp8Block = 128;   // hidden channels per FP8 scale

struct DispatchParams {
    const uint16_t* x;                 // [G][H]
    // normal / cached
    const int* send_head;              // [G][R]
    const long long* recv_rank_offset; // [R+1]
    int64_t recv_capacity;             // rows of recv_x
    // normal only (metadata rows)
    const int64_t* topk_idx;           // [G][K]
    const float* topk_weights;         // [G][K] or null
    int64_t* recv_topk_idx;            // [cap][K] or null
    float* recv_topk_weights;          // [cap][K] or null
    int* recv_src_idx;                 // [cap] or null
    // low latency
    int* slot_map;                     // [G][K]: read (slot scan) or written (direct slots)
    const int* rank_mask;              // [R], 0 active / 1 masked
    int64_t ll_capacity;               // R * Tmax slots per expert
    // direct slots (ll_rank_kernel ran before; null ll_cnt: slots from slot_map)
    const int* ll_cnt;                 // [R][E] tokens of source s naming e
    const int* ll_within;              // [G][K] rank of the token among its source's tokens naming e
    int* ll_src_info;                  // [E][ll_capacity] written by the copy
    int* ll_layout_range;              // [E][R][2] written by the copy
    int* ll_count;                     // [E] written by the copy
    uint16_t* recv_x;                  // normal/cached: [cap][H]; LL: [E][ll_cap][H]
    // low latency, FP8 form (recv_x unused)
    uint8_t* recv_fp8;                 // [E][ll_cap][H] E4M3 codes
    float* recv_scales;                // [E][ll_cap][H/128]
    // sharded: destination d's rows live in shard d / ranks_per_shard's buffers,
    // starting at row dst_offset[d] (pointers valid on this GPU: own or peer memory)
    const long long* dst_offset;       // [R]
    int ranks_per_shard;
    uint16_t* shard_rows[kMaxShards];  // [cap][H] per shard
    int64_t* shard_idx[kMaxShards];    // [cap][K] per shard, or null
    float* shard_w[kMaxShards];        // [cap][K] per shard, or null
    int* shard_src[kMaxShards];        // [cap] per shard, or null
    int* err;
    long long G;
    int R, E, L, T, K, H;
    int splits;                        // warps per token (column slices of the row)
    int num_sms;                       // the device's SM count (launch geometry)
};
// after_scan: launched right behind the handle / slot scan kernel, which lets
// it start early (programmatic dependent launch); only the normal and packed
// forms make use of it.
cudaError_t launch_dispatch(int mode, const DispatchParams& p, cudaStream_t stream, bool after_scan = false);

// ----------------------------------------------------------------- combine
struct CombineParams {
    const uint16_t* y;                 // [y_rows][H]
    int64_t y_rows;
    const int* send_head;              // [G][R]
    const long long* recv_rank_offset; // [R+1]
    const float* recv_topk_weights;    // [y_rows][K] or null
    const uint16_t* bias0;             // [G][H] or null
    const uint16_t* bias1;             // [G][H] or null
    uint16_t* out_x;                   // [G][H]
    float* out_topk_weights;           // [G][K] or null
    // sharded: the rows of destination d are read from shard d / ranks_per_shard
    // (own or peer memory), from row dst_offset[d]; recv_rank_offset / y unused
    bool sharded;
    const long long* dst_offset;       // [R]
    int ranks_per_shard;
    const uint16_t* shard_y[kMaxShards];   // [y_rows][H] per shard
    const float* shard_w[kMaxShards];      // [y_rows][K] per shard, or null
    int self_shard;                        // the tables' index of this GPU's own buffers
    int* err;
    long long G;
    int R, K, H;
    int splits;                        // warps per token (column slices of the row)
};
cudaError_t launch_combine(const CombineParams& p, int num_sms, cudaStream_t stream);

// ---------------------------------------------------------- sharded offsets
// From the gathered layout counts of all R ranks, for the shard hosting ranks
// [r0, r0 + ranks_per_shard): the tokens of earlier shards per destination (the
// scan's base), each destination's first row in its shard's receive buffer,
// this shard's receive rows and its local experts' receive counts.
struct ShardOffsetsParams {
    const int* num_tokens_per_rank_all;    // [R][R]
    const int* num_tokens_per_expert_all;  // [R][E]
    int* base;                             // [R]
    long long* dst_offset;                 // [R]
    long long* num_recv_rows;              // [1] or null
    int* num_recv_tokens_per_expert;       // [ranks_per_shard][L] or null
    int R, E, L, r0, ranks_per_shard;
};
cudaError_t launch_shard_offsets(const ShardOffsetsParams& p, cudaStream_t stream);

// ------------------------------------------------------------ low latency
// Low-latency slot assignment: a decoupled-lookback scan over 256-token tiles
// whose columns are the E experts (the same scheme as the handle scan).
struct LLCountParams {
    const int64_t* topk_idx;   // [G][K]
    int* slot_map;             // [G][K]
    int* packed_recv_count;    // [E]  (= [R][L])
    int* src_info;             // [E][ll_cap]
    int* layout_range;         // [E][R][2]
    unsigned long long* status;    // [num_tiles][E] tile status words (call-tagged, never cleared)
    unsigned long long* src_begin; // [R][E] first slot of each source (call-tagged), sources of > 1 tile
    unsigned long long* ticket;    // block ticket, only ever incremented
    const int* rank_mask;      // [R], 0 active / 1 masked
    int* err;
    long long G;
    int R, E, T, K;
    int64_t ll_capacity;
    int tiles_per_src;         // ceil(T / kLLTile)
    int num_tiles;             // R * tiles_per_src
};
constexpr int kLLTile = 256;   // tokens per tile == threads per block
cudaError_t launch_ll_count(const LLCountParams& p, cudaStream_t stream);

// Direct low-latency slots, for sources of at most kLLDirectMaxT tokens (decode
// batches): slot(s, t, e) = base[s][e] + within[s][t][e], where within counts
// the tokens t' < t of source s naming e and base the tokens of sources s' < s
// naming e.  ll_rank_kernel (one block per source, one thread per token) writes
// the source's per-expert counts and every (token, k)'s within; the copy kernel,
// launched behind it, sums the counts of the earlier sources (base) and writes
// src_info, layout_range and the per-expert counts.  No block waits on another.
struct LLRankParams {
    const int64_t* topk_idx;   // [G][K]
    const int* rank_mask;      // [R]
    int* cnt;                  // [R][E] tokens of source s naming e
    int* within;               // [G][K] tokens before t in its source naming slot k's expert (-1: not sent)
    int* err;
    int R, E, T, K;
};
#ifndef EP_LL_DIRECT_MAX_T
#define EP_LL_DIRECT_MAX_T 256
#endif
constexpr int kLLDirectMaxT = EP_LL_DIRECT_MAX_T;   // <= kLLTile: one block per source
cudaError_t launch_ll_rank(const LLRankParams& p, cudaStream_t stream);
cudaError_t ll_prepare(int E);   // once per device: shared-memory opt-in

struct LLCombineParams {
    const uint16_t* y;          // [E][ll_cap][H]
    const int64_t* topk_idx;    // [G][K]
    const float* topk_weights;  // [G][K]
    const int* src_info;        // [E][ll_cap]
    const int* layout_range;    // [E][R][2]
    const int* rank_mask;       // [R], 0 active / 1 masked
    const int* slot_hint;       // [G][K] slots of the last low-latency dispatch, or null (checked against the handle)
    uint16_t* out_x;            // [G][H]
    int* err;
    long long G;
    int R, E, T, K, H;
    int64_t ll_capacity;
    int splits;                 // warps per token (column slices of the row)
};
cudaError_t launch_ll_combine(const LLCombineParams& p, int num_sms, cudaStream_t stream);
cudaError_t launch_set_mask(int* rank_mask, int rank, int value, cudaStream_t stream);

// ------------------------------------------------------------ load balance
struct LBParams {
    uint16_t* expert;           // prefetch: expert weights [E][W] (read); reduce: expert grads (in/out)
    uint16_t* redundant;        // prefetch: replica weights [N][W] (written); reduce: replica grads (read)
    const int* mapping;         // [N] replica -> original expert, -1 unused
    int* err;
    long long Wv;               // 16-byte vectors per expert block (W / 8)
    int E, N;
};
cudaError_t launch_lb_prefetch(const LBParams& p, cudaStream_t stream);
cudaError_t launch_lb_reduce(const LBParams& p, cudaStream_t stream);

}  // namespace ep
