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
    const int64_t* topk_idx;   // [G][K]
    uint8_t* is_token_in_rank; // [G][R]
    int* num_tokens_per_rank;  // [R][R], zeroed before launch
    int* num_tokens_per_expert;// [R][E], zeroed before launch
    int* err;
    int R, E, L, T, K;
};
constexpr int kLayoutThreads = 256;
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
constexpr int kScanTile = 256;   // tokens per tile == threads per block
cudaError_t launch_scan(const ScanParams& p, cudaStream_t stream);

// ---------------------------------------------------- dispatch (row copies)
enum DispatchMode { kModeNormal = 0, kModeCached = 1, kModeLowLatency = 2, kModeLowLatencyFp8 = 3 };
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
    const int* slot_map;               // [G][K]
    const int* rank_mask;              // [R], 0 active / 1 masked
    int64_t ll_capacity;               // R * Tmax slots per expert
    uint16_t* recv_x;                  // normal/cached: [cap][H]; LL: [E][ll_cap][H]
    // low latency, FP8 form (recv_x unused)
    uint8_t* recv_fp8;                 // [E][ll_cap][H] E4M3 codes
    float* recv_scales;                // [E][ll_cap][H/128]
    int* err;
    long long G;
    int R, E, L, T, K, H;
    int splits;                        // warps per token (column slices of the row)
};
cudaError_t launch_dispatch(int mode, const DispatchParams& p, cudaStream_t stream);

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
    int* err;
    long long G;
    int R, K, H;
    int splits;                        // warps per token (column slices of the row)
};
cudaError_t launch_combine(const CombineParams& p, int num_sms, cudaStream_t stream);

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
cudaError_t ll_prepare(int E);   // once per device: shared-memory opt-in

struct LLCombineParams {
    const uint16_t* y;          // [E][ll_cap][H]
    const int64_t* topk_idx;    // [G][K]
    const float* topk_weights;  // [G][K]
    const int* src_info;        // [E][ll_cap]
    const int* layout_range;    // [E][R][2]
    const int* rank_mask;       // [R], 0 active / 1 masked
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
