/*
 * ep.h -- C ABI of the B200 MoE dispatch/combine library (libep.so).
 *
 * Mixture-of-experts token dispatch and combine, as DeepSeek's DeepEP `Buffer`
 * defines them, for R "virtual" expert-parallel ranks that all live on one
 * GPU: rank s owns the token rows x[s] of one [R][T][H] tensor, so dispatch
 * and combine are permutations of device memory.
 *
 * Sources of the operations (web pages about DeepEP):
 *   [API]   "DeepEP Buffer Class API for Expert Parallel Communication:
 *            Architecture and Usage"
 *   [REUSE] "How DeepEP Optimizes Handle Reuse for Repeated Dispatches"
 *   [ARCH]  "Architecture" (DeepEP-Lib)
 *   [CORE]  "Core-Implementation" (DeepEP C++ runtime)
 *
 * Conventions for every call
 *   - Tensor pointers are DEVICE memory allocated by the caller, contiguous,
 *     row-major, 16-byte aligned.  The library never takes ownership and
 *     allocates nothing per call (ep_create allocates a fixed workspace).
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Every call is ordered on the caller's stream; a non-null wait_event is
 *     waited on first (the pages' `previous_event`).
 *   - Return value: an ep_status.  Argument errors are found on the host
 *     before anything is launched.  Errors that only the GPU can see (an
 *     expert id out of range, a receive buffer too small, a device wait that
 *     ran out) are recorded in a device error word and returned by the next
 *     ep_sync_status; kernels never trap.
 *
 * Notation: R = num_ranks, E = num_experts, L = E / R local experts per rank,
 * T = num_tokens per rank, H = hidden, K = topk, C = num_channels,
 * Tmax = ll_max_tokens_per_rank, G = R * T global tokens, g = s * T + t.
 * Expert e lives on rank e / L as local expert e % L; -1 marks an unused slot.
 */
#ifndef EP_B200_H
#define EP_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define EP_API __attribute__((visibility("default")))
#else
#define EP_API
#endif

/* Same types as cudaStream_t / cudaEvent_t; declared here so the header
 * needs no CUDA include. */
typedef struct CUstream_st* ep_stream_t;
typedef struct CUevent_st* ep_event_t;

typedef enum ep_status {
    EP_OK = 0,
    EP_ERR_INVALID_ARG = 1,     /* bad argument or unsupported shape */
    EP_ERR_ALIGNMENT = 2,       /* pointer not 16-byte aligned (x of the FP8 packing: 32), or
                                   H*2 not a multiple of 16 */
    EP_ERR_CAPACITY = 3,        /* a receive buffer is too small */
    EP_ERR_BAD_TOPK = 4,        /* an expert id outside [-1, E) */
    EP_ERR_HANDLE_MISMATCH = 5, /* handle arrays missing or not made for this context */
    EP_ERR_TIMEOUT = 6,         /* a bounded device wait ran out */
    EP_ERR_CUDA = 7,            /* a CUDA runtime call failed */
    EP_ERR_UNIMPLEMENTED = 8
} ep_status;

/* Problem shape.  [ARCH] "Configuration System" tunes kernels per rank
 * count; here launch geometry is derived from the device, and only the
 * channel count (which shapes the channel prefix matrices) is configurable.
 * Limits: 1 <= R <= 32; E % R == 0, E <= 4096; T >= 0; 1 <= K <= 32;
 * H % 8 == 0, 8 <= H <= 32768; 1 <= C <= 1024; Tmax == 0 (means T) or
 * Tmax >= T; R * T * max(R, K) < 2^31. */
typedef struct ep_config {
    int32_t num_ranks;
    int32_t num_experts;
    int32_t num_tokens;
    int32_t hidden;
    int32_t topk;
    int32_t num_channels;
    int32_t ll_max_tokens_per_rank;
} ep_config;

typedef struct ep_ctx ep_ctx;

/* The dispatch handle ([REUSE] "What the Handle Contains"): rank_prefix_matrix,
 * channel_prefix_matrix, recv_channel_prefix_matrix, recv_src_idx,
 * is_token_in_rank and send_head, plus two conveniences (the receive offsets
 * and per-expert receive counts).  All arrays are caller-allocated device
 * memory, filled by ep_dispatch and read by ep_dispatch_cached / ep_combine.
 *
 *   rank_prefix_matrix[i][d]         i32 [R][R]    sum_{s<=i} tokens s -> d
 *   channel_prefix_matrix[s][d][c]   i32 [R][R][C] tokens of s for d in channels 0..c
 *   recv_channel_prefix_matrix[d][s][c] i32 [R][R][C] first receive position of
 *                                    block (s, c) within rank d's rows
 *   recv_src_idx[n]                  i32 [capacity] source token t of receive row n
 *   is_token_in_rank[s][t][d]        u8  [R][T][R]
 *   send_head[s][t][d]               i32 [R][T][R] receive position of (s, t)
 *                                    within rank d's rows, or -1
 *   recv_rank_offset[d]              i64 [R+1]     first row of rank d; [R] = N
 *   num_recv_tokens_per_expert[d][j] i32 [R][L]
 *
 * Receive rows of rank d are [recv_rank_offset[d], recv_rank_offset[d+1]) of
 * one concatenated buffer, ordered by source rank, then token.  Channel c of
 * a rank covers tokens [min(c*q, T), min((c+1)*q, T)), q = ceil(T / C).
 * The handle stays valid only while topk_idx is unchanged ([REUSE]
 * "Performance Contract and Constraints"). */
typedef struct ep_handle {
    int32_t* rank_prefix_matrix;
    int32_t* channel_prefix_matrix;
    int32_t* recv_channel_prefix_matrix;
    int32_t* recv_src_idx;
    uint8_t* is_token_in_rank;
    int32_t* send_head;
    int64_t* recv_rank_offset;
    int32_t* num_recv_tokens_per_expert;
} ep_handle;

/* Element counts of each handle array (recv_src_idx: worst case R*T*min(R,K)),
 * and of the low-latency arrays, for a context. */
typedef struct ep_handle_sizes {
    int64_t rank_prefix_matrix;
    int64_t channel_prefix_matrix;
    int64_t recv_channel_prefix_matrix;
    int64_t recv_src_idx_max;
    int64_t is_token_in_rank;
    int64_t send_head;
    int64_t recv_rank_offset;
    int64_t num_recv_tokens_per_expert;
    int64_t ll_packed_recv_x;     /* bf16 elements of [R][L][R*Tmax][H] */
    int64_t ll_packed_recv_count; /* [R][L] */
    int64_t ll_src_info;          /* [R][L][R*Tmax] */
    int64_t ll_layout_range;      /* [R][L][R][2] */
} ep_handle_sizes;

/* Create a context on the current CUDA device: validates the shape ([CORE]
 * "Memory Alignment and Validation": rows must be whole 16-byte vectors) and
 * allocates the fixed device workspace (scan state, error word, internal
 * layout arrays).  *out is set only on EP_OK.  Host-only validation runs
 * before any CUDA call, so a bad shape fails without a GPU.
 *
 * Concurrency: a context's workspace is shared by its calls -- the handle
 * scan's ticket counter and status words, the low-latency slot scan's counter,
 * status words and slot map (which ep_ll_combine reads as a hint), the direct
 * slots' per-source counts and ranks, the rank mask, the internal layout arrays
 * and the error word.  Calls on one context
 * must therefore be ordered with respect to each other on the GPU: issue them
 * on one stream (or order the streams with events), and from one host thread
 * at a time.  Two dispatches of one context running at once would interleave
 * their tickets and break the scans' call tags.  Different contexts are
 * independent and may run concurrently. */
EP_API int ep_create(const ep_config* cfg, ep_ctx** out);

/* Free the context and its workspace ([API] "Explicit Resource Cleanup").
 * Waits for nothing: the caller must not have work in flight that uses it. */
EP_API int ep_destroy(ep_ctx* ctx);

/* Bytes of device workspace the context holds. */
EP_API int ep_workspace_bytes(const ep_ctx* ctx, size_t* bytes);

/* Sizes of the handle and low-latency arrays for this context. */
EP_API int ep_handle_layout(const ep_ctx* ctx, ep_handle_sizes* sizes);

/* Human-readable name of a status code (static string). */
EP_API const char* ep_status_string(int status);

/* Description of the last host-side error on this context (static buffer in
 * the context; empty if none). */
EP_API const char* ep_last_error(const ep_ctx* ctx);

/* Synchronize `stream`, then return and clear the device error word (EP_OK if
 * no kernel recorded an error since the last call).  The only blocking call
 * besides ep_get_num_recv, ep_dispatch with num_recv_host and the mask query. */
EP_API int ep_sync_status(ep_ctx* ctx, ep_stream_t stream);
/* (When it reports EP_ERR_TIMEOUT it also moves the scans' ticket counters up
 * to the next multiple of their tile counts, so the following calls start from
 * a consistent state.) */

/* Test support for the bounded waits.  Synchronizes the device, then adds
 * `delta` to the ticket counters of the handle scan and the low-latency slot
 * scan.  A delta that is not a multiple of a scan's tile count makes the
 * scan's next call give its tiles two different call tags: the tiles waiting
 * for a word tagged with the other number give up after the wait limit (about
 * a second) and record EP_ERR_TIMEOUT; that call's outputs are then undefined.
 * ep_sync_status realigns the counters. */
EP_API int ep_test_offset_tickets(ep_ctx* ctx, int64_t delta);

/* Number of kernels this library has launched in this process (all contexts). */
EP_API uint64_t ep_kernel_launch_count(void);

/* Handle check for the reuse contract ([REUSE] "Performance Contract and
 * Constraints": a handle stays valid only while topk_idx is unchanged).
 * Recomputes each token's destination ranks from topk_idx (i64 [R][T][K]) and
 * compares them with the handle's is_token_in_rank and send_head (>= 0 exactly
 * for those ranks, and below each rank's receive count from recv_rank_offset).
 * A difference records EP_ERR_HANDLE_MISMATCH for ep_sync_status.  Reads
 * G*(K*8 + R*5) bytes; stream-ordered; blocks nothing.  Not on a sharded
 * context. */
EP_API int ep_check_handle(ep_ctx* ctx, const int64_t* topk_idx, const ep_handle* handle,
                           ep_stream_t stream, ep_event_t wait_event);

/* Dispatch layout ([API] "Configuration and Layout Helpers", [ARCH] table
 * "Buffer.get_dispatch_layout").
 *   topk_idx              i64 [R][T][K]  input
 *   num_tokens_per_rank   i32 [R][R]     out: [s][d] tokens of s with an expert on d
 *   num_tokens_per_expert i32 [R][E]     out: [s][e] slots of s naming e
 *   is_token_in_rank      u8  [R][T][R]  out
 * Expert ids outside [-1, E) record EP_ERR_BAD_TOPK and count as -1. */
EP_API int ep_get_dispatch_layout(ep_ctx* ctx, const int64_t* topk_idx,
                           int32_t* num_tokens_per_rank, int32_t* num_tokens_per_expert,
                           uint8_t* is_token_in_rank, ep_stream_t stream, ep_event_t wait_event);

/* Dispatch ([API] "Dispatch Operation"; [REUSE] "Handle Creation").
 * Builds the handle and scatters every token row, with its top-k ids and
 * weights, into the receive rows of each rank that owns one of its experts.
 *   x                 bf16 [R][T][H]
 *   topk_idx          i64  [R][T][K]
 *   topk_weights      f32  [R][T][K]   nullable (then recv_topk_weights is not written)
 *   num_tokens_per_rank / num_tokens_per_expert / is_token_in_rank: the
 *                     layout from ep_get_dispatch_layout; pass all three or
 *                     all null (then the layout is computed here, into
 *                     handle->is_token_in_rank)
 *   handle            arrays to fill (see ep_handle)
 *   recv_x            bf16 [recv_capacity_rows][H]  out; nullable together with
 *                     capacity 0 to build only the handle
 *   recv_topk_idx     i64  [capacity][K] out, nullable: local expert id on the
 *                     receiving rank, -1 for slots owned elsewhere
 *   recv_topk_weights f32  [capacity][K] out, nullable: weight, 0 elsewhere
 *   num_recv_host     nullable host pointer: if set, the call synchronizes the
 *                     stream once after the handle is built, stores the
 *                     number of receive rows N there and returns
 *                     EP_ERR_CAPACITY before writing any row if N > capacity
 *                     (the pages' CPU-GPU sync to learn receive counts).
 * Without num_recv_host nothing blocks; rows beyond the capacity are dropped
 * and EP_ERR_CAPACITY is recorded for ep_sync_status. */
EP_API int ep_dispatch(ep_ctx* ctx, const uint16_t* x, const int64_t* topk_idx, const float* topk_weights,
                const int32_t* num_tokens_per_rank, const int32_t* num_tokens_per_expert,
                const uint8_t* is_token_in_rank, const ep_handle* handle,
                uint16_t* recv_x, int64_t* recv_topk_idx, float* recv_topk_weights,
                int64_t recv_capacity_rows, int64_t* num_recv_host,
                ep_stream_t stream, ep_event_t wait_event);

/* Receive counts from a layout ([REUSE] "Performance Contract and Constraints":
 * the number of tokens each rank receives is only known after the layout, and
 * learning it costs one CPU-GPU synchronisation).  Copies num_tokens_per_rank
 * (i32 [R][R], device, from ep_get_dispatch_layout on this stream) to the host,
 * synchronizes the stream once, and writes
 *   *num_recv_host               = N = sum over s, d of num_tokens_per_rank[s][d]
 *   num_recv_per_rank_host[d]    = N_d = sum over s of num_tokens_per_rank[s][d]
 *                                  (nullable; R int64 values in host memory)
 * N is the receive capacity ep_dispatch needs.  Not on a sharded context
 * (ep_sharded_handle returns each GPU's count). */
EP_API int ep_get_num_recv(ep_ctx* ctx, const int32_t* num_tokens_per_rank, int64_t* num_recv_host,
                           int64_t* num_recv_per_rank_host, ep_stream_t stream, ep_event_t wait_event);

/* Cached dispatch ([REUSE] "Fast Path Dispatch with Handle Reuse"): scatter
 * new rows x with a handle from an earlier ep_dispatch of the same routing.
 * No layout, no prefix work, no host synchronization; top-k arrays are not
 * accepted (the handle already fixes the layout).
 *   x       bf16 [R][T][H]; recv_x bf16 [recv_capacity_rows][H] out. */
EP_API int ep_dispatch_cached(ep_ctx* ctx, const uint16_t* x, const ep_handle* handle,
                       uint16_t* recv_x, int64_t recv_capacity_rows,
                       ep_stream_t stream, ep_event_t wait_event);

/* Combine ([API] "Combine Operation"): reduce by addition, back in source
 * order, the expert outputs y that sit in the receive rows of a dispatch:
 *   out_x[s][t] = bf16( sum over d ascending with h = send_head[s][t][d] >= 0
 *                       of y[recv_rank_offset[d] + h]  (+ bias0[s][t] + bias1[s][t]) )
 * accumulated in fp32 in that fixed order, rounded once to bf16 (nearest even).
 *   y                 bf16 [num_recv_rows][H]
 *   recv_topk_weights f32  [num_recv_rows][K] nullable; if given with
 *                     out_topk_weights, out_topk_weights[s][t][k] is the same
 *                     ascending-rank fp32 sum of the received weight rows
 *   bias0, bias1      bf16 [R][T][H] nullable
 *   out_x             bf16 [R][T][H] out
 * A token routed nowhere gets bf16(bias0 + bias1), i.e. +0 without bias.
 * Rows at or past num_recv_rows are never read (EP_ERR_CAPACITY recorded). */
EP_API int ep_combine(ep_ctx* ctx, const uint16_t* y, int64_t num_recv_rows, const ep_handle* handle,
               const float* recv_topk_weights, const uint16_t* bias0, const uint16_t* bias1,
               uint16_t* out_x, float* out_topk_weights,
               ep_stream_t stream, ep_event_t wait_event);

/* Low-latency dispatch ([API] "IB-GDA Kernels", "Low-Latency Inference with
 * FP8" (bf16 here)): pack tokens expert-major, bounded by Tmax per rank.
 *   x                 bf16 [R][T][H], topk_idx i64 [R][T][K]
 *   packed_recv_x     bf16 [R][L][R*Tmax][H] out: slot p of expert (d, j) holds
 *                     the p-th token, in (source rank, token) order, that names
 *                     that expert (a token counts once per expert)
 *   packed_recv_count i32  [R][L] out
 *   src_info          i32  [R][L][R*Tmax] out: token index t of each slot
 *   layout_range      i32  [R][L][R][2] out: {first slot, slot count} of each
 *                     source rank
 * Slots at or past the count are left untouched. */
EP_API int ep_ll_dispatch(ep_ctx* ctx, const uint16_t* x, const int64_t* topk_idx,
                   uint16_t* packed_recv_x, int32_t* packed_recv_count,
                   int32_t* src_info, int32_t* layout_range,
                   ep_stream_t stream, ep_event_t wait_event);

/* Low-latency dispatch with FP8 packing ([API] "IB-GDA Kernels", "Low-Latency
 * Inference with FP8": use_fp8, the packed result becomes a pair).  Same
 * packing, counts, src_info and layout_range as ep_ll_dispatch; each packed row
 * is stored as OCP E4M3 codes with one fp32 scale per 128 hidden channels:
 *   scale = amax(|x| over the block) / 448 (fp32, nearest even),
 *   code  = E4M3(x * (448 / amax)) (fp32 quotient and product, each nearest
 *           even; E4M3 nearest even, saturating at +-448);
 * an all-zero block has scale 1 and zero codes; x ~= value(code) * scale.
 *   packed_recv_x_fp8   u8  [R][L][R*Tmax][H]      out (16-byte aligned)
 *   packed_recv_scales  f32 [R][L][R*Tmax][H/128]  out
 * Requires H % 128 == 0 (EP_ERR_INVALID_ARG otherwise) and x 32-byte aligned
 * (EP_ERR_ALIGNMENT otherwise: the copy reads x in 32-byte vectors). */
EP_API int ep_ll_dispatch_fp8(ep_ctx* ctx, const uint16_t* x, const int64_t* topk_idx,
                              uint8_t* packed_recv_x_fp8, float* packed_recv_scales,
                              int32_t* packed_recv_count, int32_t* src_info, int32_t* layout_range,
                              ep_stream_t stream, ep_event_t wait_event);

/* Low-latency combine ([API] "IB-GDA Kernels"): weighted reduction of expert
 * outputs back to token positions,
 *   out_x[s][t] = bf16( fp32 fused multiply-add chain, starting at 0, over the
 *                 token's valid slots in ascending (expert id, k):
 *                 acc = fma(topk_weights[s][t][k], y[d][j][slot], acc) )
 * where slot is the token's position in expert (d, j)'s packed list (located
 * through layout_range and src_info from ep_ll_dispatch of the same topk_idx).
 *   y bf16 [R][L][R*Tmax][H]; topk_weights f32 [R][T][K]; out_x bf16 [R][T][H]. */
EP_API int ep_ll_combine(ep_ctx* ctx, const uint16_t* y, const int64_t* topk_idx,
                  const float* topk_weights, const int32_t* src_info,
                  const int32_t* layout_range, uint16_t* out_x,
                  ep_stream_t stream, ep_event_t wait_event);

/* Load balance for redundant experts ("第 10 章 V2：EP 之外的 Buffer 与扩展能力",
 * section 10.2: replica weights are fetched before the expert compute and the
 * replicas' gradients are folded back into the original experts in the
 * backward pass, keyed by redundancy_mapping).  Every expert's weights (or
 * gradients) are one block of W bf16 values, W % 8 == 0 (EP_ERR_ALIGNMENT):
 *   redundancy_mapping  i32 [N]: original expert (in [0, E)) of replica i, -1 = unused
 *   ep_lb_prefetch_weights: redundant_weights[i] = expert_weights[mapping[i]]
 *     (expert_weights bf16 [E][W], redundant_weights bf16 [N][W]; rows of unused
 *     replicas are left untouched)
 *   ep_lb_reduce_grads: expert_grads[e] = bf16( expert_grads[e] + sum over
 *     replicas i of e, ascending i, of redundant_grads[i] ), fp32 accumulation
 *     in that order, one rounding; experts without replicas are untouched
 *     (expert_grads bf16 [E][W] in/out, redundant_grads bf16 [N][W])
 * E is the context's num_experts; N <= 65535, at most 1024 replicas per expert.
 * Mapping entries outside [-1, E) record EP_ERR_BAD_TOPK for ep_sync_status. */
EP_API int ep_lb_prefetch_weights(ep_ctx* ctx, const uint16_t* expert_weights, int64_t elems_per_expert,
                                  const int32_t* redundancy_mapping, int32_t num_redundant,
                                  uint16_t* redundant_weights, ep_stream_t stream, ep_event_t wait_event);
EP_API int ep_lb_reduce_grads(ep_ctx* ctx, const uint16_t* redundant_grads, int64_t elems_per_expert,
                              const int32_t* redundancy_mapping, int32_t num_redundant,
                              uint16_t* expert_grads, ep_stream_t stream, ep_event_t wait_event);

/* Size of the library's static device scratch array (512 KiB on every GPU that
 * loads the library, held until the process exits). */
#define EP_STATIC_SCRATCH_BYTES (512u * 1024u)

/* Dispatch-handle build that allocates nothing.  No counterpart on the pages:
 * this is a convenience of this library for callers that cannot call
 * cudaMalloc -- for example a process whose device memory is all reserved by a
 * framework's caching allocator or a fixed serving budget, or code that must
 * not risk the device-wide synchronisation cudaMalloc/cudaFree can cause.  It
 * needs no ep_ctx (ep_create allocates) and uses the library's static scratch
 * array instead of a workspace.
 *
 * Computes what ep_dispatch's handle step computes, from a layout:
 *   is_token_in_rank      u8  [R][T][R] input (4-byte aligned)
 *   num_tokens_per_expert i32 [R][E]    input
 *   handle                outputs: send_head, rank_prefix_matrix,
 *                         channel_prefix_matrix, recv_channel_prefix_matrix,
 *                         recv_rank_offset, num_recv_tokens_per_expert
 *                         (recv_src_idx and is_token_in_rank are not touched)
 *   error_word            device int32, zeroed by the caller; a device wait that
 *                         runs out stores EP_ERR_TIMEOUT there.  Required when
 *                         R * T > 0 (EP_ERR_INVALID_ARG if null): without it a
 *                         timeout could not be reported
 * Limits as for ep_config; in addition the scratch it needs,
 *   256 + round_up(8 * R * ceil(R*T / 256), 256) + 8 * R * R bytes,
 * must fit in EP_STATIC_SCRATCH_BYTES, or the call returns EP_ERR_CAPACITY
 * before launching anything (R = 32, T = 8192 needs 270,592 bytes = 264.25 KiB;
 * the channel count does not enter).
 * The first call on a device looks up the array's device address (once, with
 * that device current); make that first call before any stream capture.  The
 * address is kept for the life of the process: a cudaDeviceReset (or any reset
 * of the device's primary context) invalidates it, so do not call this entry
 * point again after one.
 * Every call shares the one array, and each call clears what must start at
 * zero: calls that may overlap on the GPU (other streams, other threads) race
 * and must be serialised by the caller. */
EP_API int ep_dispatch_handle_static(int32_t num_ranks, int32_t num_experts, int32_t num_tokens,
                                     int32_t num_channels, const uint8_t* is_token_in_rank,
                                     const int32_t* num_tokens_per_expert, const ep_handle* handle,
                                     int32_t* error_word, ep_stream_t stream);

/* Dynamic rank masking for the low-latency calls ([API] "Dynamic Rank
 * Masking": leave ranks, e.g. failed nodes, out of the exchange without
 * tearing it down; query reports 0 = active, 1 = masked; clean resets all).
 * A masked rank neither sends nor receives in ep_ll_dispatch[_fp8]: its tokens
 * are not packed and its experts receive nothing; in ep_ll_combine slots on a
 * masked rank contribute nothing and the masked rank's own tokens get +0.
 * Every rank starts active.  Updates and clean are stream-ordered (they apply
 * to low-latency calls issued after them on the stream); query synchronizes
 * the stream and writes R int32 values to host memory. */
EP_API int ep_ll_update_mask(ep_ctx* ctx, int32_t rank, int32_t masked, ep_stream_t stream);
EP_API int ep_ll_query_mask(ep_ctx* ctx, int32_t* host_out, ep_stream_t stream);
EP_API int ep_ll_clean_mask(ep_ctx* ctx, ep_stream_t stream);

/* ---------------------------------------------------------------------------
 * Sharded exchange: the R virtual ranks spread over W GPUs of one node, GPU w
 * hosting ranks [w*R/W, (w+1)*R/W) -- the pages' ranks are GPUs joined by
 * NVLink, with buffers allocated per rank and their IPC handles exchanged
 * ([API] "Construction and Resource Allocation"; [ARCH] intranode mode).
 * Each GPU keeps registered receive buffers (one cudaMalloc each, see
 * ep_shared_alloc) that every other GPU maps with ep_ipc_open.  Dispatch writes
 * every row straight into the receive buffer of the GPU hosting its
 * destination, and combine reads the expert outputs back from there: the
 * all-to-all happens inside the copy and the reduction, over NVLink.  The
 * receive order is the one-GPU order, so send_head and the rows of rank d
 * equal those ep_dispatch gives for the whole problem.
 *
 * Per step, on every GPU (shard w, Rl = R/W local ranks, local tokens G = Rl*T):
 *   1. ep_get_dispatch_layout on the shard's topk_idx [Rl][T][K] gives
 *      is_token_in_rank [Rl][T][R], num_tokens_per_rank [Rl][R],
 *      num_tokens_per_expert [Rl][E];
 *   2. the caller gathers the W layouts' counts in shard order into
 *      num_tokens_per_rank_all [R][R] and num_tokens_per_expert_all [R][E]
 *      (an all-gather of a few KB);
 *   3. ep_sharded_handle -> send_head [Rl][T][R] (P(g)[d] over all R*T tokens),
 *      dst_offset [R] (first row of rank d in its GPU's receive buffer),
 *      num_recv_rows (rows this GPU receives), num_recv_tokens_per_expert
 *      [Rl][L] for this GPU's experts;
 *   4. ep_sharded_dispatch writes the rows (and metadata) into the GPUs' buffers;
 *   5. a barrier across the GPUs (every dispatch finished) before the experts
 *      read their rows, and again (every expert output written) before
 *   6. ep_sharded_combine, which reduces, for each local token, the rows of its
 *      destination ranks in ascending rank order (fp32, one rounding), reading
 *      them from the GPUs hosting them.
 * Pointer tables (`num_shards` entries, indexed by shard) hold device pointers
 * valid in the calling process: its own buffer at its own index, the mapped
 * peers' elsewhere.  Every buffer of a table has at least `capacity` rows.
 * The kernels never wait on another GPU; the barriers are the caller's.
 * Rows from or to a row index >= capacity record EP_ERR_CAPACITY. */

/* Context for shard `shard` of `num_shards` (1 <= W <= 32, R % W == 0) on the
 * current device.  cfg describes the whole problem (R, E, T per rank, ...).
 * ep_get_dispatch_layout works on the shard's ranks; ep_dispatch,
 * ep_dispatch_cached, ep_combine and the low-latency calls are refused
 * (EP_ERR_INVALID_ARG) on a context of W > 1. */
EP_API int ep_create_sharded(const ep_config* cfg, int num_shards, int shard, ep_ctx** out);

/* Step 3 above.  num_tokens_per_rank_all i32 [R][R], num_tokens_per_expert_all
 * i32 [R][E] (inputs, gathered); send_head i32 [Rl][T][R], dst_offset i64 [R],
 * num_recv_rows i64 [1] (nullable), num_recv_tokens_per_expert i32 [Rl][L]
 * (nullable): outputs on this device. */
EP_API int ep_sharded_handle(ep_ctx* ctx, const uint8_t* is_token_in_rank, const int32_t* num_tokens_per_rank_all,
                             const int32_t* num_tokens_per_expert_all, int32_t* send_head, int64_t* dst_offset,
                             int64_t* num_recv_rows, int32_t* num_recv_tokens_per_expert,
                             ep_stream_t stream, ep_event_t wait_event);

/* Step 4.  x bf16 [Rl][T][H], topk_idx i64 [Rl][T][K], topk_weights f32
 * [Rl][T][K] (nullable unless recv_topk_weights is given).  Tables of
 * num_shards pointers: recv_x bf16 [capacity][H] (required), recv_topk_idx
 * i64 [capacity][K], recv_topk_weights f32 [capacity][K], recv_src_idx i32
 * [capacity] (each table nullable; written as by ep_dispatch, in the receive
 * buffer of the GPU hosting the destination). */
EP_API int ep_sharded_dispatch(ep_ctx* ctx, const uint16_t* x, const int64_t* topk_idx, const float* topk_weights,
                               const int32_t* send_head, const int64_t* dst_offset, int num_shards,
                               uint16_t* const* recv_x, int64_t* const* recv_topk_idx,
                               float* const* recv_topk_weights, int32_t* const* recv_src_idx,
                               int64_t capacity, ep_stream_t stream, ep_event_t wait_event);

/* Step 6.  Tables of num_shards pointers: y bf16 [capacity][H] (the expert
 * outputs, row for row as received; required), recv_topk_weights f32
 * [capacity][K] (required iff out_topk_weights is given).  bias0 / bias1 bf16
 * [Rl][T][H] nullable; out_x bf16 [Rl][T][H]; out_topk_weights f32 [Rl][T][K]
 * nullable.  Same arithmetic as ep_combine. */
EP_API int ep_sharded_combine(ep_ctx* ctx, int num_shards, const uint16_t* const* y,
                              const float* const* recv_topk_weights, int64_t capacity, const int32_t* send_head,
                              const int64_t* dst_offset, const uint16_t* bias0, const uint16_t* bias1,
                              uint16_t* out_x, float* out_topk_weights, ep_stream_t stream, ep_event_t wait_event);

/* Registered buffers: ep_shared_alloc makes one device allocation of `bytes`
 * on the current device and writes its CUDA IPC handle (EP_IPC_HANDLE_BYTES
 * bytes) to ipc_handle; release it with ep_shared_free.  Another process maps
 * it with ep_ipc_open (peer access enabled on demand) and unmaps it with
 * ep_ipc_close.  A process cannot open its own handles. */
#define EP_IPC_HANDLE_BYTES 64
EP_API int ep_shared_alloc(size_t bytes, void** ptr, uint8_t* ipc_handle);
EP_API int ep_shared_free(void* ptr);
EP_API int ep_ipc_open(const uint8_t* ipc_handle, void** ptr);
EP_API int ep_ipc_close(void* ptr);

/* Optional per-kernel timing (CUDA events around each launch on the call's
 * stream; inside a stream capture they become event-record nodes, recorded
 * each time the graph runs).  ep_profile_read synchronizes the recorded events and returns,
 * per kernel kind, the number of launches and total milliseconds since the
 * last read; kinds: 0 layout, 1 scan (handle), 2 dispatch, 3 cached dispatch,
 * 4 combine, 5 ll slots, 6 ll copy, 7 ll combine, 8 ll copy (FP8),
 * 9 lb prefetch, 10 lb reduce. */
#define EP_PROFILE_KINDS 11
EP_API int ep_profile_enable(ep_ctx* ctx, int enable);
EP_API int ep_profile_read(ep_ctx* ctx, int64_t* launches, double* total_ms);

#ifdef __cplusplus
}
#endif

#endif /* EP_B200_H */
