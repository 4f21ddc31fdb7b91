// ep_dispatch_handle_static: the dispatch-handle build (the decoupled-lookback
// scan) for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: a process whose device memory is all
// reserved up front by a framework's caching allocator or a serving runtime's
// fixed budget, or code that must not risk the device-wide synchronisation that
// cudaMalloc/cudaFree can cause.  ep_create allocates a workspace, so those
// callers cannot use the context-based calls.  This entry point needs no
// context: the scan's scratch (tile status words, the tile ticket and the
// rank-start words) lives in the file-scope array below, which
// every GPU that loads the library holds until the process exits.  The caller
// still passes all inputs and outputs.
//
// In host code `g_static_scratch` names a host-side stand-in, not device
// memory; its device address is looked up once per device with
// cudaGetSymbolAddress (on the first call on that device, with that device
// current) and passed to the kernel.  The looked-up address is kept for the
// life of the process; a reset of the device's primary context (for example
// cudaDeviceReset) reloads the module and invalidates it, which the header
// states as a limit of this entry point.

#include <cstdint>
#include <mutex>

#include "../../include/ep.h"
#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char g_static_scratch[EP_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
constexpr size_t kCounterBytes = 256;   // the tile ticket, padded

std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set-up on first use).
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

extern "C" EP_API int ep_dispatch_handle_static(int32_t num_ranks, int32_t num_experts,
                                                int32_t num_tokens, int32_t num_channels,
                                                const uint8_t* is_token_in_rank,
                                                const int32_t* num_tokens_per_expert,
                                                const ep_handle* handle, int32_t* error_word,
                                                ep_stream_t stream) {
    const int R = num_ranks, E = num_experts, T = num_tokens, C = num_channels;
    if (R < 1 || R > 32 || E < R || E > 4096 || E % R != 0 || T < 0 || C < 1 || C > 1024)
        return EP_ERR_INVALID_ARG;
    const long long G = (long long)R * T;
    if (G * R >= (1LL << 31)) return EP_ERR_INVALID_ARG;
    if (handle == nullptr || handle->rank_prefix_matrix == nullptr ||
        handle->channel_prefix_matrix == nullptr || handle->recv_channel_prefix_matrix == nullptr ||
        handle->recv_rank_offset == nullptr || handle->num_recv_tokens_per_expert == nullptr ||
        num_tokens_per_expert == nullptr)
        return EP_ERR_INVALID_ARG;
    if (G > 0 && (is_token_in_rank == nullptr || handle->send_head == nullptr || error_word == nullptr))
        return EP_ERR_INVALID_ARG;   // (a timeout of the scan's waits is reported through error_word)
    if ((reinterpret_cast<uintptr_t>(is_token_in_rank) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(handle->recv_rank_offset) & 7u) != 0)
        return EP_ERR_ALIGNMENT;

    const int tiles = (int)((G + ep::kScanTile - 1) / ep::kScanTile);
    const size_t status_bytes = (size_t)tiles * R * sizeof(unsigned long long);
    const size_t rank_start_bytes = (size_t)R * R * sizeof(unsigned long long);
    if (kCounterBytes + round256(status_bytes) + rank_start_bytes > EP_STATIC_SCRATCH_BYTES)
        return EP_ERR_CAPACITY;   // the problem needs more scratch than the static array holds

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (G == 0) {
        const size_t mat = sizeof(int) * (size_t)R * R * C;
        cudaError_t e = cudaMemsetAsync(handle->rank_prefix_matrix, 0, sizeof(int) * R * R, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(handle->channel_prefix_matrix, 0, mat, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(handle->recv_channel_prefix_matrix, 0, mat, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(handle->recv_rank_offset, 0, sizeof(int64_t) * (R + 1), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(handle->num_recv_tokens_per_expert, 0, sizeof(int) * (size_t)E, s);
        return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
    }

    void* base = nullptr;
    if (scratch_address(&base) != cudaSuccess) return EP_ERR_CUDA;
    unsigned char* scratch = static_cast<unsigned char*>(base);
    // The array keeps the previous call's contents, possibly from a call of
    // another shape: the ticket, status and rank-start words start at zero on
    // every call (the ticket restarts at call 0; zeroed words never match its tag).
    if (cudaMemsetAsync(scratch, 0, kCounterBytes + round256(status_bytes) + rank_start_bytes, s) != cudaSuccess)
        return EP_ERR_CUDA;

    ep::ScanParams p{};
    p.is_token_in_rank = is_token_in_rank;
    p.num_tokens_per_expert = num_tokens_per_expert;
    p.ticket = reinterpret_cast<unsigned long long*>(scratch);
    p.status = reinterpret_cast<unsigned long long*>(scratch + kCounterBytes);
    p.rank_start = reinterpret_cast<unsigned long long*>(scratch + kCounterBytes + round256(status_bytes));
    p.send_head = handle->send_head;
    p.rank_prefix_matrix = handle->rank_prefix_matrix;
    p.channel_prefix_matrix = handle->channel_prefix_matrix;
    p.recv_channel_prefix_matrix = handle->recv_channel_prefix_matrix;
    p.recv_rank_offset = reinterpret_cast<long long*>(handle->recv_rank_offset);
    p.num_recv_tokens_per_expert = handle->num_recv_tokens_per_expert;
    p.err = error_word;
    p.G = G;
    p.R = R;
    p.E = E;
    p.L = E / R;
    p.T = T;
    p.C = C;
    p.q = (T + C - 1) / C;
    p.num_tiles = tiles;
    return ep::launch_scan(p, s) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}
