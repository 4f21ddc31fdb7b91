// C ABI of libep.so: argument validation, the context's fixed workspace, and
// the order of kernel launches for each entry point.  See include/ep.h for the
// contract of every call.
//
// Entry point -> kernels (all on the caller's stream):
//   ep_get_dispatch_layout : layout_kernel (one CTA cluster per source; a memset only when T = 0)
//   ep_dispatch            : [layout_kernel] + scan_kernel (call-tagged scan state, nothing to clear)
//                            [+ one host read of N] + dispatch_kernel<normal> (programmatic
//                            launch behind the scan)
//   ep_get_num_recv        : one device-to-host copy of the [R][R] counts + a stream sync
//   ep_dispatch_cached     : dispatch_kernel<cached>
//   ep_combine             : combine_kernel
//   ep_ll_dispatch[_fp8]   : T <= 256: ll_rank_kernel (per-source counts and each token's
//                            rank within its source) + dispatch_kernel<packed> /
//                            ll_fp8_copy_kernel (programmatic launch behind it; they add
//                            the earlier sources' counts and write src_info, layout_range,
//                            the counts); larger T: ll_slot_kernel (call-tagged scan state,
//                            nothing to clear) + the same copy kernels reading its slot map
//   ep_ll_combine          : ll_combine_kernel
//   ep_lb_prefetch_weights : lb_prefetch_kernel;  ep_lb_reduce_grads : lb_reduce_kernel
//   ep_sharded_handle      : shard_offsets_kernel + scan_kernel (with the shard's base)
//   ep_sharded_dispatch    : dispatch_kernel<sharded>;  ep_sharded_combine : combine_kernel<sharded>
//   ep_check_handle        : handle_check_kernel
//   ep_ll_update_mask / ep_ll_clean_mask : set_mask_kernel / memset

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <vector>

#include "../../include/ep.h"
#include "check.h"
#include "kernels.h"

struct ep_prof_rec {
    int kind;
    cudaEvent_t start, stop;
};

struct ep_ctx {
    ep_config cfg;
    int R, E, L, T, H, K, C, Tmax;
    long long G;                // tokens of this context's source ranks: Rl * T
    int num_shards, shard;      // sharded exchange: this GPU hosts ranks [r0, r0 + Rl)
    int Rl, r0;                 // (one shard: Rl = R, r0 = 0)
    int64_t ll_cap;
    int device;
    int num_sms;
    // device workspace (one allocation)
    char* ws;
    size_t ws_bytes;
    int* err;
    unsigned long long* scan_status;   // [scan_tiles][R] call-tagged tile status (never cleared)
    unsigned long long* scan_ticket;   // block ticket (only incremented)
    int scan_tiles;
    unsigned long long* rank_start;    // [R][R] call-tagged P(s*T)[d] of the handle scan
    int* ntr_ws;                // [R][R]   (layout computed inside ep_dispatch)
    int* nte_ws;                // [R][E]
    int* slot_map;              // [G][K]   (low-latency slots)
    unsigned long long* ll_status;  // [ll_tiles][E] call-tagged tile status of the LL slot scan
    unsigned long long* ll_src_begin;  // [R][E] call-tagged first slot per source
    unsigned long long* ll_ticket;  // LL slot scan block ticket (only ever incremented)
    int ll_tiles_per_src;
    int ll_tiles;
    int* ll_cnt;                // [R][E] direct low-latency slots: tokens of source s naming e
    int* ll_within;             // [G][K] direct low-latency slots: rank of a token among its source's
    int* rank_mask;             // [R] low-latency rank mask (0 active, 1 masked)
    int* shard_base;            // [R] tokens of earlier shards per destination (sharded scan base)
    char last_error[256];
    bool prof;
    std::vector<ep_prof_rec> pending;
    int64_t prof_launches[EP_PROFILE_KINDS];
    double prof_ms[EP_PROFILE_KINDS];
};

namespace {

std::atomic<uint64_t> g_launches{0};

enum Kind { kLayout = 0, kScan = 1, kDispatch = 2, kCached = 3, kCombine = 4,
            kLLCount = 5, kLLCopy = 6, kLLCombine = 7, kLLCopyFp8 = 8, kLBPrefetch = 9, kLBReduce = 10 };

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

int fail(ep_ctx* c, int code, const char* fmt, ...) __attribute__((format(printf, 3, 4)));
int fail(ep_ctx* c, int code, const char* fmt, ...) {
    if (c != nullptr) {
        va_list ap;
        va_start(ap, fmt);
        vsnprintf(c->last_error, sizeof c->last_error, fmt, ap);
        va_end(ap);
    }
    return code;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int validate_config(const ep_config* c) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (c->num_ranks < 1 || c->num_ranks > 32) return EP_ERR_INVALID_ARG;
    if (c->num_experts < c->num_ranks || c->num_experts > 4096 || c->num_experts % c->num_ranks != 0)
        return EP_ERR_INVALID_ARG;
    if (c->num_tokens < 0) return EP_ERR_INVALID_ARG;
    if (c->topk < 1 || c->topk > 32) return EP_ERR_INVALID_ARG;
    if (c->hidden < 8 || c->hidden > 32768) return EP_ERR_INVALID_ARG;
    if (c->hidden % 8 != 0) return EP_ERR_ALIGNMENT;   // rows must be whole 16-byte vectors
    if (c->num_channels < 1 || c->num_channels > 1024) return EP_ERR_INVALID_ARG;
    if (c->ll_max_tokens_per_rank < 0) return EP_ERR_INVALID_ARG;
    if (c->ll_max_tokens_per_rank != 0 && c->ll_max_tokens_per_rank < c->num_tokens)
        return EP_ERR_INVALID_ARG;
    const long long G = (long long)c->num_ranks * c->num_tokens;
    const long long fan = c->num_ranks > c->topk ? c->num_ranks : c->topk;
    if (G * fan >= (1LL << 31)) return EP_ERR_INVALID_ARG;
    const long long tmax = c->ll_max_tokens_per_rank ? c->ll_max_tokens_per_rank : c->num_tokens;
    if ((long long)c->num_ranks * tmax >= (1LL << 31)) return EP_ERR_INVALID_ARG;
    return EP_OK;
}

// Keep the context's device current for the duration of a call.
struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
    }
    ~DeviceGuard() {
        int cur;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

// Record a profiling event; inside a stream capture it becomes an event-record
// node of the graph (so it is recorded each time the graph runs).
cudaError_t record_event(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &st) == cudaSuccess && st == cudaStreamCaptureStatusActive)
        return cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
    return cudaEventRecord(ev, s);
}

template <class F>
int launch(ep_ctx* c, int kind, bool has_work, cudaStream_t s, F&& f) {
    if (!has_work) return EP_OK;
    cudaEvent_t a = nullptr, b = nullptr;
    if (c->prof && kind >= 0) {
        if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess)
            return fail(c, EP_ERR_CUDA, "cudaEventCreate failed");
        record_event(a, s);
    }
    const cudaError_t e = f();
    if (e != cudaSuccess) {
        if (a) cudaEventDestroy(a);
        if (b) cudaEventDestroy(b);
        return fail(c, EP_ERR_CUDA, "kernel launch failed: %s", cudaGetErrorString(e));
    }
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (c->prof && kind >= 0) {
        record_event(b, s);
        c->pending.push_back({kind, a, b});
    }
    return EP_OK;
}

int cuda_check(ep_ctx* c, cudaError_t e, const char* what) {
    if (e == cudaSuccess) return EP_OK;
    return fail(c, EP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

int begin_call(ep_ctx* c, cudaStream_t s, cudaEvent_t wait_event) {
    c->last_error[0] = '\0';
    if (wait_event != nullptr) return cuda_check(c, cudaStreamWaitEvent(s, wait_event, 0), "cudaStreamWaitEvent");
    return EP_OK;
}

int check_handle(ep_ctx* c, const ep_handle* h) {
    // per-token arrays are empty (and may be null) when there are no tokens
    const bool tokens = c->G > 0;
    if (h == nullptr || h->rank_prefix_matrix == nullptr || h->channel_prefix_matrix == nullptr ||
        h->recv_channel_prefix_matrix == nullptr || (tokens && h->is_token_in_rank == nullptr) ||
        (tokens && h->send_head == nullptr) || h->recv_rank_offset == nullptr ||
        h->num_recv_tokens_per_expert == nullptr)
        return fail(c, EP_ERR_HANDLE_MISMATCH, "handle array missing");
    if (!aligned(h->recv_rank_offset, 8) || !aligned(h->send_head, 4) || !aligned(h->is_token_in_rank, 4))
        return fail(c, EP_ERR_ALIGNMENT, "handle array misaligned");
    return EP_OK;
}

}  // namespace

extern "C" {

const char* ep_status_string(int status) {
    switch (status) {
        case EP_OK: return "EP_OK";
        case EP_ERR_INVALID_ARG: return "EP_ERR_INVALID_ARG";
        case EP_ERR_ALIGNMENT: return "EP_ERR_ALIGNMENT";
        case EP_ERR_CAPACITY: return "EP_ERR_CAPACITY";
        case EP_ERR_BAD_TOPK: return "EP_ERR_BAD_TOPK";
        case EP_ERR_HANDLE_MISMATCH: return "EP_ERR_HANDLE_MISMATCH";
        case EP_ERR_TIMEOUT: return "EP_ERR_TIMEOUT";
        case EP_ERR_CUDA: return "EP_ERR_CUDA";
        case EP_ERR_UNIMPLEMENTED: return "EP_ERR_UNIMPLEMENTED";
        default: return "EP_ERR_UNKNOWN";
    }
}

uint64_t ep_kernel_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

}  // extern "C"

namespace {

int create_impl(const ep_config* cfg, int num_shards, int shard, ep_ctx** out) {
    if (out == nullptr) return EP_ERR_INVALID_ARG;
    *out = nullptr;
    const int v = validate_config(cfg);
    if (v != EP_OK) return v;
    if (num_shards < 1 || num_shards > ep::kMaxShards || cfg->num_ranks % num_shards != 0 || shard < 0 ||
        shard >= num_shards)
        return EP_ERR_INVALID_ARG;

    ep_ctx* c = new ep_ctx();
    c->cfg = *cfg;
    c->R = cfg->num_ranks;
    c->E = cfg->num_experts;
    c->L = c->E / c->R;
    c->T = cfg->num_tokens;
    c->H = cfg->hidden;
    c->K = cfg->topk;
    c->C = cfg->num_channels;
    c->Tmax = cfg->ll_max_tokens_per_rank ? cfg->ll_max_tokens_per_rank : cfg->num_tokens;
    c->num_shards = num_shards;
    c->shard = shard;
    c->Rl = c->R / num_shards;
    c->r0 = shard * c->Rl;
    c->G = (long long)c->Rl * c->T;
    c->ll_cap = (int64_t)c->R * c->Tmax;

    int rc = EP_OK;
    cudaDeviceProp prop;
    if (cudaGetDevice(&c->device) != cudaSuccess || cudaGetDeviceProperties(&prop, c->device) != cudaSuccess) {
        delete c;
        return EP_ERR_CUDA;
    }
    if (prop.major != 10 || prop.minor != 0) {   // built for sm_100a only
        delete c;
        return EP_ERR_CUDA;
    }
    c->num_sms = prop.multiProcessorCount;
    c->scan_tiles = (int)((c->G + ep::kScanTile - 1) / ep::kScanTile);

    // workspace layout
    size_t off = 0;
    const size_t off_err = off;            off += align256(sizeof(int));
    const size_t off_scan = off;
    const size_t status_bytes = (size_t)c->scan_tiles * c->R * sizeof(unsigned long long);
    off += align256(status_bytes + sizeof(unsigned long long));
    const size_t off_rs = off;             off += align256((size_t)c->R * c->R * sizeof(unsigned long long));
    const size_t off_ntr = off;            off += align256((size_t)c->R * c->R * sizeof(int));
    const size_t off_nte = off;            off += align256((size_t)c->R * c->E * sizeof(int));
    const size_t off_slot = off;           off += align256((size_t)c->G * c->K * sizeof(int));
    c->ll_tiles_per_src = (c->T + ep::kLLTile - 1) / ep::kLLTile;
    c->ll_tiles = c->R * c->ll_tiles_per_src;
    const size_t off_lls = off;            off += align256((size_t)c->ll_tiles * c->E * sizeof(unsigned long long));
    const size_t off_llb = off;            off += align256((size_t)c->R * c->E * sizeof(unsigned long long));
    const size_t off_llc = off;            off += align256(sizeof(unsigned long long));
    const size_t off_llh = off;            off += align256((size_t)c->R * c->E * sizeof(int));
    const size_t off_llwithin = off;       off += align256((size_t)c->G * c->K * sizeof(int));
    const size_t off_mask = off;           off += align256((size_t)c->R * sizeof(int));
    const size_t off_sbase = off;          off += align256((size_t)c->R * sizeof(int));
    c->ws_bytes = off;
    if (cudaMalloc(&c->ws, c->ws_bytes) != cudaSuccess) {
        delete c;
        return EP_ERR_CUDA;
    }
    c->err = reinterpret_cast<int*>(c->ws + off_err);
    c->scan_status = reinterpret_cast<unsigned long long*>(c->ws + off_scan);
    c->scan_ticket = reinterpret_cast<unsigned long long*>(c->ws + off_scan + status_bytes);
    c->rank_start = reinterpret_cast<unsigned long long*>(c->ws + off_rs);
    c->ntr_ws = reinterpret_cast<int*>(c->ws + off_ntr);
    c->nte_ws = reinterpret_cast<int*>(c->ws + off_nte);
    c->slot_map = reinterpret_cast<int*>(c->ws + off_slot);
    c->ll_status = reinterpret_cast<unsigned long long*>(c->ws + off_lls);
    c->ll_src_begin = reinterpret_cast<unsigned long long*>(c->ws + off_llb);
    c->ll_ticket = reinterpret_cast<unsigned long long*>(c->ws + off_llc);
    c->ll_cnt = reinterpret_cast<int*>(c->ws + off_llh);
    c->ll_within = reinterpret_cast<int*>(c->ws + off_llwithin);
    c->rank_mask = reinterpret_cast<int*>(c->ws + off_mask);   // zeroed below: every rank active
    c->shard_base = reinterpret_cast<int*>(c->ws + off_sbase);
    if (cudaMemset(c->ws, 0, c->ws_bytes) != cudaSuccess) rc = EP_ERR_CUDA;
    if (rc == EP_OK && ep::ll_prepare(c->E) != cudaSuccess) rc = EP_ERR_CUDA;
    if (rc != EP_OK) {
        cudaFree(c->ws);
        delete c;
        return rc;
    }
    *out = c;
    return EP_OK;
}

}  // namespace

extern "C" {

int ep_create(const ep_config* cfg, ep_ctx** out) { return create_impl(cfg, 1, 0, out); }

int ep_create_sharded(const ep_config* cfg, int num_shards, int shard, ep_ctx** out) {
    return create_impl(cfg, num_shards, shard, out);
}

int ep_destroy(ep_ctx* c) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    DeviceGuard guard(c->device);
    for (auto& r : c->pending) {
        cudaEventDestroy(r.start);
        cudaEventDestroy(r.stop);
    }
    const cudaError_t e = cudaFree(c->ws);
    delete c;
    return e == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

int ep_workspace_bytes(const ep_ctx* c, size_t* bytes) {
    if (c == nullptr || bytes == nullptr) return EP_ERR_INVALID_ARG;
    *bytes = c->ws_bytes;
    return EP_OK;
}

int ep_handle_layout(const ep_ctx* c, ep_handle_sizes* s) {
    if (c == nullptr || s == nullptr) return EP_ERR_INVALID_ARG;
    const int64_t R = c->R, C = c->C, L = c->L, H = c->H;
    const int64_t fan = c->R < c->K ? c->R : c->K;
    s->rank_prefix_matrix = R * R;
    s->channel_prefix_matrix = R * R * C;
    s->recv_channel_prefix_matrix = R * R * C;
    s->recv_src_idx_max = c->G * fan;
    s->is_token_in_rank = c->G * R;
    s->send_head = c->G * R;
    s->recv_rank_offset = R + 1;
    s->num_recv_tokens_per_expert = R * L;
    s->ll_packed_recv_x = R * L * c->ll_cap * H;
    s->ll_packed_recv_count = R * L;
    s->ll_src_info = R * L * c->ll_cap;
    s->ll_layout_range = R * L * R * 2;
    return EP_OK;
}

const char* ep_last_error(const ep_ctx* c) { return c == nullptr ? "null context" : c->last_error; }

namespace {

int realign_tickets(ep_ctx* c) {
    struct { unsigned long long* ticket; long long tiles; } t[2] = {
        {c->scan_ticket, c->scan_tiles}, {c->ll_ticket, c->ll_tiles}};
    for (auto& x : t) {
        if (x.tiles <= 0) continue;
        unsigned long long v = 0;
        int rc = cuda_check(c, cudaMemcpy(&v, x.ticket, sizeof v, cudaMemcpyDeviceToHost), "read ticket");
        if (rc != EP_OK) return rc;
        const unsigned long long n = (unsigned long long)x.tiles;
        v = (v + n - 1) / n * n;
        rc = cuda_check(c, cudaMemcpy(x.ticket, &v, sizeof v, cudaMemcpyHostToDevice), "write ticket");
        if (rc != EP_OK) return rc;
    }
    return EP_OK;
}

}  // namespace

int ep_test_offset_tickets(ep_ctx* c, int64_t delta) {
    if (c == nullptr || delta < 0) return EP_ERR_INVALID_ARG;
    DeviceGuard guard(c->device);
    int rc = cuda_check(c, cudaDeviceSynchronize(), "cudaDeviceSynchronize");
    for (unsigned long long* tk : {c->scan_ticket, c->ll_ticket}) {
        if (rc != EP_OK) return rc;
        unsigned long long v = 0;
        rc = cuda_check(c, cudaMemcpy(&v, tk, sizeof v, cudaMemcpyDeviceToHost), "read ticket");
        if (rc != EP_OK) return rc;
        v += (unsigned long long)delta;
        rc = cuda_check(c, cudaMemcpy(tk, &v, sizeof v, cudaMemcpyHostToDevice), "write ticket");
    }
    return rc;
}

int ep_sync_status(ep_ctx* c, ep_stream_t stream) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int rc = cuda_check(c, cudaStreamSynchronize(s), "cudaStreamSynchronize");
    if (rc != EP_OK) return rc;
    int code = 0;
    rc = cuda_check(c, cudaMemcpy(&code, c->err, sizeof(int), cudaMemcpyDeviceToHost), "read error word");
    if (rc != EP_OK) return rc;
    if (code != 0) {
        rc = cuda_check(c, cudaMemset(c->err, 0, sizeof(int)), "clear error word");
        // a scan that gave up leaves its ticket possibly off a multiple of its tile
        // count: move each ticket up to the next multiple (a new call number that
        // no status word carries yet), so the next calls start consistent
        if (rc == EP_OK && code == EP_ERR_TIMEOUT) rc = realign_tickets(c);
        if (rc != EP_OK) return rc;
        return fail(c, code, "device reported %s", ep_status_string(code));
    }
    return EP_OK;
}

int ep_get_dispatch_layout(ep_ctx* c, const int64_t* topk_idx, int32_t* num_tokens_per_rank,
                           int32_t* num_tokens_per_expert, uint8_t* is_token_in_rank,
                           ep_stream_t stream, ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (c->G > 0 && (topk_idx == nullptr || is_token_in_rank == nullptr))
        return fail(c, EP_ERR_INVALID_ARG, "topk_idx / is_token_in_rank missing");
    if (num_tokens_per_rank == nullptr || num_tokens_per_expert == nullptr)
        return fail(c, EP_ERR_INVALID_ARG, "histogram outputs missing");
    if (!aligned(topk_idx, 8) || !aligned(is_token_in_rank, 4))
        return fail(c, EP_ERR_ALIGNMENT, "layout arrays misaligned");
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;
    if (c->G == 0) {   // no tokens: zero counts, nothing to launch (the kernel writes every count otherwise)
        rc = cuda_check(c, cudaMemsetAsync(num_tokens_per_rank, 0, sizeof(int) * c->Rl * c->R, s), "memset");
        if (rc == EP_OK)
            rc = cuda_check(c, cudaMemsetAsync(num_tokens_per_expert, 0, sizeof(int) * (size_t)c->Rl * c->E, s),
                            "memset");
        return rc;
    }
    ep::LayoutParams p{topk_idx, is_token_in_rank, num_tokens_per_rank, num_tokens_per_expert, c->err,
                       c->R, c->E, c->L, c->T, c->K, c->Rl};
    return launch(c, kLayout, c->G > 0, s, [&] { return ep::launch_layout(p, s); });
}

int ep_dispatch(ep_ctx* c, const uint16_t* x, const int64_t* topk_idx, const float* topk_weights,
                const int32_t* num_tokens_per_rank, const int32_t* num_tokens_per_expert,
                const uint8_t* is_token_in_rank, const ep_handle* h, uint16_t* recv_x,
                int64_t* recv_topk_idx, float* recv_topk_weights, int64_t recv_capacity_rows,
                int64_t* num_recv_host, ep_stream_t stream, ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (c->num_shards > 1) return fail(c, EP_ERR_INVALID_ARG, "sharded context: use the ep_sharded_* calls");
    int rc = check_handle(c, h);
    if (rc != EP_OK) return rc;
    if (recv_capacity_rows < 0) return fail(c, EP_ERR_INVALID_ARG, "negative capacity");
    if (c->G > 0 && (x == nullptr || topk_idx == nullptr)) return fail(c, EP_ERR_INVALID_ARG, "x / topk_idx missing");
    if (recv_capacity_rows > 0 && h->recv_src_idx == nullptr)
        return fail(c, EP_ERR_HANDLE_MISMATCH, "handle recv_src_idx missing");
    // (with no tokens, is_token_in_rank is empty and may be null)
    const int given = (num_tokens_per_rank != nullptr) + (num_tokens_per_expert != nullptr) +
                      (is_token_in_rank != nullptr || (c->G == 0 && num_tokens_per_rank != nullptr));
    if (given != 0 && given != 3) return fail(c, EP_ERR_INVALID_ARG, "pass all three layout arrays or none");
    if (!aligned16(x) || !aligned16(recv_x)) return fail(c, EP_ERR_ALIGNMENT, "row buffers must be 16-byte aligned");
    if (!aligned(topk_idx, 8) || !aligned(recv_topk_idx, 8) || !aligned(topk_weights, 4) ||
        !aligned(recv_topk_weights, 4) || !aligned(is_token_in_rank, 4))
        return fail(c, EP_ERR_ALIGNMENT, "top-k arrays misaligned");
    if (recv_topk_weights != nullptr && topk_weights == nullptr)
        return fail(c, EP_ERR_INVALID_ARG, "recv_topk_weights needs topk_weights");

    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;

    if (c->G == 0) {
        // no tokens: every matrix is zero
        const size_t rc2 = sizeof(int) * (size_t)c->R * c->R * c->C;
        cudaError_t e = cudaMemsetAsync(h->rank_prefix_matrix, 0, sizeof(int) * c->R * c->R, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(h->channel_prefix_matrix, 0, rc2, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(h->recv_channel_prefix_matrix, 0, rc2, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(h->recv_rank_offset, 0, sizeof(int64_t) * (c->R + 1), s);
        if (e == cudaSuccess) e = cudaMemsetAsync(h->num_recv_tokens_per_expert, 0, sizeof(int) * (size_t)c->E, s);
        rc = cuda_check(c, e, "zero handle");
        if (rc != EP_OK) return rc;
        if (num_recv_host != nullptr) *num_recv_host = 0;
        return EP_OK;
    }
    // 1. layout
    const int* nte = num_tokens_per_expert;
    if (given == 0) {
        ep::LayoutParams lp{topk_idx, h->is_token_in_rank, c->ntr_ws, c->nte_ws, c->err, c->R, c->E, c->L, c->T, c->K,
                            c->R};
        rc = launch(c, kLayout, c->G > 0, s, [&] { return ep::launch_layout(lp, s); });
        if (rc != EP_OK) return rc;
        nte = c->nte_ws;
    } else if (is_token_in_rank != h->is_token_in_rank && c->G > 0) {
        rc = cuda_check(c, cudaMemcpyAsync(h->is_token_in_rank, is_token_in_rank, (size_t)c->G * c->R,
                                           cudaMemcpyDeviceToDevice, s), "copy is_token_in_rank");
        if (rc != EP_OK) return rc;
    }

    // 2. handle (prefix scan)
    ep::ScanParams sp{};
    sp.is_token_in_rank = h->is_token_in_rank;
    sp.num_tokens_per_expert = nte;
    sp.status = c->scan_status;
    sp.ticket = c->scan_ticket;
    sp.rank_start = c->rank_start;
    sp.send_head = h->send_head;
    sp.rank_prefix_matrix = h->rank_prefix_matrix;
    sp.channel_prefix_matrix = h->channel_prefix_matrix;
    sp.recv_channel_prefix_matrix = h->recv_channel_prefix_matrix;
    sp.recv_rank_offset = reinterpret_cast<long long*>(h->recv_rank_offset);
    sp.num_recv_tokens_per_expert = h->num_recv_tokens_per_expert;
    sp.err = c->err;
    sp.G = c->G;
    sp.R = c->R; sp.E = c->E; sp.L = c->L; sp.T = c->T; sp.C = c->C;
    sp.q = (c->T + c->C - 1) / c->C;
    sp.num_tiles = c->scan_tiles;
    rc = launch(c, kScan, true, s, [&] { return ep::launch_scan(sp, s); });
    if (rc != EP_OK) return rc;

    // 3. optional host read of the receive count
    if (num_recv_host != nullptr) {
        int64_t n = 0;
        rc = cuda_check(c, cudaMemcpyAsync(&n, h->recv_rank_offset + c->R, sizeof n, cudaMemcpyDeviceToHost, s), "read N");
        if (rc == EP_OK) rc = cuda_check(c, cudaStreamSynchronize(s), "cudaStreamSynchronize");
        if (rc != EP_OK) return rc;
        *num_recv_host = n;
        if (n > recv_capacity_rows)
            return fail(c, EP_ERR_CAPACITY, "%lld receive rows, capacity %lld", (long long)n,
                        (long long)recv_capacity_rows);
    }

    // 4. rows + metadata
    ep::DispatchParams dp{};
    dp.x = x;
    dp.send_head = h->send_head;
    dp.recv_rank_offset = reinterpret_cast<const long long*>(h->recv_rank_offset);
    dp.recv_capacity = recv_capacity_rows;
    dp.topk_idx = topk_idx;
    dp.topk_weights = topk_weights;
    dp.recv_topk_idx = recv_topk_idx;
    dp.recv_topk_weights = recv_topk_weights;
    dp.recv_src_idx = h->recv_src_idx;
    dp.recv_x = recv_x;
    dp.err = c->err;
    dp.G = c->G;
    dp.R = c->R; dp.E = c->E; dp.L = c->L; dp.T = c->T; dp.K = c->K; dp.H = c->H;
    dp.splits = ep::dispatch_splits(c->H);
    return launch(c, kDispatch, true, s,
                  [&] { return ep::launch_dispatch(ep::kModeNormal, dp, s, num_recv_host == nullptr); });
}

int ep_get_num_recv(ep_ctx* c, const int32_t* num_tokens_per_rank, int64_t* num_recv_host,
                    int64_t* num_recv_per_rank_host, ep_stream_t stream, ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (c->num_shards > 1) return fail(c, EP_ERR_INVALID_ARG, "sharded context: ep_sharded_handle gives the count");
    if (num_tokens_per_rank == nullptr || num_recv_host == nullptr)
        return fail(c, EP_ERR_INVALID_ARG, "num_tokens_per_rank / num_recv_host missing");
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;
    std::vector<int32_t> ntr((size_t)c->R * c->R);
    rc = cuda_check(c, cudaMemcpyAsync(ntr.data(), num_tokens_per_rank, sizeof(int32_t) * ntr.size(),
                                       cudaMemcpyDeviceToHost, s), "read num_tokens_per_rank");
    if (rc == EP_OK) rc = cuda_check(c, cudaStreamSynchronize(s), "cudaStreamSynchronize");
    if (rc != EP_OK) return rc;
    int64_t total = 0;
    for (int d = 0; d < c->R; ++d) {
        int64_t nd = 0;
        for (int src = 0; src < c->R; ++src) nd += ntr[(size_t)src * c->R + d];
        if (num_recv_per_rank_host != nullptr) num_recv_per_rank_host[d] = nd;
        total += nd;
    }
    *num_recv_host = total;
    return EP_OK;
}

int ep_dispatch_cached(ep_ctx* c, const uint16_t* x, const ep_handle* h, uint16_t* recv_x,
                       int64_t recv_capacity_rows, ep_stream_t stream, ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (c->num_shards > 1) return fail(c, EP_ERR_INVALID_ARG, "sharded context: use the ep_sharded_* calls");
    int rc = check_handle(c, h);
    if (rc != EP_OK) return rc;
    if (recv_capacity_rows < 0) return fail(c, EP_ERR_INVALID_ARG, "negative capacity");
    if (c->G > 0 && x == nullptr) return fail(c, EP_ERR_INVALID_ARG, "x missing");
    if (recv_x == nullptr && recv_capacity_rows > 0) return fail(c, EP_ERR_INVALID_ARG, "recv_x missing");
    if (!aligned16(x) || !aligned16(recv_x)) return fail(c, EP_ERR_ALIGNMENT, "row buffers must be 16-byte aligned");
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;
    ep::DispatchParams dp{};
    dp.x = x;
    dp.send_head = h->send_head;
    dp.recv_rank_offset = reinterpret_cast<const long long*>(h->recv_rank_offset);
    dp.recv_capacity = recv_capacity_rows;
    dp.recv_x = recv_x;
    dp.err = c->err;
    dp.G = c->G;
    dp.R = c->R; dp.E = c->E; dp.L = c->L; dp.T = c->T; dp.K = c->K; dp.H = c->H;
    dp.splits = ep::dispatch_splits(c->H);
    return launch(c, kCached, c->G > 0 && recv_x != nullptr, s,
                  [&] { return ep::launch_dispatch(ep::kModeCached, dp, s); });
}

int ep_combine(ep_ctx* c, const uint16_t* y, int64_t num_recv_rows, const ep_handle* h,
               const float* recv_topk_weights, const uint16_t* bias0, const uint16_t* bias1,
               uint16_t* out_x, float* out_topk_weights, ep_stream_t stream, ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (c->num_shards > 1) return fail(c, EP_ERR_INVALID_ARG, "sharded context: use the ep_sharded_* calls");
    if (h == nullptr || (c->G > 0 && h->send_head == nullptr) || h->recv_rank_offset == nullptr)
        return fail(c, EP_ERR_HANDLE_MISMATCH, "handle send_head / recv_rank_offset missing");
    if (num_recv_rows < 0) return fail(c, EP_ERR_INVALID_ARG, "negative row count");
    if (c->G > 0 && out_x == nullptr) return fail(c, EP_ERR_INVALID_ARG, "out_x missing");
    if (num_recv_rows > 0 && y == nullptr) return fail(c, EP_ERR_INVALID_ARG, "y missing");
    if (!aligned16(y) || !aligned16(out_x) || !aligned16(bias0) || !aligned16(bias1))
        return fail(c, EP_ERR_ALIGNMENT, "row buffers must be 16-byte aligned");
    if (!aligned(recv_topk_weights, 4) || !aligned(out_topk_weights, 4))
        return fail(c, EP_ERR_ALIGNMENT, "weight arrays misaligned");
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;
    ep::CombineParams p{};
    p.y = y;
    p.y_rows = num_recv_rows;
    p.send_head = h->send_head;
    p.recv_rank_offset = reinterpret_cast<const long long*>(h->recv_rank_offset);
    p.recv_topk_weights = recv_topk_weights;
    p.bias0 = bias0;
    p.bias1 = bias1;
    p.out_x = out_x;
    p.out_topk_weights = out_topk_weights;
    p.err = c->err;
    p.G = c->G;
    p.R = c->R; p.K = c->K; p.H = c->H;
    p.splits = ep::combine_splits(c->H);
    return launch(c, kCombine, c->G > 0, s, [&] { return ep::launch_combine(p, c->num_sms, s); });
}

}  // extern "C"

namespace {

int ll_dispatch_impl(ep_ctx* c, const uint16_t* x, const int64_t* topk_idx, uint16_t* packed_recv_x,
                     uint8_t* packed_fp8, float* packed_scales, int32_t* packed_recv_count,
                     int32_t* src_info, int32_t* layout_range, ep_stream_t stream, ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (c->num_shards > 1) return fail(c, EP_ERR_INVALID_ARG, "sharded context: use the ep_sharded_* calls");
    const bool fp8 = packed_fp8 != nullptr || packed_scales != nullptr;
    if (packed_recv_count == nullptr || layout_range == nullptr || src_info == nullptr)
        return fail(c, EP_ERR_INVALID_ARG, "low-latency outputs missing");
    if (fp8 && c->H % ep::kFp8Block != 0)
        return fail(c, EP_ERR_INVALID_ARG, "FP8 packing needs hidden %% 128 == 0");
    if (c->G > 0 && (x == nullptr || topk_idx == nullptr ||
                     (fp8 ? (packed_fp8 == nullptr || packed_scales == nullptr) : packed_recv_x == nullptr)))
        return fail(c, EP_ERR_INVALID_ARG, "x / topk_idx / packed outputs missing");
    if (!aligned16(x) || !aligned16(packed_recv_x) || !aligned16(packed_fp8))
        return fail(c, EP_ERR_ALIGNMENT, "row buffers must be 16-byte aligned");
    if (!aligned(topk_idx, 8) || !aligned(packed_scales, 4)) return fail(c, EP_ERR_ALIGNMENT, "array misaligned");
    if (fp8 && !aligned(x, 32))   // the FP8 copy reads x in 32-byte vectors
        return fail(c, EP_ERR_ALIGNMENT, "FP8 packing needs x 32-byte aligned");
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;
    if (c->G == 0) {
        cudaError_t e = cudaMemsetAsync(packed_recv_count, 0, sizeof(int) * (size_t)c->E, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(layout_range, 0, sizeof(int) * 2 * (size_t)c->E * c->R, s);
        return cuda_check(c, e, "zero low-latency counts");
    }
    // slots: direct (per-source ranking; the copy adds the earlier sources' counts)
    // for sources of up to kLLDirectMaxT tokens, else the lookback scan
    const bool direct = c->T <= ep::kLLDirectMaxT;
    if (direct) {
        ep::LLRankParams rp{topk_idx, c->rank_mask, c->ll_cnt, c->ll_within, c->err, c->R, c->E, c->T, c->K};
        rc = launch(c, kLLCount, true, s, [&] { return ep::launch_ll_rank(rp, s); });
    } else {
        ep::LLCountParams cp{topk_idx, c->slot_map, packed_recv_count, src_info, layout_range,
                             c->ll_status, c->ll_src_begin, c->ll_ticket,
                             c->rank_mask, c->err, c->G, c->R, c->E, c->T, c->K, c->ll_cap,
                             c->ll_tiles_per_src, c->ll_tiles};
        rc = launch(c, kLLCount, true, s, [&] { return ep::launch_ll_count(cp, s); });
    }
    if (rc != EP_OK) return rc;
    ep::DispatchParams dp{};
    dp.x = x;
    dp.topk_idx = topk_idx;
    dp.slot_map = c->slot_map;
    dp.ll_cnt = direct ? c->ll_cnt : nullptr;
    dp.ll_within = c->ll_within;
    dp.ll_src_info = src_info;
    dp.ll_layout_range = layout_range;
    dp.ll_count = packed_recv_count;
    dp.num_sms = c->num_sms;
    dp.rank_mask = c->rank_mask;
    dp.ll_capacity = c->ll_cap;
    dp.recv_x = packed_recv_x;
    dp.recv_fp8 = packed_fp8;
    dp.recv_scales = packed_scales;
    dp.err = c->err;
    dp.G = c->G;
    dp.R = c->R; dp.E = c->E; dp.L = c->L; dp.T = c->T; dp.K = c->K; dp.H = c->H;
    dp.splits = ep::dispatch_splits(c->H);
    const int mode = fp8 ? ep::kModeLowLatencyFp8 : ep::kModeLowLatency;
    return launch(c, fp8 ? kLLCopyFp8 : kLLCopy, true, s, [&] { return ep::launch_dispatch(mode, dp, s, true); });
}

}  // namespace

extern "C" {

int ep_ll_dispatch(ep_ctx* c, const uint16_t* x, const int64_t* topk_idx, uint16_t* packed_recv_x,
                   int32_t* packed_recv_count, int32_t* src_info, int32_t* layout_range,
                   ep_stream_t stream, ep_event_t wait_event) {
    if (c != nullptr && c->G > 0 && packed_recv_x == nullptr)
        return fail(c, EP_ERR_INVALID_ARG, "packed_recv_x missing");
    return ll_dispatch_impl(c, x, topk_idx, packed_recv_x, nullptr, nullptr, packed_recv_count, src_info,
                            layout_range, stream, wait_event);
}

int ep_ll_dispatch_fp8(ep_ctx* c, const uint16_t* x, const int64_t* topk_idx, uint8_t* packed_recv_x_fp8,
                       float* packed_recv_scales, int32_t* packed_recv_count, int32_t* src_info,
                       int32_t* layout_range, ep_stream_t stream, ep_event_t wait_event) {
    if (c != nullptr && c->G > 0 && (packed_recv_x_fp8 == nullptr || packed_recv_scales == nullptr))
        return fail(c, EP_ERR_INVALID_ARG, "FP8 outputs missing");
    return ll_dispatch_impl(c, x, topk_idx, nullptr, packed_recv_x_fp8, packed_recv_scales, packed_recv_count,
                            src_info, layout_range, stream, wait_event);
}

int ep_ll_combine(ep_ctx* c, const uint16_t* y, const int64_t* topk_idx, const float* topk_weights,
                  const int32_t* src_info, const int32_t* layout_range, uint16_t* out_x,
                  ep_stream_t stream, ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (c->num_shards > 1) return fail(c, EP_ERR_INVALID_ARG, "sharded context: use the ep_sharded_* calls");
    if (c->G > 0 && (y == nullptr || topk_idx == nullptr || topk_weights == nullptr || src_info == nullptr ||
                     layout_range == nullptr || out_x == nullptr))
        return fail(c, EP_ERR_INVALID_ARG, "low-latency combine argument missing");
    if (!aligned16(y) || !aligned16(out_x)) return fail(c, EP_ERR_ALIGNMENT, "row buffers must be 16-byte aligned");
    if (!aligned(topk_idx, 8) || !aligned(topk_weights, 4)) return fail(c, EP_ERR_ALIGNMENT, "top-k arrays misaligned");
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;
    ep::LLCombineParams p{y, topk_idx, topk_weights, src_info, layout_range, c->rank_mask, c->slot_map, out_x, c->err,
                          c->G, c->R, c->E, c->T, c->K, c->H, c->ll_cap,
                          ep::combine_splits(c->H)};
    return launch(c, kLLCombine, c->G > 0, s, [&] { return ep::launch_ll_combine(p, c->num_sms, s); });
}

int ep_lb_prefetch_weights(ep_ctx* c, const uint16_t* expert_weights, int64_t elems_per_expert,
                           const int32_t* redundancy_mapping, int32_t num_redundant,
                           uint16_t* redundant_weights, ep_stream_t stream, ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (elems_per_expert < 0 || num_redundant < 0 || num_redundant > 65535)
        return fail(c, EP_ERR_INVALID_ARG, "bad sizes");
    if (elems_per_expert % 8 != 0) return fail(c, EP_ERR_ALIGNMENT, "elems_per_expert must be a multiple of 8");
    if (num_redundant > 0 && elems_per_expert > 0 &&
        (expert_weights == nullptr || redundancy_mapping == nullptr || redundant_weights == nullptr))
        return fail(c, EP_ERR_INVALID_ARG, "argument missing");
    if (!aligned16(expert_weights) || !aligned16(redundant_weights) || !aligned(redundancy_mapping, 4))
        return fail(c, EP_ERR_ALIGNMENT, "buffers misaligned");
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;
    ep::LBParams p{const_cast<uint16_t*>(expert_weights), redundant_weights, redundancy_mapping, c->err,
                   elems_per_expert / 8, c->E, num_redundant};
    return launch(c, kLBPrefetch, num_redundant > 0 && elems_per_expert > 0, s,
                  [&] { return ep::launch_lb_prefetch(p, s); });
}

int ep_lb_reduce_grads(ep_ctx* c, const uint16_t* redundant_grads, int64_t elems_per_expert,
                       const int32_t* redundancy_mapping, int32_t num_redundant,
                       uint16_t* expert_grads, ep_stream_t stream, ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (elems_per_expert < 0 || num_redundant < 0 || num_redundant > 65535)
        return fail(c, EP_ERR_INVALID_ARG, "bad sizes");
    if (elems_per_expert % 8 != 0) return fail(c, EP_ERR_ALIGNMENT, "elems_per_expert must be a multiple of 8");
    if (num_redundant > 0 && elems_per_expert > 0 &&
        (redundant_grads == nullptr || redundancy_mapping == nullptr || expert_grads == nullptr))
        return fail(c, EP_ERR_INVALID_ARG, "argument missing");
    if (!aligned16(redundant_grads) || !aligned16(expert_grads) || !aligned(redundancy_mapping, 4))
        return fail(c, EP_ERR_ALIGNMENT, "buffers misaligned");
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;
    ep::LBParams p{expert_grads, const_cast<uint16_t*>(redundant_grads), redundancy_mapping, c->err,
                   elems_per_expert / 8, c->E, num_redundant};
    return launch(c, kLBReduce, num_redundant > 0 && elems_per_expert > 0, s,
                  [&] { return ep::launch_lb_reduce(p, s); });
}

int ep_ll_update_mask(ep_ctx* c, int32_t rank, int32_t masked, ep_stream_t stream) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (rank < 0 || rank >= c->R) return fail(c, EP_ERR_INVALID_ARG, "rank %d out of range", rank);
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return launch(c, -1, true, s, [&] { return ep::launch_set_mask(c->rank_mask, rank, masked ? 1 : 0, s); });
}

int ep_ll_query_mask(ep_ctx* c, int32_t* host_out, ep_stream_t stream) {
    if (c == nullptr || host_out == nullptr) return EP_ERR_INVALID_ARG;
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int rc = cuda_check(c, cudaMemcpyAsync(host_out, c->rank_mask, sizeof(int32_t) * c->R, cudaMemcpyDeviceToHost, s),
                        "read rank mask");
    if (rc == EP_OK) rc = cuda_check(c, cudaStreamSynchronize(s), "cudaStreamSynchronize");
    return rc;
}

int ep_ll_clean_mask(ep_ctx* c, ep_stream_t stream) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    DeviceGuard guard(c->device);
    return cuda_check(c, cudaMemsetAsync(c->rank_mask, 0, sizeof(int) * c->R, reinterpret_cast<cudaStream_t>(stream)),
                      "clear rank mask");
}

// ------------------------------------------------------------ sharded exchange

int ep_sharded_handle(ep_ctx* c, const uint8_t* is_token_in_rank, const int32_t* num_tokens_per_rank_all,
                      const int32_t* num_tokens_per_expert_all, int32_t* send_head, int64_t* dst_offset,
                      int64_t* num_recv_rows, int32_t* num_recv_tokens_per_expert, ep_stream_t stream,
                      ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (num_tokens_per_rank_all == nullptr || num_tokens_per_expert_all == nullptr || dst_offset == nullptr)
        return fail(c, EP_ERR_INVALID_ARG, "gathered counts / dst_offset missing");
    if (c->G > 0 && (is_token_in_rank == nullptr || send_head == nullptr))
        return fail(c, EP_ERR_INVALID_ARG, "is_token_in_rank / send_head missing");
    if (!aligned(is_token_in_rank, 4) || !aligned(dst_offset, 8) || !aligned(num_recv_rows, 8))
        return fail(c, EP_ERR_ALIGNMENT, "sharded handle arrays misaligned");
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;
    ep::ShardOffsetsParams op{num_tokens_per_rank_all, num_tokens_per_expert_all, c->shard_base,
                              reinterpret_cast<long long*>(dst_offset), reinterpret_cast<long long*>(num_recv_rows),
                              num_recv_tokens_per_expert, c->R, c->E, c->L, c->r0, c->Rl};
    rc = launch(c, -1, true, s, [&] { return ep::launch_shard_offsets(op, s); });
    if (rc != EP_OK || c->G == 0) return rc;
    ep::ScanParams sp{};
    sp.is_token_in_rank = is_token_in_rank;
    sp.status = c->scan_status;
    sp.ticket = c->scan_ticket;
    sp.rank_start = c->rank_start;
    sp.base = c->shard_base;
    sp.send_head = send_head;
    sp.err = c->err;
    sp.G = c->G;
    sp.R = c->R; sp.E = c->E; sp.L = c->L; sp.T = c->T; sp.C = c->C;
    sp.q = (c->T + c->C - 1) / c->C;
    sp.num_tiles = c->scan_tiles;
    return launch(c, kScan, true, s, [&] { return ep::launch_scan(sp, s); });
}

namespace {

int check_shard_table(ep_ctx* c, int num_shards, const void* const* table, bool required, const char* what,
                      size_t align) {
    if (table == nullptr) {
        if (required) return fail(c, EP_ERR_INVALID_ARG, "%s pointer table missing", what);
        return EP_OK;
    }
    for (int w = 0; w < num_shards; ++w) {
        if (table[w] == nullptr) return fail(c, EP_ERR_INVALID_ARG, "%s of shard %d missing", what, w);
        if (!aligned(table[w], align)) return fail(c, EP_ERR_ALIGNMENT, "%s of shard %d misaligned", what, w);
    }
    return EP_OK;
}

}  // namespace

int ep_sharded_dispatch(ep_ctx* c, const uint16_t* x, const int64_t* topk_idx, const float* topk_weights,
                        const int32_t* send_head, const int64_t* dst_offset, int num_shards,
                        uint16_t* const* recv_x, int64_t* const* recv_topk_idx,
                        float* const* recv_topk_weights, int32_t* const* recv_src_idx,
                        int64_t recv_capacity_rows, ep_stream_t stream, ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (num_shards != c->num_shards) return fail(c, EP_ERR_INVALID_ARG, "%d shard tables for %d shards",
                                                 num_shards, c->num_shards);
    if (recv_capacity_rows < 0) return fail(c, EP_ERR_INVALID_ARG, "negative capacity");
    if (c->G > 0 && (x == nullptr || topk_idx == nullptr || send_head == nullptr || dst_offset == nullptr))
        return fail(c, EP_ERR_INVALID_ARG, "x / topk_idx / send_head / dst_offset missing");
    if (recv_topk_weights != nullptr && topk_weights == nullptr)
        return fail(c, EP_ERR_INVALID_ARG, "recv_topk_weights needs topk_weights");
    if (!aligned16(x) || !aligned(topk_idx, 8) || !aligned(topk_weights, 4) || !aligned(dst_offset, 8))
        return fail(c, EP_ERR_ALIGNMENT, "inputs misaligned");
    int rc = check_shard_table(c, num_shards, reinterpret_cast<const void* const*>(recv_x), true, "recv_x", 16);
    if (rc == EP_OK)
        rc = check_shard_table(c, num_shards, reinterpret_cast<const void* const*>(recv_topk_idx), false,
                               "recv_topk_idx", 8);
    if (rc == EP_OK)
        rc = check_shard_table(c, num_shards, reinterpret_cast<const void* const*>(recv_topk_weights), false,
                               "recv_topk_weights", 4);
    if (rc == EP_OK)
        rc = check_shard_table(c, num_shards, reinterpret_cast<const void* const*>(recv_src_idx), false,
                               "recv_src_idx", 4);
    if (rc != EP_OK) return rc;
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;
    ep::DispatchParams dp{};
    dp.x = x;
    dp.send_head = send_head;
    dp.recv_capacity = recv_capacity_rows;
    dp.topk_idx = topk_idx;
    dp.topk_weights = topk_weights;
    dp.dst_offset = reinterpret_cast<const long long*>(dst_offset);
    dp.ranks_per_shard = c->Rl;
    for (int w = 0; w < num_shards; ++w) {
        dp.shard_rows[w] = recv_x[w];
        dp.shard_idx[w] = recv_topk_idx ? recv_topk_idx[w] : nullptr;
        dp.shard_w[w] = recv_topk_weights ? recv_topk_weights[w] : nullptr;
        dp.shard_src[w] = recv_src_idx ? recv_src_idx[w] : nullptr;
    }
    dp.err = c->err;
    dp.G = c->G;
    dp.R = c->R; dp.E = c->E; dp.L = c->L; dp.T = c->T; dp.K = c->K; dp.H = c->H;
    dp.splits = ep::dispatch_splits(c->H);
    return launch(c, kDispatch, c->G > 0, s, [&] { return ep::launch_dispatch(ep::kModeSharded, dp, s); });
}

int ep_sharded_combine(ep_ctx* c, int num_shards, const uint16_t* const* y, const float* const* recv_topk_weights,
                       int64_t y_capacity_rows, const int32_t* send_head, const int64_t* dst_offset,
                       const uint16_t* bias0, const uint16_t* bias1, uint16_t* out_x, float* out_topk_weights,
                       ep_stream_t stream, ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (num_shards != c->num_shards) return fail(c, EP_ERR_INVALID_ARG, "%d shard tables for %d shards",
                                                 num_shards, c->num_shards);
    if (y_capacity_rows < 0) return fail(c, EP_ERR_INVALID_ARG, "negative capacity");
    if (c->G > 0 && (send_head == nullptr || dst_offset == nullptr || out_x == nullptr))
        return fail(c, EP_ERR_INVALID_ARG, "send_head / dst_offset / out_x missing");
    if (out_topk_weights != nullptr && recv_topk_weights == nullptr)
        return fail(c, EP_ERR_INVALID_ARG, "out_topk_weights needs the shards' recv_topk_weights");
    if (!aligned16(out_x) || !aligned16(bias0) || !aligned16(bias1) || !aligned(out_topk_weights, 4) ||
        !aligned(dst_offset, 8))
        return fail(c, EP_ERR_ALIGNMENT, "arrays misaligned");
    int rc = check_shard_table(c, num_shards, reinterpret_cast<const void* const*>(y), true, "y", 16);
    if (rc == EP_OK)
        rc = check_shard_table(c, num_shards, reinterpret_cast<const void* const*>(recv_topk_weights), false,
                               "recv_topk_weights", 4);
    if (rc != EP_OK) return rc;
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;
    ep::CombineParams p{};
    p.y_rows = y_capacity_rows;
    p.send_head = send_head;
    p.bias0 = bias0;
    p.bias1 = bias1;
    p.out_x = out_x;
    p.out_topk_weights = out_topk_weights;
    p.sharded = true;
    p.self_shard = c->shard;
    p.dst_offset = reinterpret_cast<const long long*>(dst_offset);
    p.ranks_per_shard = c->Rl;
    for (int w = 0; w < num_shards; ++w) {
        p.shard_y[w] = y[w];
        p.shard_w[w] = recv_topk_weights ? recv_topk_weights[w] : nullptr;
    }
    p.err = c->err;
    p.G = c->G;
    p.R = c->R; p.K = c->K; p.H = c->H;
    p.splits = ep::combine_splits(c->H);
    return launch(c, kCombine, c->G > 0, s, [&] { return ep::launch_combine(p, c->num_sms, s); });
}

// Device memory that another process can map (CUDA IPC): one cudaMalloc per
// buffer, so the handle covers exactly the buffer.
int ep_shared_alloc(size_t bytes, void** ptr, uint8_t* ipc_handle) {
    if (ptr == nullptr || ipc_handle == nullptr || bytes == 0) return EP_ERR_INVALID_ARG;
    *ptr = nullptr;
    void* p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) return EP_ERR_CUDA;
    cudaIpcMemHandle_t h;
    if (cudaIpcGetMemHandle(&h, p) != cudaSuccess) {
        cudaFree(p);
        return EP_ERR_CUDA;
    }
    static_assert(sizeof(h) == EP_IPC_HANDLE_BYTES, "IPC handle size");
    std::memcpy(ipc_handle, &h, sizeof h);
    *ptr = p;
    return EP_OK;
}

int ep_shared_free(void* ptr) { return cudaFree(ptr) == cudaSuccess ? EP_OK : EP_ERR_CUDA; }

int ep_ipc_open(const uint8_t* ipc_handle, void** ptr) {
    if (ipc_handle == nullptr || ptr == nullptr) return EP_ERR_INVALID_ARG;
    *ptr = nullptr;
    cudaIpcMemHandle_t h;
    std::memcpy(&h, ipc_handle, sizeof h);
    return cudaIpcOpenMemHandle(ptr, h, cudaIpcMemLazyEnablePeerAccess) == cudaSuccess ? EP_OK : EP_ERR_CUDA;
}

int ep_ipc_close(void* ptr) { return cudaIpcCloseMemHandle(ptr) == cudaSuccess ? EP_OK : EP_ERR_CUDA; }

int ep_check_handle(ep_ctx* c, const int64_t* topk_idx, const ep_handle* h, ep_stream_t stream,
                    ep_event_t wait_event) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    if (c->num_shards > 1) return fail(c, EP_ERR_INVALID_ARG, "sharded context: the handle check is one-GPU");
    int rc = check_handle(c, h);
    if (rc != EP_OK) return rc;
    if (c->G > 0 && topk_idx == nullptr) return fail(c, EP_ERR_INVALID_ARG, "topk_idx missing");
    if (!aligned(topk_idx, 8)) return fail(c, EP_ERR_ALIGNMENT, "topk_idx misaligned");
    DeviceGuard guard(c->device);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    rc = begin_call(c, s, reinterpret_cast<cudaEvent_t>(wait_event));
    if (rc != EP_OK) return rc;
    ep::HandleCheckParams p{topk_idx, h->is_token_in_rank, h->send_head,
                            reinterpret_cast<const long long*>(h->recv_rank_offset), c->err, c->G,
                            c->R, c->E, c->L, c->K};
    return launch(c, -1, c->G > 0, s, [&] { return ep::launch_handle_check(p, s); });
}

int ep_profile_enable(ep_ctx* c, int enable) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    c->prof = enable != 0;
    return EP_OK;
}

int ep_profile_read(ep_ctx* c, int64_t* launches, double* total_ms) {
    if (c == nullptr) return EP_ERR_INVALID_ARG;
    DeviceGuard guard(c->device);
    int rc = EP_OK;
    for (auto& r : c->pending) {
        float ms = 0.f;
        if (rc == EP_OK && cudaEventSynchronize(r.stop) == cudaSuccess &&
            cudaEventElapsedTime(&ms, r.start, r.stop) == cudaSuccess) {
            c->prof_launches[r.kind] += 1;
            c->prof_ms[r.kind] += ms;
        } else {
            rc = EP_ERR_CUDA;
        }
        cudaEventDestroy(r.start);
        cudaEventDestroy(r.stop);
    }
    c->pending.clear();
    for (int k = 0; k < EP_PROFILE_KINDS; ++k) {
        if (launches) launches[k] = c->prof_launches[k];
        if (total_ms) total_ms[k] = c->prof_ms[k];
        c->prof_launches[k] = 0;
        c->prof_ms[k] = 0.0;
    }
    return rc;
}

}  // extern "C"
