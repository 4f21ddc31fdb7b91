// Handle check (see check.cu): parameters and launcher.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace ep {

struct HandleCheckParams {
    const int64_t* topk_idx;           // [G][K]
    const uint8_t* is_token_in_rank;   // [G][R]
    const int* send_head;              // [G][R]
    const long long* recv_rank_offset; // [R+1]
    int* err;
    long long G;
    int R, E, L, K;
};
cudaError_t launch_handle_check(const HandleCheckParams& p, cudaStream_t stream);

}  // namespace ep
