// bwd_kernels.cuh -- backward pass (placeholder until the kernels land).
#pragma once

#include "schedule.cuh"
#include "sm100.cuh"

namespace fa {

struct BwdArgs {
    Geometry g;
    int d;
    const void *q, *k, *v, *o, *dO;
    const float* lse;
    void *dq, *dk, *dv;
    float* D;
    float scale;
    int num_sms;
    int* error_word;
    uint64_t timeout_ns;
};

inline size_t bwd_workspace_bytes(int64_t rows, int H) {
    return static_cast<size_t>((rows * H * 4 + 255) / 256 * 256);
}

inline cudaError_t bwd_set_smem_limits() { return cudaSuccess; }

inline cudaError_t bwd_launch(const BwdArgs&, const CUtensorMap*, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace fa
