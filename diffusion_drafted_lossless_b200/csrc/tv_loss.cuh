// tv_loss.cuh — internal interface of the TV self-distillation loss kernels.
#pragma once

#include "common.cuh"

namespace uno {

struct TVArgs {
    const void* teacher;
    const void* student;
    uno_dtype dtype;
    int64_t N, V;
    const uint8_t* mask;
    float grad_scale;
    float* out_tv;
    float* out_mean;
    void* grad;
};

size_t tv_loss_workspace_bytes(int64_t N, int64_t V, uno_dtype dtype);
uno_status tv_loss_launch(const TVArgs& a, void* workspace, cudaStream_t stream);

}  // namespace uno
