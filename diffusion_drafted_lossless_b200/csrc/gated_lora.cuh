// gated_lora.cuh — internal interface of the row-gated LoRA linear kernels.
#pragma once

#include "common.cuh"

namespace uno {

struct GatedLoraArgs {
    const void* x;
    const void* w0;
    const void* a;
    const void* b;
    const float* gate;
    float scale;
    int64_t M, d_in, d_out, rank;
    uno_dtype dtype;
    void* y;
};

size_t gated_lora_workspace_bytes(int64_t M, int64_t d_in, int64_t d_out, int64_t rank, uno_dtype dtype);
uno_status gated_lora_launch(const GatedLoraArgs& g, void* workspace, cudaStream_t stream);

}  // namespace uno
