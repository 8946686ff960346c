// noise.cu — the block-noised copy, noise mode random_uniform.
//
// LoopUno project page, "Training is self-distillation" (the student reads a block-noised
// copy of each sequence) and "How it works" (position 0 of a block is the exact AR token;
// the adapter is on only for the noise positions); uno-qwen3-8B model card, "Evaluation
// protocol" (noise mode random_uniform). Position 0 keeps its token; every draft position
// gets min(V - 1, floor(u * V)) from its float32 uniform u, in fp64 (exact for V < 2^24);
// the optional row gate is 0 at position 0 and 1 at the noise positions.
#include "common.cuh"

namespace uno {
namespace {

__global__ void noise_kernel(const int32_t* __restrict__ clean, const float* __restrict__ u, int64_t n, int K, int V,
                             int32_t* __restrict__ out, float* __restrict__ gate) {
    for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < n; o += (int64_t)gridDim.x * blockDim.x) {
        const int i = (int)(o % K);
        int32_t t;
        if (i == 0) {
            t = clean[o];
        } else {
            const double x = floor((double)u[o] * (double)V);
            t = x > (double)(V - 1) ? V - 1 : (int32_t)x;
        }
        out[o] = t;
        if (gate) gate[o] = i == 0 ? 0.f : 1.f;
    }
}

bool misaligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) != 0; }

}  // namespace
}  // namespace uno

extern "C" uno_status uno_block_noise(const int32_t* clean_tokens, const float* uniforms, int32_t B, int32_t K,
                                      int32_t V, int32_t* noised_tokens, float* row_gate, uno_stream_t stream) {
    using namespace uno;
    if (B < 0 || K < 1) return set_error(UNO_ERR_INVALID_ARG, "need B >= 0 and K >= 1");
    if (V < 1 || V >= (1 << 24)) return set_error(UNO_ERR_INVALID_ARG, "need 1 <= V < 2^24");
    if (B == 0) return UNO_OK;
    if (!clean_tokens || !uniforms || !noised_tokens)
        return set_error(UNO_ERR_INVALID_ARG, "clean_tokens, uniforms and noised_tokens are required");
    if (misaligned4(clean_tokens) || misaligned4(uniforms) || misaligned4(noised_tokens) ||
        (row_gate && misaligned4(row_gate)))
        return set_error(UNO_ERR_UNSUPPORTED, "pointers must be 4-byte aligned");
    const int64_t n = (int64_t)B * K;
    const int64_t blocks = (n + 255) / 256;
    noise_kernel<<<(unsigned)(blocks < 1184 ? blocks : 1184), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        clean_tokens, uniforms, n, K, V, noised_tokens, row_gate);
    return check_cuda(cudaGetLastError(), "launch(block noise)");
}
