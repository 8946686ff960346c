// gated_lora.cu — row-gated LoRA linear (placeholder until the tcgen05 kernel lands).
#include "gated_lora.cuh"

namespace uno {

size_t gated_lora_workspace_bytes(int64_t M, int64_t d_in, int64_t d_out, int64_t rank, uno_dtype dtype) {
    (void)M; (void)d_in; (void)d_out; (void)rank; (void)dtype;
    return 256;
}

uno_status gated_lora_launch(const GatedLoraArgs& g, void* workspace, cudaStream_t stream) {
    (void)g; (void)workspace; (void)stream;
    return set_error(UNO_ERR_UNSUPPORTED, "gated LoRA linear is not built yet");
}

}  // namespace uno
