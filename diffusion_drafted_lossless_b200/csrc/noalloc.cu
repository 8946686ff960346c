// noalloc.cu — block verify with library-owned scratch, for callers that cannot allocate.
//
// uno_block_verify needs a device workspace from its caller. Some callers have none to
// give: a plugin or embedded runtime that only receives device pointers and a stream
// from its host application has no allocator of its own, and a latency-bound serving
// loop may not call cudaMalloc, which can synchronise the whole device. For them this
// entry point uses a fixed scratch array compiled into the library: a file-scope
// __device__ array of UNO_NOALLOC_SCRATCH_BYTES, present on every device that loads the
// library until the process exits. It allocates nothing and frees nothing.
//
// The array's name is only a host-side stand-in for the device storage, so host code
// asks the runtime for its device address (cudaGetSymbolAddress), once per device with
// that device current, on the first call made on that device; that first call should
// come before any stream capture. All calls on a device share the one array and it keeps
// whatever the last call left there; nothing in it has to start at zero (every word the
// verify reads is written earlier in the same call). Calls that can overlap on the GPU
// (other streams, other host threads) race on the array: order them on one stream or
// synchronise between them.
#include <mutex>

#include "common.cuh"

namespace uno {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[UNO_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

uno_status scratch_for_current_device(void** out) {
    int dev = 0;
    uno_status s = check_cuda(cudaGetDevice(&dev), "cudaGetDevice");
    if (s != UNO_OK) return s;
    if (dev < 0 || dev >= kMaxDevices) return set_error(UNO_ERR_UNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        s = check_cuda(cudaGetSymbolAddress(&p, g_noalloc_scratch), "cudaGetSymbolAddress(no-alloc scratch)");
        if (s != UNO_OK) return s;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return UNO_OK;
}

}  // namespace
}  // namespace uno

extern "C" uno_status uno_block_verify_noalloc(const void* verifier_logits, const void* drafter_logits,
                                               uno_dtype dtype, int32_t B, int32_t K, int32_t V, float temperature,
                                               int32_t top_k, float top_p, const int32_t* draft_tokens,
                                               const int32_t* pos0_tokens, const float* uniforms,
                                               int32_t* out_tokens, int32_t* out_count, int32_t* out_next_token,
                                               float* out_p_tok, float* out_q_tok, float* out_tv,
                                               uno_stream_t stream) {
    const size_t need = uno_block_verify_min_workspace_size(B, K, V, top_k, top_p, dtype);
    if (need > (size_t)UNO_NOALLOC_SCRATCH_BYTES)
        return uno::set_error(UNO_ERR_UNSUPPORTED,
                              "uno_block_verify_noalloc: this batch needs %zu bytes of scratch; the fixed array "
                              "holds %zu (use uno_block_verify with a workspace)",
                              need, (size_t)UNO_NOALLOC_SCRATCH_BYTES);
    void* scratch = nullptr;
    if (need > 0) {
        uno_status s = uno::scratch_for_current_device(&scratch);
        if (s != UNO_OK) return s;
    }
    return uno_block_verify(verifier_logits, drafter_logits, dtype, B, K, V, temperature, top_k, top_p, draft_tokens,
                            pos0_tokens, uniforms, out_tokens, out_count, out_next_token, out_p_tok, out_q_tok,
                            out_tv, scratch, need > 0 ? (size_t)UNO_NOALLOC_SCRATCH_BYTES : 0, stream);
}
