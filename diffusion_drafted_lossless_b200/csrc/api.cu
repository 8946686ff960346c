// api.cu — the extern "C" entry points declared in include/uno.h: argument validation on
// the host, workspace sizing, dispatch to the kernels, and error reporting.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "gated_lora.cuh"
#include "tv_loss.cuh"
#include "verify.cuh"

namespace uno {

__device__ uint32_t g_device_status = 0u;

namespace {
thread_local char t_last_error[512] = "";
constexpr int kMaxDevices = 64;
std::mutex g_status_mu;
uint32_t* g_status_ptr[kMaxDevices] = {};
}

// The device address of the status word on the current device, looked up once per device
// (the cache is shared by all host threads, so it is filled under a lock).
uint32_t* device_status_ptr() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (!g_status_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
        g_status_ptr[dev] = static_cast<uint32_t*>(p);
    }
    return g_status_ptr[dev];
}

uno_status set_error(uno_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
    va_end(ap);
    return s;
}

uno_status check_cuda(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return UNO_OK;
    return set_error(UNO_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

static bool misaligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

static uno_status check_workspace(void* ws, size_t have, size_t need) {
    if (need == 0) return UNO_OK;
    if (ws == nullptr) return set_error(UNO_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return set_error(UNO_ERR_WORKSPACE, "workspace not 256-byte aligned");
    if (have < need) return set_error(UNO_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", have, need);
    return UNO_OK;
}

}  // namespace uno

using namespace uno;

extern "C" {

const char* uno_status_string(uno_status s) {
    switch (s) {
        case UNO_OK: return "UNO_OK";
        case UNO_ERR_INVALID_ARG: return "UNO_ERR_INVALID_ARG";
        case UNO_ERR_UNSUPPORTED: return "UNO_ERR_UNSUPPORTED";
        case UNO_ERR_CUDA: return "UNO_ERR_CUDA";
        case UNO_ERR_TIMEOUT: return "UNO_ERR_TIMEOUT";
        case UNO_ERR_WORKSPACE: return "UNO_ERR_WORKSPACE";
    }
    return "UNO_ERR_UNKNOWN";
}

const char* uno_last_error_string(void) { return t_last_error; }

int uno_version(void) { return 10000; }

uno_status uno_read_device_status(uint32_t* code) {
    if (!code) return set_error(UNO_ERR_INVALID_ARG, "code is NULL");
    uno_status s = check_cuda(cudaDeviceSynchronize(), "cudaDeviceSynchronize");
    if (s != UNO_OK) return s;
    uint32_t v = 0, zero = 0;
    s = check_cuda(cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)), "cudaMemcpyFromSymbol(status)");
    if (s != UNO_OK) return s;
    s = check_cuda(cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)), "cudaMemcpyToSymbol(status)");
    if (s != UNO_OK) return s;
    *code = v;
    return UNO_OK;
}

// ---------------------------------------------------------------------------------------
// gated LoRA linear
// ---------------------------------------------------------------------------------------
static uno_status lora_validate(const void* x, const void* w0, const void* a, const void* b, int64_t M,
                                int64_t d_in, int64_t d_out, int64_t rank, uno_dtype dtype, const void* y) {
    if (!x || !w0 || !a || !b || !y) return set_error(UNO_ERR_INVALID_ARG, "a tensor pointer is NULL");
    if (M < 1 || d_in < 1 || d_out < 1 || rank < 1)
        return set_error(UNO_ERR_INVALID_ARG, "sizes must be positive (M=%lld d_in=%lld d_out=%lld rank=%lld)",
                         (long long)M, (long long)d_in, (long long)d_out, (long long)rank);
    if (dtype != UNO_BF16 && dtype != UNO_F32) return set_error(UNO_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (d_in % 64 || d_out % 64) return set_error(UNO_ERR_UNSUPPORTED, "d_in and d_out must be multiples of 64");
    if (rank % 8 || rank > 256) return set_error(UNO_ERR_UNSUPPORTED, "rank must be a multiple of 8 and <= 256");
    if (M > (1 << 20) || d_in > 65536 || d_out > 65536)
        return set_error(UNO_ERR_UNSUPPORTED, "M <= 2^20 and d_in, d_out <= 65536 are supported");
    if (misaligned(x) || misaligned(w0) || misaligned(a) || misaligned(b) || misaligned(y))
        return set_error(UNO_ERR_UNSUPPORTED, "tensor pointers must be 16-byte aligned");
    return UNO_OK;
}

size_t uno_gated_lora_linear_workspace_size(int64_t M, int64_t d_in, int64_t d_out, int64_t rank, uno_dtype dtype) {
    if (M < 1 || d_in < 1 || d_out < 1 || rank < 1) return 0;
    return gated_lora_workspace_bytes(M, d_in, d_out, rank, dtype);
}

uno_status uno_gated_lora_linear(const void* x, const void* w0, const void* lora_a, const void* lora_b,
                                 const float* row_gate, float scale, int64_t M, int64_t d_in, int64_t d_out,
                                 int64_t rank, uno_dtype dtype, void* y, void* workspace, size_t workspace_bytes,
                                 uno_stream_t stream) {
    uno_status s = lora_validate(x, w0, lora_a, lora_b, M, d_in, d_out, rank, dtype, y);
    if (s != UNO_OK) return s;
    if (row_gate && misaligned(row_gate)) return set_error(UNO_ERR_UNSUPPORTED, "row_gate must be 16-byte aligned");
    s = check_workspace(workspace, workspace_bytes, gated_lora_workspace_bytes(M, d_in, d_out, rank, dtype));
    if (s != UNO_OK) return s;
    GatedLoraArgs g{x, w0, lora_a, lora_b, row_gate, scale, M, d_in, d_out, rank, dtype, y};
    return gated_lora_launch(g, workspace, reinterpret_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------------------
// block verify
// ---------------------------------------------------------------------------------------
static uno_status verify_args(VerifyArgs& a, const void* P, const void* Q, uno_dtype dtype, int32_t B, int32_t K,
                              int32_t V, float temperature, int32_t top_k, float top_p) {
    if (dtype != UNO_BF16 && dtype != UNO_F32) return set_error(UNO_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (B < 0 || K < 1 || V < 1) return set_error(UNO_ERR_INVALID_ARG, "need B >= 0, K >= 1, V >= 1");
    if (!(temperature > 0.0f) || !(temperature < INFINITY))
        return set_error(UNO_ERR_INVALID_ARG, "temperature must be positive and finite");
    if (!(top_p > 0.0f)) return set_error(UNO_ERR_INVALID_ARG, "top_p must be > 0 (>= 1 turns it off)");
    if (top_k < 0) return set_error(UNO_ERR_INVALID_ARG, "top_k must be >= 0");
    if (K > 32) return set_error(UNO_ERR_UNSUPPORTED, "block size K <= 32 is supported");
    if (V > 0x7FFFF000) return set_error(UNO_ERR_UNSUPPORTED, "V < 2^31 - 4096 is supported");
    if ((double)B * K * V >= 1099511627776.0) return set_error(UNO_ERR_UNSUPPORTED, "B * K * V < 2^40 is supported");
    if (top_k > 1024 && top_k < V) return set_error(UNO_ERR_UNSUPPORTED, "top_k <= 1024 is supported");
    a = VerifyArgs{};
    a.P = P;
    a.Q = Q;
    a.dtype = dtype;
    a.B = B;
    a.K = K;
    a.V = V;
    a.temperature = temperature;
    a.top_k = (top_k >= V) ? 0 : top_k;
    a.top_p = top_p >= 1.0f ? 1.0f : top_p;
    return UNO_OK;
}

size_t uno_block_verify_workspace_size(int32_t B, int32_t K, int32_t V, int32_t top_k, float top_p, uno_dtype dtype) {
    VerifyArgs a;
    if (verify_args(a, nullptr, nullptr, dtype, B, K, V, 1.0f, top_k, top_p) != UNO_OK) return 0;
    return verify_workspace_bytes(a, false);
}

size_t uno_block_verify_min_workspace_size(int32_t B, int32_t K, int32_t V, int32_t top_k, float top_p,
                                           uno_dtype dtype) {
    VerifyArgs a;
    if (verify_args(a, nullptr, nullptr, dtype, B, K, V, 1.0f, top_k, top_p) != UNO_OK) return 0;
    return verify_workspace_bytes(a, true);
}

uno_status uno_block_verify(const void* verifier_logits, const void* drafter_logits, uno_dtype dtype, int32_t B,
                            int32_t K, int32_t V, float temperature, int32_t top_k, float top_p,
                            const int32_t* draft_tokens, const int32_t* pos0_tokens, const float* uniforms,
                            int32_t* out_tokens, int32_t* out_count, int32_t* out_next_token, float* out_p_tok,
                            float* out_q_tok, float* out_tv, void* workspace, size_t workspace_bytes,
                            uno_stream_t stream) {
    VerifyArgs a;
    uno_status s = verify_args(a, verifier_logits, drafter_logits, dtype, B, K, V, temperature, top_k, top_p);
    if (s != UNO_OK) return s;
    if (B == 0) return UNO_OK;
    if (!verifier_logits || !drafter_logits || !uniforms || !out_tokens || !out_count)
        return set_error(UNO_ERR_INVALID_ARG, "verifier/drafter logits, uniforms, out_tokens, out_count are required");
    const void* ptrs[] = {verifier_logits, drafter_logits, draft_tokens, pos0_tokens, uniforms, out_tokens,
                          out_count, out_next_token, out_p_tok, out_q_tok, out_tv};
    for (const void* p : ptrs)
        if (p && misaligned(p)) return set_error(UNO_ERR_UNSUPPORTED, "tensor pointers must be 16-byte aligned");
    a.drafts = draft_tokens;
    a.pos0 = pos0_tokens;
    a.u = uniforms;
    a.out_tokens = out_tokens;
    a.out_count = out_count;
    a.out_next = out_next_token;
    a.out_p = out_p_tok;
    a.out_q = out_q_tok;
    a.out_tv = out_tv;
    s = check_workspace(workspace, workspace_bytes, verify_workspace_bytes(a, true));
    if (s != UNO_OK) return s;
    return verify_launch(a, workspace, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

// ---------------------------------------------------------------------------------------
// TV loss
// ---------------------------------------------------------------------------------------
size_t uno_tv_loss_workspace_size(int64_t N, int64_t V, uno_dtype dtype) {
    if (N < 0 || V < 1) return 0;
    return tv_loss_workspace_bytes(N, V, dtype);
}

uno_status uno_tv_loss(const void* teacher_logits, const void* student_logits, uno_dtype dtype, int64_t N, int64_t V,
                       const uint8_t* response_mask, float grad_scale, float* out_tv, float* out_mean,
                       void* grad_student, void* workspace, size_t workspace_bytes, uno_stream_t stream) {
    if (dtype != UNO_BF16 && dtype != UNO_F32) return set_error(UNO_ERR_INVALID_ARG, "unknown dtype %d", (int)dtype);
    if (N < 0 || V < 1) return set_error(UNO_ERR_INVALID_ARG, "need N >= 0 and V >= 1");
    if (!(grad_scale == grad_scale) || grad_scale == INFINITY || grad_scale == -INFINITY)
        return set_error(UNO_ERR_INVALID_ARG, "grad_scale must be finite");
    if (V > 0x7FFFF000) return set_error(UNO_ERR_UNSUPPORTED, "V < 2^31 - 4096 is supported");
    if ((double)N * V >= 1099511627776.0) return set_error(UNO_ERR_UNSUPPORTED, "N * V < 2^40 is supported");
    if (!out_mean || (N > 0 && (!teacher_logits || !student_logits || !out_tv)))
        return set_error(UNO_ERR_INVALID_ARG, "teacher/student logits, out_tv and out_mean are required");
    const void* ptrs[] = {teacher_logits, student_logits, response_mask, out_tv, out_mean, grad_student};
    for (const void* p : ptrs)
        if (p && misaligned(p)) return set_error(UNO_ERR_UNSUPPORTED, "tensor pointers must be 16-byte aligned");
    uno_status s = check_workspace(workspace, workspace_bytes, tv_loss_workspace_bytes(N, V, dtype));
    if (s != UNO_OK) return s;
    TVArgs t{teacher_logits, student_logits, dtype, N, V, response_mask, grad_scale, out_tv, out_mean, grad_student};
    return tv_loss_launch(t, workspace, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
