// verify.cuh — internal interface of the block-verify kernels (not part of the C ABI).
#pragma once

#include "common.cuh"

namespace uno {

struct VerifyArgs {
    const void* P;   // verifier logits [B, K, V]
    const void* Q;   // drafter logits  [B, K, V]
    uno_dtype dtype;
    int B, K, V;
    float temperature;
    int top_k;       // normalised: 0 = off (also when >= V)
    float top_p;     // normalised: >= 1 = off
    const int32_t* drafts;
    const int32_t* pos0;
    const float* u;
    int32_t* out_tokens;
    int32_t* out_count;
    int32_t* out_next;
    float* out_p;
    float* out_q;
    float* out_tv;
};

// Bytes of workspace the verify uses for these arguments (0 if B == 0): the fastest path's,
// or (minimal) the least it accepts.
size_t verify_workspace_bytes(const VerifyArgs& a, bool minimal);

// Enqueue the verify on `stream`; the workspace is at least verify_workspace_bytes(a, true).
uno_status verify_launch(const VerifyArgs& a, void* workspace, size_t workspace_bytes, cudaStream_t stream);

}  // namespace uno
