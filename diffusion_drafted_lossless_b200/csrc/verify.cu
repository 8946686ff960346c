// verify.cu — dispatch of the block verify to the top-k path or the full-vocabulary path.
#include "verify_common.cuh"

namespace uno {

size_t verify_workspace_bytes(const VerifyArgs& a) {
    if (a.B == 0) return 0;
    return a.top_k > 0 ? verify_topk_workspace_bytes(a) : verify_full_workspace_bytes(a);
}

uno_status verify_launch(const VerifyArgs& a, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    (void)workspace_bytes;
    if (a.B == 0) return UNO_OK;
    return a.top_k > 0 ? verify_topk_launch(a, workspace, stream) : verify_full_launch(a, workspace, stream);
}

}  // namespace uno
