// verify.cu — dispatch of the block verify. Top-k batches go to the streaming path
// (verify_topk.cu: every row read once by independent CTAs, per-warp exact top-k lists
// merged per row); top-k-off batches to the item path (verify_full.cu: one thread-block
// cluster per block position, rows resident in shared memory). UNO_VERIFY_TOPK=local or
// =window sends the top-k batches the item path supports (bf16 rows whose length is a
// multiple of 8, 16-byte aligned, k <= 256) to its cluster kernels instead.
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "verify_common.cuh"

namespace uno {

static bool topk_cluster_selected() {
    const char* e = getenv("UNO_VERIFY_TOPK");
    return e && (strcmp(e, "local") == 0 || strcmp(e, "window") == 0);
}

size_t verify_workspace_bytes(const VerifyArgs& a) {
    if (a.B == 0) return 0;
    if (a.top_k == 0) return verify_full_workspace_bytes(a);
    return std::max(verify_topk_workspace_bytes(a), verify_full_workspace_bytes(a));
}

uno_status verify_launch(const VerifyArgs& a, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    (void)workspace_bytes;
    if (a.B == 0) return UNO_OK;
    bool taken = false;
    if (a.top_k == 0) return verify_full_launch(a, workspace, stream, true, &taken);
    if (topk_cluster_selected()) {
        const uno_status s = verify_full_launch(a, workspace, stream, false, &taken);
        if (s != UNO_OK || taken) return s;
    }
    return verify_topk_launch(a, workspace, stream);
}

}  // namespace uno
