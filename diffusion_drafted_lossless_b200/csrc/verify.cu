// verify.cu — dispatch of the block verify. Top-k batches go to the streaming path
// (verify_topk.cu: every row read once by independent CTAs, per-warp exact top-k lists
// merged per row); top-k-off batches to verify_full.cu (bf16 rows: a row-streaming pass that
// decides each row's exact top-p cut, then an item pass over the rows' candidate lists;
// otherwise the cluster-per-position or generic kernels). UNO_VERIFY_TOPK=local or =window
// sends the top-k batches the cluster kernels support (bf16 rows whose length is a multiple
// of 8, 16-byte aligned, k <= 256) to them instead.
#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "verify_common.cuh"

namespace uno {

static bool topk_cluster_selected() {
    const char* e = getenv("UNO_VERIFY_TOPK");
    return e && (strcmp(e, "local") == 0 || strcmp(e, "window") == 0);
}

size_t verify_workspace_bytes(const VerifyArgs& a, bool minimal) {
    if (a.B == 0) return 0;
    if (a.top_k == 0) return verify_full_workspace_bytes(a, !minimal);
    return std::max(verify_topk_workspace_bytes(a), verify_full_workspace_bytes(a, false));
}

uno_status verify_launch(const VerifyArgs& a, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (a.B == 0) return UNO_OK;
    bool taken = false;
    if (a.top_k == 0) return verify_full_launch(a, workspace, workspace_bytes, stream, true, &taken);
    if (topk_cluster_selected()) {
        const uno_status s = verify_full_launch(a, workspace, workspace_bytes, stream, false, &taken);
        if (s != UNO_OK || taken) return s;
    }
    return verify_topk_launch(a, workspace, stream);
}

}  // namespace uno
