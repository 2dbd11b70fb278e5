// gdn_prefill.cu -- chunked GDN prefill (being rebuilt; see gdn_decode.cu for the
// decode step).  Until the tcgen05 prefill kernel lands, the launcher reports
// cudaErrorNotSupported so that gdn_prefill returns GDN_ERR_CUDA.
#include "gdn_internal.h"

namespace gdn {

size_t prefill_workspace_bytes(int N, int T, int H_qk, int H_v, bool bf16) {
    (void)N;
    if (bf16) return 0;
    auto up = [](size_t b) { return (b + 255) & ~size_t(255); };
    return up((size_t)T * H_qk * 128 * 2) * 2 + up((size_t)T * H_v * 128 * 2);
}

cudaError_t launch_prefill(const void*, const void*, const void*, const float*, const float*,
                           const float*, const int32_t*, int, int, int, int, bool, void*,
                           float*, void*, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace gdn
