// prefill.cu -- opening-context prefill (placeholder until the chunked SSD path lands).
#include "prefill.cuh"

namespace vc {

size_t prefill_workspace_bytes(int, int, int, int, int, int, int, int, int, int, int, int, int) { return 256; }

cudaError_t run_prefill(const PrefillCtx&, const uint16_t*, int, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace vc
