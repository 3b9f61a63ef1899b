// bf16 path: placeholder that routes to the SIMT kernels until the
// tensor-core kernels land.
#include "jmix_internal.cuh"

namespace jmix {
size_t fast_ws_bytes(const Problem& p) { return simple_ws_bytes(p); }
cudaError_t run_fast(Problem& p) { return run_simple(p); }
}  // namespace jmix
