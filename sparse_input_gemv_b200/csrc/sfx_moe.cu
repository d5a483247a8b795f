// MoE layer with intra-expert activation sparsity (placeholder until the
// routed-expert kernels land; the entry point reports the shape unsupported).
#include "sfx_common.cuh"
#include "sfx_internal.h"

namespace sfx {

size_t moe_workspace_bytes(int, int, int, int, int, int) { return 256; }

int run_moe(const void*, int, const float*, int, int, int, int, int, const void*, const void*,
            const void*, const float*, const void*, const void*, int, void*, int, float*,
            int32_t*, int, unsigned char*, size_t, unsigned*, cudaStream_t) {
  return SFX_ERR_UNSUPPORTED;
}

}  // namespace sfx
