// Instantiations of the input-sparse GEMV kernel: f16 weights, f16 activations,
// column tiles 1024 and 2048.
#include "sfx_gemv_kernel.cuh"

namespace sfx {

int gemv_f16_f16_large(const GemvPlan& p, const GemvArgs& a, cudaStream_t s, bool pdl) {
  if (p.NT == 1024 && p.BMAX == 1) return launch_t<__half, __half, 1024, 1>(p, a, s, pdl);
  if (p.NT == 1024 && p.BMAX == 2) return launch_t<__half, __half, 1024, 2>(p, a, s, pdl);
  if (p.NT == 1024 && p.BMAX == 4) return launch_t<__half, __half, 1024, 4>(p, a, s, pdl);
  if (p.NT == 1024 && p.BMAX == 8) return launch_t<__half, __half, 1024, 8>(p, a, s, pdl);
  if (p.NT == 1024 && p.BMAX == 16) return launch_t<__half, __half, 1024, 16>(p, a, s, pdl);
  if (p.NT == 2048 && p.BMAX == 1) return launch_t<__half, __half, 2048, 1>(p, a, s, pdl);
  if (p.NT == 2048 && p.BMAX == 2) return launch_t<__half, __half, 2048, 2>(p, a, s, pdl);
  if (p.NT == 2048 && p.BMAX == 4) return launch_t<__half, __half, 2048, 4>(p, a, s, pdl);
  if (p.NT == 2048 && p.BMAX == 8) return launch_t<__half, __half, 2048, 8>(p, a, s, pdl);
  if (p.NT == 2048 && p.BMAX == 16) return launch_t<__half, __half, 2048, 16>(p, a, s, pdl);
  return SFX_ERR_UNSUPPORTED;
}

}  // namespace sfx
