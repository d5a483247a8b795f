// Instantiations of the input-sparse GEMV kernel: f16 weights, f16 activations,
// column tiles 256 and 512.
#include "sfx_gemv_kernel.cuh"

namespace sfx {

int gemv_f16_f16_small(const GemvPlan& p, const GemvArgs& a, cudaStream_t s, bool pdl) {
  if (p.NT == 256 && p.BMAX == 1) return launch_t<__half, __half, 256, 1>(p, a, s, pdl);
  if (p.NT == 256 && p.BMAX == 2) return launch_t<__half, __half, 256, 2>(p, a, s, pdl);
  if (p.NT == 256 && p.BMAX == 4) return launch_t<__half, __half, 256, 4>(p, a, s, pdl);
  if (p.NT == 256 && p.BMAX == 8) return launch_t<__half, __half, 256, 8>(p, a, s, pdl);
  if (p.NT == 256 && p.BMAX == 16) return launch_t<__half, __half, 256, 16>(p, a, s, pdl);
  if (p.NT == 512 && p.BMAX == 1) return launch_t<__half, __half, 512, 1>(p, a, s, pdl);
  if (p.NT == 512 && p.BMAX == 2) return launch_t<__half, __half, 512, 2>(p, a, s, pdl);
  if (p.NT == 512 && p.BMAX == 4) return launch_t<__half, __half, 512, 4>(p, a, s, pdl);
  if (p.NT == 512 && p.BMAX == 8) return launch_t<__half, __half, 512, 8>(p, a, s, pdl);
  if (p.NT == 512 && p.BMAX == 16) return launch_t<__half, __half, 512, 16>(p, a, s, pdl);
  return SFX_ERR_UNSUPPORTED;
}

}  // namespace sfx
