// Instantiations of the input-sparse GEMV kernel: bf16 weights, bf16 activations,
// column tiles 256 and 512.
#include "sfx_gemv_kernel.cuh"

namespace sfx {

int gemv_bf16_bf16_small(const GemvPlan& p, const GemvArgs& a, cudaStream_t s, bool pdl) {
  if (p.NT == 256 && p.BMAX == 1) return launch_t<__nv_bfloat16, __nv_bfloat16, 256, 1>(p, a, s, pdl);
  if (p.NT == 256 && p.BMAX == 2) return launch_t<__nv_bfloat16, __nv_bfloat16, 256, 2>(p, a, s, pdl);
  if (p.NT == 256 && p.BMAX == 4) return launch_t<__nv_bfloat16, __nv_bfloat16, 256, 4>(p, a, s, pdl);
  if (p.NT == 256 && p.BMAX == 8) return launch_t<__nv_bfloat16, __nv_bfloat16, 256, 8>(p, a, s, pdl);
  if (p.NT == 256 && p.BMAX == 16) return launch_t<__nv_bfloat16, __nv_bfloat16, 256, 16>(p, a, s, pdl);
  if (p.NT == 512 && p.BMAX == 1) return launch_t<__nv_bfloat16, __nv_bfloat16, 512, 1>(p, a, s, pdl);
  if (p.NT == 512 && p.BMAX == 2) return launch_t<__nv_bfloat16, __nv_bfloat16, 512, 2>(p, a, s, pdl);
  if (p.NT == 512 && p.BMAX == 4) return launch_t<__nv_bfloat16, __nv_bfloat16, 512, 4>(p, a, s, pdl);
  if (p.NT == 512 && p.BMAX == 8) return launch_t<__nv_bfloat16, __nv_bfloat16, 512, 8>(p, a, s, pdl);
  if (p.NT == 512 && p.BMAX == 16) return launch_t<__nv_bfloat16, __nv_bfloat16, 512, 16>(p, a, s, pdl);
  return SFX_ERR_UNSUPPORTED;
}

}  // namespace sfx
