// Instantiations of the input-sparse GEMV kernel: bf16 weights, bf16 activations,
// column tiles 1024 and 2048.
#include "sfx_gemv_kernel.cuh"

namespace sfx {

int gemv_bf16_bf16_large(const GemvPlan& p, const GemvArgs& a, cudaStream_t s, bool pdl) {
  if (p.NT == 1024 && p.BMAX == 1) return launch_t<__nv_bfloat16, __nv_bfloat16, 1024, 1>(p, a, s, pdl);
  if (p.NT == 1024 && p.BMAX == 2) return launch_t<__nv_bfloat16, __nv_bfloat16, 1024, 2>(p, a, s, pdl);
  if (p.NT == 1024 && p.BMAX == 4) return launch_t<__nv_bfloat16, __nv_bfloat16, 1024, 4>(p, a, s, pdl);
  if (p.NT == 1024 && p.BMAX == 8) return launch_t<__nv_bfloat16, __nv_bfloat16, 1024, 8>(p, a, s, pdl);
  if (p.NT == 1024 && p.BMAX == 16) return launch_t<__nv_bfloat16, __nv_bfloat16, 1024, 16>(p, a, s, pdl);
  if (p.NT == 2048 && p.BMAX == 1) return launch_t<__nv_bfloat16, __nv_bfloat16, 2048, 1>(p, a, s, pdl);
  if (p.NT == 2048 && p.BMAX == 2) return launch_t<__nv_bfloat16, __nv_bfloat16, 2048, 2>(p, a, s, pdl);
  if (p.NT == 2048 && p.BMAX == 4) return launch_t<__nv_bfloat16, __nv_bfloat16, 2048, 4>(p, a, s, pdl);
  if (p.NT == 2048 && p.BMAX == 8) return launch_t<__nv_bfloat16, __nv_bfloat16, 2048, 8>(p, a, s, pdl);
  if (p.NT == 2048 && p.BMAX == 16) return launch_t<__nv_bfloat16, __nv_bfloat16, 2048, 16>(p, a, s, pdl);
  return SFX_ERR_UNSUPPORTED;
}

}  // namespace sfx
