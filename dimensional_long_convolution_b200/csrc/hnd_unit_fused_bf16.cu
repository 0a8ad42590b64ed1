// bf16 instantiations of the fused 2D tier.
#include <cuda_bf16.h>
#define HND_T __nv_bfloat16
#define HND_FN launch_fused2d_bf16
#include "hnd_unit_fused.inc"
