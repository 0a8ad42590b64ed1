// fp32 instantiations of the fused 2D tier.
#define HND_T float
#define HND_FN launch_fused2d_f32
#include "hnd_unit_fused.inc"
