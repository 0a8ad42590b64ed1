// bf16 instantiations of the fused 2D tier.
#define HND_IO IOBF16
#define HND_FN launch_fused2d_bf16
#include "hnd_unit_fused.inc"
