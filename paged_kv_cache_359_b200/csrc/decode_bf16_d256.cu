// Decode kernel instances for bf16, head_dim 256 (all block sizes and group sizes).
#include "launch.cuh"

PA_DEFINE_DECODE_LAUNCHER(launch_decode_bf16_d256, __nv_bfloat16, 256)
