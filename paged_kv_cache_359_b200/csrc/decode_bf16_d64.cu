// Decode kernel instances for bf16, head_dim 64 (all block sizes and group sizes).
#include "launch.cuh"

PA_DEFINE_DECODE_LAUNCHER(launch_decode_bf16_d64, __nv_bfloat16, 64)
