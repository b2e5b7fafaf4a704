// Decode kernel instances for f32, head_dim 256 (all block sizes and group sizes).
#include "launch.cuh"

PA_DEFINE_DECODE_LAUNCHER(launch_decode_f32_d256, float, 256)
