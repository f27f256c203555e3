// The fused decode step built with 256-thread CTAs and at most 110 KB of shared memory, so two
// CTAs share an SM: for batches with more (sequence, kv-head) groups than SMs, where one
// 512-thread CTA per group leaves the SM waiting on its serial phases.  Same source.
#define TWL_FUSED_THREADS 256
#define TWL_FUSED_NS fused256
#include "twl_fused.cu"
