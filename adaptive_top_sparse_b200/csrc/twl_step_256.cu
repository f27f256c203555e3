// The decode step's persistent kernel built with 256-thread CTAs, two resident per SM
// (namespace twl::step256): the same source as twl_step.cu, for batches with more (sequence,
// kv-head) groups than SMs, where two items in flight per SM hide each other's latency.
#define TWL_STEP_THREADS 256
#define TWL_STEP_NS step256
#include "twl_step.cu"
