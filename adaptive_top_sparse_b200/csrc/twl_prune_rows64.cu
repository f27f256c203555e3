// The read-once top-p pruner built with 64 weights per thread in CTAs of up to 512 threads (128
// registers each): for rows above 16384 weights, where the per-row scans and reductions that every
// warp of a 1024-thread CTA repeats would dominate.  Same source.
#define TWL_PRUNE_RE 64
#define TWL_PRUNE_MAX_THREADS 512
#define TWL_PRUNE_NS rows64
#include "twl_prune_rows.cu"
