"""B200 (sm_100a) library for hierarchical top-p sparse decode attention: Quest-style page
selection, INT4-K weight estimation, bisection top-p pruning and split-KV sparse attention, exposed
through the C ABI in include/twl.h (libtwl.so) and the ctypes binding in ``twl``."""
