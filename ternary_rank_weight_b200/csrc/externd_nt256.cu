// The ALS machinery of externd.cu compiled with 256 threads per CTA, in its own namespace
// (externd_nt256), for plans where one CTA's work per half-step is small: fewer warps shorten the
// barrier-bound chain of each half-step (single matrices up to about 2048 x 2048, small batches).
// Only externd_run_nt256 is exported; every C-ABI entry point stays in externd.cu, which chooses
// the block size.
#define EXTERND_NT 256
#define EXTERND_SECONDARY 1
#define externd externd_nt256
#include "externd.cu"
#undef externd

int externd_run_nt256(const void* in, int np, const void* opt, cudaStream_t stream, int* statuses,
                      externd_stats* stats, void* fixed_base, size_t fixed_cap) {
    return run_secondary(in, np, opt, stream, statuses, stats, fixed_base, fixed_cap);
}
