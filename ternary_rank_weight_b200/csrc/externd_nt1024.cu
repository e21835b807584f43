// The ALS machinery of externd.cu compiled with 1024 threads per CTA, in its own namespace
// (externd_nt1024), for plans where one CTA's work per half-step is large: its share of the
// residual plus the vectors it thresholds (e.g. 16 matrices of 1536 x 1536 over 9 CTAs each).
// Only externd_run_nt1024 is exported; every C-ABI entry point stays in externd.cu, which chooses
// the block size.
#define EXTERND_NT 1024
#define EXTERND_SECONDARY 1
#define externd externd_nt1024
#include "externd.cu"
#undef externd

int externd_run_nt1024(const void* in, int np, const void* opt, cudaStream_t stream, int* statuses,
                       externd_stats* stats, void* fixed_base, size_t fixed_cap) {
    return run_secondary(in, np, opt, stream, statuses, stats, fixed_base, fixed_cap);
}
