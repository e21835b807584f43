// The ALS machinery of externd.cu compiled a second time with 1024 threads per CTA, in its own
// namespace (externd_nt1024), for the factorization plans of groups of 2 to 12 CTAs: with few CTAs
// per matrix each CTA's share of the threshold pass, the change lists and the GEMV rows is large,
// and twice the threads shorten the half-step (the 16-matrix 1536 x 1536 batch, 9 CTAs per matrix,
// runs about 13 % faster; single large matrices, 148 CTAs, about 5 % slower, so they stay at 512).
// Only externd_run_nt1024 is exported; every C-ABI entry point stays in externd.cu.
#define EXTERND_NT 1024
#define EXTERND_SECONDARY 1
#define externd externd_nt1024
#include "externd.cu"
#undef externd

int externd_run_nt1024(const void* in, int np, const void* opt, cudaStream_t stream, int* statuses,
                       externd_stats* stats) {
    const int rc = run(static_cast<const ProbIn*>(in), np, *static_cast<const RunOpts*>(opt), stream, statuses);
    *stats = g_last;
    return rc;
}
