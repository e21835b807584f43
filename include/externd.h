/*
 * externd.h -- C ABI of the B200 (sm_100a) library for ExTernD greedy
 * sequential ternary ALS.
 *
 * Method: "ExTernD: Expanded-Rank Ternary Decomposition" (arXiv 2607.13511),
 *   §2.1  A ~ Ahat = B diag(D) C, B in {-1,0,1}^{m x k}, C in {-1,0,1}^{k x n},
 *         k = mu * min(m, n); energy E = 1 - ||A - Ahat||_F^2 / ||A||_F^2.
 *   §2.2  T_tau(x)_i = sign(x_i) * 1[|x_i| > tau * mean_j |x_j|], keeping the
 *         single largest entry when the result would be all-zero.
 *   §2.3  R <- A; per component: 15 x {v <- T_tau(R^T u), u <- T_tau(R v)},
 *         d = u^T R v / (||u||^2 ||v||^2), R <- R - d u v^T.
 *
 * Readings where the pages are silent (start vector, tie-breaks, k rounding)
 * are fixed below and documented with the library.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Matrices are fp32, row-major, leading dimension = number of columns.
 * - Pointers may be device memory or host memory (pageable or pinned); the
 *   library detects which with cudaPointerGetAttributes.  Host buffers are
 *   staged through device memory on `stream` (copies inside the call).
 *   Device buffers of B/C rows must be 16-byte aligned.
 * - `stream` is a cudaStream_t (NULL = legacy default stream) of the current
 *   device.  Every call is stream-ordered and SYNCHRONOUS: it returns after
 *   the work finished, because the return code carries the device status --
 *   except the factorizations given an async_status int (externd_options,
 *   externd_batch_options), which return once their work is queued and deliver
 *   the status through that int, and externd_matvec.
 * - The library keeps no pointer after return (an asynchronous call's queued
 *   work still uses the caller's buffers until the stream reaches its end).
 *   Workspace (the residual in two layouts, each entry an fp32 pair hi + lo;
 *   exchange buffers, start trits) is allocated stream-ordered inside the call
 *   and released before it returns (asynchronous calls: released in stream
 *   order).
 * - Ternary outputs are packed 2 bits per trit: 00 = 0, 01 = +1, 11 = -1
 *   (10 is never written).  Trit j of a row sits in byte j/4, bits 2*(j%4).
 *   A row of `len` trits occupies externd_trit_bytes(len) bytes (ceil(len/4)
 *   rounded up to 16); padding trits are 0.
 * - Start vector of component i (0-based): u0 = T_tau(z), z_j ~ N(0,1) for
 *   j < m from Philox4x32-10 (Salmon et al., SC'11) with counter
 *   (j, i, 1, 0) and key (seed & 0xffffffff, seed >> 32); two 53-bit uniforms
 *   u1 = words (1:0), u2 = words (3:2), each ((w >> 11) + 0.5) * 2^-53;
 *   z = sqrt(-2 ln u1) * cos(2 pi u2).
 * - "15 iterations" = 15 (V-step, U-step) pairs; d uses the final u and the v
 *   of the same pair.  T_tau's mean runs over the vector's own length.  The
 *   all-zero fallback keeps the lowest index among the largest magnitudes;
 *   an identically zero vector becomes +1 at index 0.  If u^T R v = 0 the
 *   component is stored with d = 0 and R is unchanged.
 */
#ifndef EXTERND_H
#define EXTERND_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    EXTERND_OK = 0,
    EXTERND_EINVAL = -1,      /* null pointer, m or n < 1, non-finite mu/tau, tau < 0, iters < 1, k < 1, misaligned rows */
    EXTERND_EZERO = -2,       /* ||A||_F = 0: the energy of §2.1 is undefined */
    EXTERND_ENONFINITE = -3,  /* A (or R) holds NaN or Inf */
    EXTERND_ENOMEM = -4,      /* workspace allocation failed */
    EXTERND_ECUDA = -5,       /* a CUDA runtime call failed */
    EXTERND_ELAUNCH = -6,     /* the cooperative ALS grid cannot be co-resident */
    EXTERND_ETIMEOUT = -7,    /* a device-side wait gave up (limit per wait, default 2 s) */
    EXTERND_ELIMIT = -8       /* shape beyond this build's limits (m + n too large for on-chip lists) */
} externd_status;

/* k = mu * min(m, n) rounded half away from zero (§2.1); -1 if m < 1, n < 1,
 * mu is not finite, or the result is < 1. */
int64_t externd_rank(int64_t m, int64_t n, double mu);

/* Bytes of one packed trit row of length `len`: ceil(len/4) rounded up to 16.
 * 0 for len < 1. */
size_t externd_trit_bytes(int64_t len);

/* Factor one matrix by greedy sequential ALS (§2.3).
 *   A          [in]  m x n fp32 row-major; not modified.
 *   mu, tau          inner-rank multiplier (k = externd_rank(m, n, mu)) and
 *                    T_tau scale (finite, >= 0).
 *   iters            alternating fits per component (the pages use 15), >= 1.
 *   seed             start-vector seed (see conventions).
 *   B_out      [out] k rows x externd_trit_bytes(m) bytes: row i = column i of B.
 *   D_out      [out] k fp32 scales d_i.
 *   C_out      [out] k rows x externd_trit_bytes(n) bytes: row i = row i of C.
 *   energy_out [out] nullable; k doubles, E after component i, accumulated
 *                    in fp64 from the exact decrease p_i^2 / (nnz(u_i) nnz(v_i)).
 * Returns EXTERND_OK or a negative externd_status. */
int externd_factor(const float* A, int64_t m, int64_t n, double mu, double tau, int iters,
                   uint64_t seed, uint8_t* B_out, float* D_out, uint8_t* C_out,
                   double* energy_out, void* stream);

/* Importance-weighted factorization (§2.5): minimizes sum_ij h~_j (A - Ahat)^2_ij with
 * h~ = h / max(h) + lambda (computed in fp64, held in fp32), by the sequential ALS of
 * §2.3 with the V-step on the plain residual R (h~ cancels there), the U-step on
 * W = R diag(h~) and the scale d = u^T R (h~ v) / (nnz(u) sum_{v_j != 0} h~_j).
 *   h          [in]  n per-input-channel (per-column) second moments, fp32, finite and
 *                    >= 0 with a positive maximum (else EXTERND_EINVAL).
 *   lambda           >= 0, finite: lambda -> infinity approaches the plain objective.
 *   energy_out [out] nullable; k doubles, the weighted energy
 *                    1 - sum h~ (A - Ahat)^2 / sum h~ A^2 after each component.
 * Other arguments, outputs and conventions are those of externd_factor. */
int externd_factor_weighted(const float* A, int64_t m, int64_t n, double mu, double tau, int iters,
                            uint64_t seed, const float* h, double lambda, uint8_t* B_out, float* D_out,
                            uint8_t* C_out, double* energy_out, void* stream);

/* Allocation-free variant of externd_factor.  The pages have no counterpart:
 * this entry point exists for callers that cannot allocate device memory while
 * it runs -- for example an inference or conversion service whose memory pool
 * has already reserved the GPU's memory, or a caller that must not take the
 * implicit device synchronisation an allocation can cause.
 *
 * It runs the same kernels as externd_factor, but its scratch (the two residual
 * layouts, exchange buffers, start trits, control words) lives in one static
 * device array of EXTERND_NOALLOC_SCRATCH_BYTES that every GPU loading this
 * library holds until the process exits.  It calls no cudaMalloc / cudaFree and
 * no allocating library routine.
 *   - A, B_out, D_out, C_out, energy_out must be DEVICE pointers (EXTERND_EINVAL
 *     otherwise: host buffers would need staging memory).
 *   - A matrix whose scratch would exceed EXTERND_NOALLOC_SCRATCH_BYTES is
 *     rejected with EXTERND_ELIMIT (about 16 m n + k ceil(m/4) bytes: the residual
 *     in two layouts, each as an fp32 pair; e.g. 1024 x 1024 at mu = 2 needs ~16.5 MiB).
 *   - Every call looks up the array's device address (cudaGetSymbolAddress, with
 *     the caller's device current), so the address stays right after a
 *     cudaDeviceReset.  The first call on a device may load the library's device
 *     code there: make that first call before any stream capture on the device.
 *   - The call is synchronous: it waits for `stream` before returning, because
 *     the return code carries the device status (also when it fails after
 *     queueing work on the array).
 *   - All calls share the one array and it keeps the previous call's contents
 *     (each call clears what must start at zero).  Calls that overlap on the GPU
 *     (e.g. on two streams, or from two host threads) race and corrupt each
 *     other: serialise them.
 *   - externd_last_stats is not updated by this call (it records no events).
 * Arguments and results are those of externd_factor. */
#define EXTERND_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int externd_factor_noalloc(const float* A, int64_t m, int64_t n, double mu, double tau, int iters,
                           uint64_t seed, uint8_t* B_out, float* D_out, uint8_t* C_out,
                           double* energy_out, void* stream);

/* Factor `count` independent matrices in one cooperative launch; the SMs are
 * split into groups and each group factors its matrices one after another.
 * Every array argument has `count` entries (host arrays of pointers/values);
 * energy_out may be NULL or hold NULL entries.  status_out[b] receives the
 * status of matrix b; the return value is EXTERND_OK if all succeeded, else
 * the first failing status (argument errors are reported before any work). */
int externd_factor_batched(int count, const float* const* A, const int64_t* m, const int64_t* n,
                           const double* mu, const double* tau, int iters, const uint64_t* seed,
                           uint8_t* const* B_out, float* const* D_out, uint8_t* const* C_out,
                           double* const* energy_out, int* status_out, void* stream);

/* Per-matrix extensions of a batched call (zero-initialise, set what is needed).
 *   h         NULL, or `count` pointers to per-column importance weights (n_b fp32 values each):
 *             the §2.5 objective ("ExTernD: Expanded-Rank Ternary Decomposition", §2.5, see
 *             externd_factor_weighted).  One launch runs one objective, so either every entry is
 *             non-NULL or h is NULL (EXTERND_EINVAL otherwise).
 *   lambda    with h: `count` values of lambda (finite, >= 0); NULL means 0 for every matrix.
 *   sweeps    refinement sweeps after extraction for every matrix (§2.4, see externd_options),
 *             0 .. 1000.
 *   sweep_energy_out  NULL, or `count` pointers (entries may be NULL) to `sweeps` doubles each.
 *   grid      CTAs per matrix (0: automatic), as externd_options.grid.
 *   cluster   kernel choice, as externd_options.cluster.
 *   block     threads per CTA, as externd_options.block.  A matrix gets the same bits from
 *             any launch with the same grid, cluster size and block size -- e.g. one slice of a
 *             batch per GPU, run with the plan of the whole batch.
 *   plan_only nonzero: validate the arguments, choose the launch (CTAs per matrix, cluster
 *             size, lazy-deflation depth, threads per CTA) exactly as the call would, record it
 *             for externd_last_stats (grid, group, cluster, pending, block, smem_bytes) and
 *             return without device work. */
typedef struct {
    const float* const* h;
    const double* lambda;
    int sweeps;
    double* const* sweep_energy_out;
    int grid;
    int cluster;
    int plan_only;
    int* async_status;   /* as externd_options.async_status: one status for the whole batch
                          * (the first matrix's failure, else EXTERND_OK) */
    int block;
} externd_batch_options;

/* externd_factor_batched with per-matrix extensions (opt may be NULL: the plain call). */
int externd_factor_batched_ex(int count, const float* const* A, const int64_t* m, const int64_t* n,
                              const double* mu, const double* tau, int iters, const uint64_t* seed,
                              uint8_t* const* B_out, float* const* D_out, uint8_t* const* C_out,
                              double* const* energy_out, int* status_out, void* stream,
                              const externd_batch_options* opt);

/* Batched block ALS with decorrelated targets ("ExTernD: Expanded-Rank Ternary Decomposition",
 * §2.4 "Batched block ALS"): components in blocks of b,
 *   V <- T_tau([(U^T U + eps I)^-1 U^T R]^T),  U <- T_tau(R V (V^T V + eps I)^-1)  column-wise,
 * `iters` times from the start vectors of the block's components (those of externd_factor, so
 * b = 1 is the sequential method), then the joint scales [(U^T U) o (V^T V)] d = diag(U^T R V)
 * and R <- R - U diag(d) V^T; blocks follow each other sequentially.  The pages leave eps open:
 * here eps = 1e-6 x the mean diagonal of the Gram matrix.  The residual is held in fp64.
 *   b          block width; 0 = the pages' default, 256 capped at floor(min(m, n) / 8).
 *   energy_out [out] nullable; k doubles: E after the block holding component i.
 *   d64_out    [out] nullable; k fp64 scales.
 * A and all outputs are DEVICE pointers (EXTERND_EINVAL otherwise).  Other arguments and the
 * output formats are those of externd_factor.  EXTERND_ELIMIT if a block's joint scale system is
 * not positive definite (a component repeated within a block) or the shape exceeds 32-bit
 * element indices.  Synchronous; allocates about 8 m n + 8 b (3 m + 2 n) bytes of stream-ordered
 * workspace.  The plain fp64 GEMMs and the b x b Cholesky factorizations and solves run in
 * cuBLAS / cuSOLVER (the V-step's solve is applied to U's m rows, R^T [U (U^T U + eps I)^-1],
 * which equals the pages' form), through handles the call creates and destroys itself. */
int externd_factor_block(const float* A, int64_t m, int64_t n, double mu, double tau, int iters,
                         uint64_t seed, int b, uint8_t* B_out, float* D_out, uint8_t* C_out,
                         double* energy_out, double* d64_out, void* stream);

/* Ahat = B diag(D) C (§2.1) with fp64 accumulation, written as fp32 m x n
 * row-major.  B, C packed as produced by externd_factor. */
int externd_reconstruct(const uint8_t* B, const float* D, const uint8_t* C, int64_t m, int64_t n,
                        int64_t k, float* A_hat_out, void* stream);

/* ---------------------------------------------------------------------------
 * Inference with the factors (§2.6 Cost model: y = B (diag(D) (C x)), k (m + n)
 * ternary add/subtracts plus k multiplies) and mask+sign storage (§2.6 Eq. 1).
 * All pointers are DEVICE pointers (EXTERND_EINVAL otherwise); trit rows are
 * in the 2-bit format above.
 * ------------------------------------------------------------------------- */

/* Transpose a matrix of trits: T has `rows` rows of `len` trits (row stride
 * externd_trit_bytes(len)); Tt_out receives `len` rows of `rows` trits (row stride
 * externd_trit_bytes(rows)), Tt[j][r] = T[r][j].  Used once per factorization to
 * lay B out for inference: externd_transpose_trits(B_out, k, m, Bt) gives Bt with
 * row r = B[r, 0..k).  Synchronous; returns EXTERND_OK or a negative status. */
int externd_transpose_trits(const uint8_t* T, int64_t rows, int64_t len, uint8_t* Tt_out, void* stream);

/* Y[b] = B diag(D) C X[b] for b < batch (§2.6).
 *   Bt      [in]  m rows x externd_trit_bytes(k): B transposed (externd_transpose_trits).
 *   D       [in]  k fp32 scales.
 *   C       [in]  k rows x externd_trit_bytes(n), as returned by externd_factor.
 *   X       [in]  batch x n fp32, row-major (one input vector per row).
 *   Y       [out] batch x m fp32, row-major.
 *   z_work  [tmp] k x min(batch, 8) fp32 scratch owned by the caller (C x per vector).
 * Bt and C must be 16-byte aligned (EXTERND_EINVAL otherwise); the padding trits of their rows
 * (past k and n) are ignored.
 * fp32 arithmetic; stream-ordered and asynchronous (no allocation, no host sync). */
int externd_matvec(const uint8_t* Bt, const float* D, const uint8_t* C, int64_t m, int64_t n, int64_t k,
                   const float* X, int64_t batch, float* Y, float* z_work, void* stream);

/* Mask+sign storage of trit rows (§2.6): one zero/nonzero bit per element and
 * one sign bit (1 = negative) per nonzero element.
 *   T                [in]  rows x externd_trit_bytes(len) 2-bit trits.
 *   mask_out         [out] rows x ceil(len / 8) bytes; bit j % 8 of byte j / 8 of
 *                          row r is T[r][j] != 0.
 *   sign_out         [out] one bit stream of sign_words 32-bit words: the signs of
 *                          row r's nonzeros, in order, start at bit
 *                          sign_offsets_out[r] (bit b = bit b % 32 of word b / 32).
 *   sign_offsets_out [out] rows + 1 int64; the last entry is the total number of
 *                          nonzeros.  EXTERND_ELIMIT if they need more than
 *                          sign_words words.
 * Synchronous (allocates a small stream-ordered buffer). */
int externd_pack_mask_sign(const uint8_t* T, int64_t rows, int64_t len, uint8_t* mask_out, uint32_t* sign_out,
                           int64_t sign_words, int64_t* sign_offsets_out, void* stream);

/* Human-readable message for a status code (static storage). */
const char* externd_strerror(int status);

/* Test hook: ONE half-step of §2.3 step 1 on a caller-given residual, run by
 * the same kernel code as externd_factor.
 *   R          [in]  m x n fp32 row-major.
 *   transpose        1: V-step x = R^T u (in_trits has m trits, outputs n);
 *                    0: U-step y = R v   (in_trits has n trits, outputs m).
 *   in_trits   [in]  packed trits (externd_trit_bytes(len_in) bytes).
 *   tau              T_tau scale.
 *   pre_out    [out] fp64 pre-threshold vector (len_out).
 *   thresh_out [out] one double: tau * mean |pre|.
 *   out_trits  [out] packed T_tau(pre) (externd_trit_bytes(len_out) bytes). */
int externd_debug_halfstep(const float* R, int64_t m, int64_t n, int transpose,
                           const uint8_t* in_trits, double tau, double* pre_out,
                           double* thresh_out, uint8_t* out_trits, void* stream);

/* Test hook: the packed start trits u0_i = T_tau(z_i) of components
 * i = 0..k-1 for a matrix with m rows (see conventions), as used by
 * externd_factor.  out: k rows x externd_trit_bytes(m) bytes. */
int externd_debug_start_trits(int64_t m, int64_t k, double tau, uint64_t seed, uint8_t* out,
                              void* stream);

/* Test hook: ONE component of §2.3 (15 alternating fits, scale) run by the kernel of
 * externd_factor on a caller-given residual state, with a trace of every half-step.
 *   R          [in]  m x n fp32 row-major: the residual as stored (device or host).
 *   u0         [in]  packed start trits of the component (externd_trit_bytes(m) bytes).
 *   n_pend           0 .. 31 rank-1 terms d_j u_j v_j^T held pending, i.e. applied as the
 *                    corrections the factorization uses for deflations not yet folded into R:
 *                    the component is fitted to R - sum_j d_j u_j v_j^T.  EXTERND_ELIMIT above
 *                    the lazy-deflation depth of the launch minus one.
 *   pend_d     [in]  n_pend fp64 scales; pend_u [in] n_pend rows of externd_trit_bytes(m);
 *                    pend_v [in] n_pend rows of externd_trit_bytes(n) (DEVICE pointers).
 *   pre_v, thr_v, trit_v, pre_u, thr_u, trit_u  [out]  the trace of externd_options with
 *                    trace_count = 1 (DEVICE pointers).
 *   D_out, d64_out   [out] the scale d in fp32 and fp64; u_out, v_out [out] the final trits.
 *   grid             CTAs serving the matrix (0 = the factorization's automatic choice).
 * Returns EXTERND_OK or a negative externd_status. */
int externd_debug_component(const float* R, int64_t m, int64_t n, double tau, int iters, const uint8_t* u0,
                            int n_pend, const double* pend_d, const uint8_t* pend_u, const uint8_t* pend_v,
                            double* pre_v, double* thr_v, uint8_t* trit_v, double* pre_u, double* thr_u,
                            uint8_t* trit_u, float* D_out, double* d64_out, uint8_t* u_out, uint8_t* v_out,
                            int grid, void* stream);

/* Knobs and extra outputs for externd_factor_ex.  Zero-initialise and set
 * only what is needed. */
typedef struct {
    int grid;              /* CTAs per matrix; 0 = automatic */
    int pending;           /* deflations held as rank-1 vector corrections before being folded into R; 0 = automatic */
    double wait_limit_s;   /* limit of each device-side wait, seconds; 0 = 2.0 */
    int fault_skip_cta;    /* test hook, used only if fault_inject != 0: this CTA never signals */
    int fault_inject;
    double* d64_out;       /* nullable: k fp64 scales */
    /* Refinement sweeps ("ExTernD: Expanded-Rank Ternary Decomposition", §2.4, "Refinement
     * sweeps"), blocks of one component: after extraction every component i is revisited
     * `sweeps` times in order: its term d_i u_i v_i^T is added back to the residual, refitted
     * by the same alternation started from the stored u_i, and re-deflated.  The refit
     * replaces the stored component only if its least-squares decrease of the added-back
     * residual is at least that of the stored pair with its least-squares scale; otherwise
     * the stored trits stay with that scale.  Every visit is therefore non-increasing in
     * ||R||.  energy_out keeps the extraction energies; D/B/C hold the refined factors.
     * Needs a lazy-deflation depth of at least 2 (EXTERND_ELIMIT otherwise). */
    int sweeps;                /* 0 = none; at most 1000 */
    double* sweep_energy_out;  /* nullable: `sweeps` doubles, the energy after each sweep */
    /* Importance weights of §2.5 (see externd_factor_weighted); h = NULL: plain objective. */
    const float* h;
    double lambda;
    /* Test hook: a trace of visits [trace_first, trace_first + trace_count) of this
     * factorization, written by the kernel that computes it.  Visit i < k is the extraction of
     * component i; with refinement sweeps, visit (s + 1) k + i is sweep s's refit of component i
     * (a refit that reaches a fixed point stops early and leaves its later rows unwritten).
     * For every V-step (x = R^T u, §2.3 step 1) and U-step (y = R v) of a traced visit it stores
     * the output vector exactly
     * as the threshold saw it (after the corrections of deflations not yet folded into R, rounded
     * to the 44 significant bits the kernel exchanges), the threshold tau * mean |.| and the
     * resulting trits.  DEVICE pointers; trace_pre_v = NULL turns the trace off.  The window must
     * lie inside [0, k (1 + sweeps)), trit rows 16-byte aligned (EXTERND_EINVAL otherwise).
     *   trace_pre_v  [trace_count][iters][n] fp64     trace_pre_u  [trace_count][iters][m] fp64
     *   trace_thr_v  [trace_count][iters] fp64        trace_thr_u  [trace_count][iters] fp64
     *   trace_trit_v [trace_count][iters] rows of externd_trit_bytes(n)
     *   trace_trit_u [trace_count][iters] rows of externd_trit_bytes(m) */
    int64_t trace_first;
    int64_t trace_count;
    double* trace_pre_v;
    double* trace_thr_v;
    uint8_t* trace_trit_v;
    double* trace_pre_u;
    double* trace_thr_u;
    uint8_t* trace_trit_u;
    /* Kernel choice: 0 = automatic (currently the one-CTA-per-stripe kernel); 1 = one CTA per
     * residual stripe (the kernel that also runs refinement sweeps); 2, 4, 8 or 16 = the
     * clustered kernel with clusters of that many CTAs, for factorizations without sweeps
     * (EXTERND_ELAUNCH if they cannot all be resident, EXTERND_EINVAL for other values).
     * Results depend on the partition: the same grid, cluster size and block size give the
     * same bits. */
    int cluster;
    /* Asynchronous call: non-NULL = a DEVICE int.  The call queues all its work on `stream` and
     * returns EXTERND_OK without waiting; when the stream reaches the end of the work, the
     * int receives the factorization's status (EXTERND_OK or a negative EXTERND_* code, e.g.
     * EXTERND_ETIMEOUT).  A, the outputs and every optional buffer must be device memory
     * (EXTERND_EINVAL otherwise: host buffers would need a synchronous copy).  The workspace
     * is released in stream order.  A non-OK return means nothing was left queued (the call
     * waited for what it had queued).  externd_last_stats records the plan only (timings,
     * byte counts and safeguard counts are 0). */
    int* async_status;
    /* Threads per CTA of the one-CTA-per-stripe kernel: 0 = automatic, else 256, 512 or 1024
     * (EXTERND_EINVAL otherwise; the clustered kernel runs at 512 only, so with cluster > 1
     * only 0 and 512 are accepted).  The automatic choice follows the work one CTA does per
     * half-step, W = m n / G + 8 (m + n) for G CTAs per matrix (the largest matrix of a batch):
     * its share of the residual plus the two vectors it thresholds.  256 below W = 170000 (512
     * with refinement sweeps, whose refits are faster there), 512 up to 230000, 1024 above --
     * unless the 1024-thread plan, which keeps more shared state per CTA, would leave a
     * lazy-deflation depth below 8 (the largest shapes), where 512 is kept.  The block size sets how the fp64 sums inside a CTA are split
     * across warps, so, as with the partition, only the same grid, cluster size and block
     * size are guaranteed to give the same bits. */
    int block;
} externd_options;

/* externd_factor with options (opt may be NULL). */
int externd_factor_ex(const float* A, int64_t m, int64_t n, double mu, double tau, int iters,
                      uint64_t seed, uint8_t* B_out, float* D_out, uint8_t* C_out,
                      double* energy_out, void* stream, const externd_options* opt);

/* Figures of the last call made by this host thread. */
typedef struct {
    double als_ms;             /* device time of the cooperative ALS kernel (CUDA events) */
    double setup_ms;           /* residual layout copy + ||A||^2 */
    double init_ms;            /* start-vector generation */
    double total_ms;           /* all device work of the call, staging copies included */
    double alg_bytes;          /* algorithmic bytes of the ALS kernel, summed over matrices: per component
                                  4 (n sum_t nnz(u_t) + m sum_t nnz(v_t)) + 8 nnz(u) nnz(v), t over the
                                  half-steps, i.e. what a direct evaluation of every GEMV touches */
    double read_bytes;         /* residual bytes this kernel reads: its GEMVs run over the trits that
                                  changed since the previous half-step of the same kind (4 (n rows +
                                  m columns) per half-step), plus the same deflation term */
    double residual_energy;    /* 1 - ||R_k||^2 / ||A||^2 from the final fp32 residual (matrix 0) */
    int64_t components;        /* components fitted, summed over matrices */
    int64_t half_steps;        /* V- and U-steps executed, summed over matrices */
    int64_t fallbacks;         /* T_tau all-zero fallbacks taken */
    int launches;              /* kernels launched by the call */
    int grid;                  /* CTAs of the ALS launch */
    int group;                 /* CTAs per matrix */
    int block;                 /* threads per CTA */
    int vec_v, vec_u;          /* vector width of the two residual layouts */
    int pending;               /* lazy-deflation depth used */
    size_t smem_bytes;         /* dynamic shared memory per CTA */
    size_t workspace_bytes;
    int64_t sweep_kept;        /* refinement visits that kept the stored pair (matrix 0) */
    int64_t phase_cycles[11];  /* [10]: exchanged words found not yet visible by CTA 0; [0..9]: SM cycles of CTA 0 of matrix 0 (diagnostics): GEMV loads, GEMV reduce +
                                  emit, publish, wait, partials + first loads, threshold, compaction,
                                  start vector, output + pending push, deflation fold */
    int64_t safeguard_hits;    /* extraction components whose ALS decrease p^2 / (nnz(u) nnz(v)) fell below the
                                  single-entry bound ||R||^2 / (m n) of §7 ("Monotone residual decrease and
                                  convergence"), summed over matrices; counted only, no component is replaced */
    int cluster;               /* CTAs per cluster of the ALS launch (1: the one-CTA-per-stripe kernel) */
    int reserved;
} externd_stats;

int externd_last_stats(externd_stats* out);

#ifdef __cplusplus
}
#endif

#endif /* EXTERND_H */
