// Device code of the ExTernD greedy sequential ALS library (sm_100a).
//
// Method: "ExTernD: Expanded-Rank Ternary Decomposition" (arXiv 2607.13511)
// §2.2 (T_tau) and §2.3 (greedy sequential ALS: alternating ternary fits,
// closed-form scale, rank-1 deflation).
//
// Design (B200):
//  * One persistent cooperative launch runs every component of a matrix.  A
//    matrix is served by a group of G CTAs, one per SM, of NT threads each.  NT is a
//    compile-time constant (EXTERND_NT: 256, 512 or 1024); the library compiles this
//    code at all three and the host picks one per launch by the work of one CTA.
//    Fewer threads shorten the barrier-bound half-step and leave more registers per
//    thread (255 at 256 threads: no spills; 128 at 512 and 64 at 1024: the fp64 sums
//    spill); more threads pay once a CTA's share of the residual is large.
//  * The residual R is kept twice in HBM, each copy cut into one private block
//    per CTA so that both half-steps read only what they need and no CTA ever
//    reads another CTA's residual:
//      V-layout: CTA q owns a stripe of columns [c0, c1) of R, stored as an
//                m x pitch row-major block.  V-step x = R^T u reads only the
//                rows r with u_r != 0 and produces x over its own columns.
//      U-layout: CTA q owns a stripe of rows [r0, r1) of R, stored as an
//                n x pitch block (column c of R restricted to the stripe is
//                contiguous).  U-step y = R v reads only the columns with
//                v_c != 0 and produces y over its own rows.
//    So each half-step needs no cross-CTA reduction of vectors, only the
//    scalar sum of |x| for the threshold: every CTA publishes its slice of the
//    output and its partial sum, meets the others at one counter, then reads
//    the whole vector back and thresholds it itself (all CTAs derive the
//    identical trit vector because they use the same data in the same order).
//  * Incremental GEMVs: within a component R is fixed, so each CTA keeps the
//    running sums g = R^T u (its columns) and R v (its rows) in shared memory
//    and each half-step reads only the rows (columns) whose trit changed since
//    the previous half-step of the same kind: g += R^T (u_new - u_old), with
//    coefficients +-1 or +-2.  The first half-steps of a component start from
//    g = 0 and the whole support.  After the first few fits only a few percent
//    of the trits change per fit, so most half-steps read a small part of R.
//  * Deflation is lazy: the last L components (d_j, u_j, v_j) are held as
//    bit masks in shared memory and applied as rank-1 corrections to each
//    GEMV output (x -= sum_j d_j (u_j . u) v_j, the integer dot products kept
//    up to date from the changed trits); every L components each CTA folds
//    them into its own two blocks in one pass.  Each residual entry is held as
//    an fp32 pair hi + lo: a fold computes hi + lo - sum_j ... in fp64 and
//    splits the result again, so the pair tracks the exact residual to ~2^-48
//    of its magnitude however many folds it went through, and the GEMVs read
//    hi alone, which is within 2^-24 of the current residual entry (a plain
//    fp32 residual would keep the rounding errors of early folds, made at the
//    scale of A, while the residual shrinks).
//  * Accumulation: every signed fp32 residual entry is added to an fp64 sum
//    (each term is exact in fp64, each add rounds once), and the threshold
//    decisions are taken on fp64 values like the oracle.
//  * Every device-side wait is bounded by %globaltimer; a wait that runs out
//    raises a status word and the kernel returns.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace externd {

#ifndef EXTERND_NT
#define EXTERND_NT 512
#endif
constexpr int NT = EXTERND_NT;        // threads per CTA of the ALS kernel
constexpr int NWARP = NT / 32;
constexpr int MAX_PENDING = 32;       // lazy deflation depth cap
constexpr unsigned FULL = 0xffffffffu;

// Status codes written by kernels (mirror externd_status).
constexpr int ST_OK = 0;
constexpr int ST_EINVAL = -1;
constexpr int ST_EZERO = -2;
constexpr int ST_ENONFINITE = -3;
constexpr int ST_ETIMEOUT = -7;
constexpr int ST_RUNNING = 1;         // set by the host before launch

// Balanced split of `len` indices into G stripes made of `vec`-wide units.
struct Part {
    int64_t len;
    int64_t units;    // ceil(len / vec)
    int vec;
    int G;
    __host__ __device__ int64_t ustart(int q) const { return ((int64_t)q * units) / G; }
    __host__ __device__ int64_t start(int q) const { int64_t s = ustart(q) * vec; return s < len ? s : len; }
    __host__ __device__ int64_t end(int q) const { int64_t e = ustart(q + 1) * vec; return e < len ? e : len; }
    __host__ __device__ int pitch(int q) const { return (int)((ustart(q + 1) - ustart(q)) * vec); }
    // stripe holding index i: the largest q with ustart(q) <= i / vec
    __host__ __device__ int owner(int64_t i) const {
        int64_t u = i / vec;
        return (int)(((u + 1) * (int64_t)G - 1) / units);
    }
    // element offset of stripe q's block when the other dimension has `other` entries
    __host__ __device__ int64_t block_offset(int q, int64_t other) const { return other * vec * ustart(q); }
    __host__ __device__ int64_t total(int64_t other) const { return other * vec * units; }
};

// 2-D partition of one matrix.
struct Grid2 {
    int64_t m, n;
    int c, NC, vecv, vecu;
    __host__ __device__ static Part mk(int64_t len, int G, int vec) {
        Part p;
        p.len = len;
        p.vec = vec;
        p.G = G;
        p.units = (len + vec - 1) / vec;
        return p;
    }
    __host__ __device__ Part qr() const { return mk(m, c, 32); }      // row quarters
    __host__ __device__ Part qc() const { return mk(n, c, 32); }      // column quarters
    // pieces of column quarter s (V-step outputs) and of row quarter s (U-step outputs)
    __host__ __device__ Part pcol(int s) const { const Part Q = qc(); return mk(Q.end(s) - Q.start(s), NC, vecv); }
    __host__ __device__ Part prow(int s) const { const Part Q = qr(); return mk(Q.end(s) - Q.start(s), NC, vecu); }
    // offset of piece (q, s) inside cluster q's stripe, and the stripe's width
    __host__ __device__ int soffV(int q, int s) const {
        int o = 0;
        for (int t = 0; t < s; ++t) o += pcol(t).pitch(q);
        return o;
    }
    __host__ __device__ int soffU(int q, int s) const {
        int o = 0;
        for (int t = 0; t < s; ++t) o += prow(t).pitch(q);
        return o;
    }
    __host__ __device__ int pitchV(int q) const { return soffV(q, c); }
    __host__ __device__ int pitchU(int q) const { return soffU(q, c); }
};

constexpr int NCTR = 8;       // arrival counters per group (spread over L2 lines)

struct GroupSync {            // one per CTA group
    int abort;                // raised by the first wait of the group that runs out
    int pad[63];
    unsigned ctr[NCTR][64];   // counter c (one per 256 B) counts arrivals of the CTAs q with q % NCTR == c
};

struct DevStats {
    unsigned long long sum_nu;      // sum of nnz(u) over V-steps (rows a direct evaluation reads)
    unsigned long long sum_nv;      // sum of nnz(v) over U-steps
    unsigned long long sum_du;      // rows read by V-steps (trit changes of u)
    unsigned long long sum_dv;      // columns read by U-steps (trit changes of v)
    unsigned long long sum_nunv;    // sum nnz(u_i) nnz(v_i)
    unsigned long long half_steps;
    unsigned long long fallbacks;
    double residual2;               // ||R_k||^2 from the final fp32 residual
    double norm_a2;
    double pad;
    unsigned long long phase[11];   // SM cycles of CTA 0 per phase (see run_problem); [10] stale words seen
    unsigned long long sweep_kept;  // refinement visits that kept the stored pair (rescaled)
    unsigned long long safeguard;   // components whose ALS decrease fell below ||R||^2 / (m n)
};

enum Mode { MODE_FACTOR = 0, MODE_HALF_V = 1, MODE_HALF_U = 2 };

struct Prob {
    const float* A;
    const float* hw;          // importance weights h~ (n, fp32) of §2.5, or null for the plain objective
    int64_t m, n, k;
    double tau;
    int iters;
    int mode;
    uint64_t seed;
    uint8_t* B;               // k rows of b_bytes
    float* D;
    uint8_t* C;               // k rows of c_bytes
    double* energy;           // nullable
    double* d64;              // nullable
    int sweeps;               // §2.4 refinement sweeps after extraction (0 = none)
    double* dk;               // k fp64 scales every CTA re-reads during sweeps (workspace; null without sweeps)
    double* sweep_energy;     // nullable: energy after each sweep
    int64_t b_bytes, c_bytes;
    float* Rv;                // V-layout blocks
    float* Ru;                // U-layout blocks
    float* Rv_lo;             // low halves of the V-layout residual: R = Rv + Rv_lo (see the fold)
    float* Ru_lo;             // low halves of the U-layout residual
    unsigned long long* xbuf; // n, published V-step outputs (tagged fp64 words, zero-initialised)
    unsigned long long* ybuf; // m, published U-step outputs (tagged fp64 words, zero-initialised)
    unsigned long long* sums; // 2 G, per-CTA partial sums, double-buffered by use (tagged, zero-initialised)
    unsigned long long* partV;// G, per-CTA sum |out| of the V-step (tagged, zero-initialised)
    unsigned long long* partU;// G, same for the U-step
    const uint32_t* start;    // start trits (k rows of start_words) or debug input (1 row)
    int64_t start_words;
    double* norm_part;        // per setup-tile partial sums of A^2
    int64_t n_norm_part;
    unsigned* nonfinite;
    int* status;
    DevStats* stats;
    int start_given;          // 1: the start trits were supplied by the caller (no generated start vector)
    int n_pend;               // pending rank-1 terms supplied by the caller, applied before component 0
    const double* pend_d;     // their scales (n_pend)
    const uint32_t* pend_u;   // their u trits (n_pend rows of b_bytes)
    const uint32_t* pend_v;   // their v trits (n_pend rows of c_bytes)
    int64_t tr_first, tr_count;   // traced visits [tr_first, tr_first + tr_count): components 0 .. k-1, then
                                  // sweep s revisits component i as visit (s + 1) k + i
    double* tr_pre_v;         // [tr_count][iters][n] published V-step outputs
    double* tr_thr_v;         // [tr_count][iters]
    double* tr_pre_u;         // [tr_count][iters][m] published U-step outputs
    double* tr_thr_u;         // [tr_count][iters]
    uint8_t* tr_trit_v;       // [tr_count][iters] rows of c_bytes: the V-step trits
    uint8_t* tr_trit_u;       // [tr_count][iters] rows of b_bytes: the U-step trits
    double* pre_out;          // debug half-step outputs
    double* thr_out;
    uint8_t* trit_out;
    Part pv;                  // column stripes (len n)
    Part pu;                  // row stripes (len m)
    Grid2 g2;                 // clustered kernel: 2-D partition over the group's clusters
    int64_t bsv, bsu;         // clustered kernel: elements per CTA block of the V- and U-layout
};

struct KCfg {
    const Prob* probs;
    int nprob;
    int Gg;                   // CTAs per group
    int NG;                   // groups
    GroupSync* gsync;         // NG
    int Lcap;                 // lazy deflation depth
    int m_max, n_max;         // for shared-memory carving
    int pv_max, pu_max;       // largest stripe pitch of the two layouts
    uint64_t limit_ns;
    int fault_skip;           // CTA rank (within group) that never arrives; -1 = off
    int weighted;             // problems carry importance weights (single-matrix launches only)
    int qr_max, qc_max;       // clustered kernel: longest row / column quarter
    int wpm;                  // clustered kernel: widest output piece (pitch)
};

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint64_t gtimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ int ld_relaxed_s32(const int* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// bits 0,2,4,...,30 of x -> bits 0..15
__host__ __device__ __forceinline__ uint32_t compact_even(uint32_t x) {
    x &= 0x55555555u;
    x = (x | (x >> 1)) & 0x33333333u;
    x = (x | (x >> 2)) & 0x0F0F0F0Fu;
    x = (x | (x >> 4)) & 0x00FF00FFu;
    x = (x | (x >> 8)) & 0x0000FFFFu;
    return x;
}

// bits 0..15 of x -> bits 0,2,...,30
__host__ __device__ __forceinline__ uint32_t spread_even(uint32_t x) {
    x &= 0x0000FFFFu;
    x = (x | (x << 8)) & 0x00FF00FFu;
    x = (x | (x << 4)) & 0x0F0F0F0Fu;
    x = (x | (x << 2)) & 0x33333333u;
    x = (x | (x << 1)) & 0x55555555u;
    return x;
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }
__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }

// Block-wide fp64 sum with a fixed combination order (same inputs -> same bits).
__device__ __forceinline__ double block_sum(double v, double* sh) {
    #pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
    if (lane_id() == 0) sh[warp_id()] = v;
    __syncthreads();
    if (warp_id() == 0) {
        double w = lane_id() < NWARP ? sh[lane_id()] : 0.0;
        #pragma unroll
        for (int o = 16; o; o >>= 1) w += __shfl_xor_sync(FULL, w, o);
        if (lane_id() == 0) sh[NWARP] = w;
    }
    __syncthreads();
    double r = sh[NWARP];
    __syncthreads();
    return r;
}

// max |.| with the lowest index on ties
__device__ __forceinline__ void maxloc_merge(double& m, long long& j, double m2, long long j2) {
    if (m2 > m || (m2 == m && j2 < j)) { m = m2; j = j2; }
}

__device__ __forceinline__ void block_maxloc(double& m, long long& j, double* shm, long long* shj) {
    #pragma unroll
    for (int o = 16; o; o >>= 1) {
        double m2 = __shfl_xor_sync(FULL, m, o);
        long long j2 = __shfl_xor_sync(FULL, j, o);
        maxloc_merge(m, j, m2, j2);
    }
    if (lane_id() == 0) { shm[warp_id()] = m; shj[warp_id()] = j; }
    __syncthreads();
    if (warp_id() == 0) {
        double mm = lane_id() < NWARP ? shm[lane_id()] : -1.0;
        long long jj = lane_id() < NWARP ? shj[lane_id()] : (long long)0x7fffffffffffffffLL;
        #pragma unroll
        for (int o = 16; o; o >>= 1) {
            double m2 = __shfl_xor_sync(FULL, mm, o);
            long long j2 = __shfl_xor_sync(FULL, jj, o);
            maxloc_merge(mm, jj, m2, j2);
        }
        if (lane_id() == 0) { shm[NWARP] = mm; shj[NWARP] = jj; }
    }
    __syncthreads();
    m = shm[NWARP];
    j = shj[NWARP];
    __syncthreads();
}

// Exclusive scan of a[0..W) in place; returns the total.  sh: NWARP+1 ints.
__device__ int block_exclusive_scan(int* a, int W, int* sh) {
    const int per = (W + NT - 1) / NT;
    const int b = threadIdx.x * per;
    const int e = min(W, b + per);
    int s = 0;
    for (int i = b; i < e; ++i) s += a[i];
    int incl = s;
    #pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(FULL, incl, o);
        if (lane_id() >= o) incl += t;
    }
    if (lane_id() == 31) sh[warp_id()] = incl;
    __syncthreads();
    if (warp_id() == 0) {
        int v = lane_id() < NWARP ? sh[lane_id()] : 0;
        int inc = v;
        #pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_up_sync(FULL, inc, o);
            if (lane_id() >= o) inc += t;
        }
        if (lane_id() < NWARP) sh[lane_id()] = inc - v;
        if (lane_id() == NWARP - 1) sh[NWARP] = inc;
    }
    __syncthreads();
    int run = sh[warp_id()] + incl - s;
    for (int i = b; i < e; ++i) { int c = a[i]; a[i] = run; run += c; }
    const int total = sh[NWARP];
    __syncthreads();
    return total;
}

// ---------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11) and Box-Muller start normals
// ---------------------------------------------------------------------------

__device__ __forceinline__ void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
    #pragma unroll
    for (int r = 0; r < 10; ++r) {
        if (r > 0) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
        const uint32_t hi0 = __umulhi(0xD2511F53u, c[0]);
        const uint32_t lo0 = 0xD2511F53u * c[0];
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c[2]);
        const uint32_t lo1 = 0xCD9E8D57u * c[2];
        const uint32_t n0 = hi1 ^ c[1] ^ k0;
        const uint32_t n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
    }
}

__device__ __forceinline__ double start_normal(uint64_t seed, uint32_t comp, uint32_t j) {
    uint32_t c[4] = {j, comp, 1u, 0u};
    philox4x32_10(c, (uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32));
    const uint64_t w1 = ((uint64_t)c[1] << 32) | c[0];
    const uint64_t w2 = ((uint64_t)c[3] << 32) | c[2];
    const double u1 = ((double)(w1 >> 11) + 0.5) * 0x1.0p-53;
    const double u2 = ((double)(w2 >> 11) + 0.5) * 0x1.0p-53;
    return sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
}

}  // namespace externd
