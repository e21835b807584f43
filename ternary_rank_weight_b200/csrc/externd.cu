// ExTernD greedy sequential ternary ALS for B200 (sm_100a): kernels + C ABI.
//
// Method: "ExTernD: Expanded-Rank Ternary Decomposition" (arXiv 2607.13511),
// §2.1 (factorization, energy), §2.2 (T_tau), §2.3 (greedy sequential ALS).
// The data layout and the synchronisation scheme are described at the top of
// externd_kernels.cuh.
#include <cooperative_groups.h>
#include <cublas_v2.h>
#include <cuda_runtime.h>
#include <cusolverDn.h>

#include <climits>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <vector>

#include "externd.h"
#include "externd_kernels.cuh"

#ifndef EXTERND_SECONDARY
// The ALS machinery of this file is compiled at three block sizes, each in its own namespace: 512
// threads per CTA here, 256 in externd_nt256.cu and 1024 in externd_nt1024.cu.  Every C-ABI entry
// point lives here; a plan whose block size is not 512 runs through the other build's run()
// (arguments as validated here; fixed_base/fixed_cap: the caller-fixed workspace or null).
int externd_run_nt256(const void* in, int np, const void* opt, cudaStream_t stream, int* statuses,
                      externd_stats* stats, void* fixed_base, size_t fixed_cap);
int externd_run_nt1024(const void* in, int np, const void* opt, cudaStream_t stream, int* statuses,
                       externd_stats* stats, void* fixed_base, size_t fixed_cap);
#endif

namespace externd {

// ---------------------------------------------------------------------------
// Setup: copy A into the two private-block layouts, ||A||^2 partials, NaN/Inf.
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(256) setup_kernel(const Prob* __restrict__ probs) {
    const Prob& P = probs[blockIdx.z];
    const int64_t m = P.m, n = P.n;
    const int64_t tiles_x = (n + 31) >> 5, tiles_y = (m + 31) >> 5;
    if ((int64_t)blockIdx.x >= tiles_x || (int64_t)blockIdx.y >= tiles_y) return;
    __shared__ float tile[32][33];
    __shared__ double red[9];
    const int64_t rbase = (int64_t)blockIdx.y * 32, cbase = (int64_t)blockIdx.x * 32;
    double ss = 0.0;
    unsigned bad = 0;
    for (int rr = threadIdx.y; rr < 32; rr += 8) {
        const int64_t r = rbase + rr, c = cbase + threadIdx.x;
        float v = 0.f;
        if (r < m && c < n) {
            v = __ldcg(P.A + r * n + c);
            if (!isfinite(v)) ++bad;
            ss += (double)v * (double)v * (P.hw ? (double)__ldg(P.hw + c) : 1.0);
            const int q = P.pv.owner(c);
            P.Rv[P.pv.block_offset(q, m) + r * P.pv.pitch(q) + (c - P.pv.start(q))] = v;
        }
        tile[rr][threadIdx.x] = v;
    }
    __syncthreads();
    for (int cc = threadIdx.y; cc < 32; cc += 8) {
        const int64_t c = cbase + cc, r = rbase + threadIdx.x;
        if (r < m && c < n) {
            const int p = P.pu.owner(r);
            P.Ru[P.pu.block_offset(p, n) + c * P.pu.pitch(p) + (r - P.pu.start(p))] = tile[threadIdx.x][cc];
        }
    }
    const int tid = threadIdx.y * 32 + threadIdx.x;
    #pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(FULL, ss, o);
    if ((tid & 31) == 0) red[tid >> 5] = ss;
    __syncthreads();
    if (tid == 0) {
        double s = 0.0;
        for (int w = 0; w < 8; ++w) s += red[w];
        P.norm_part[blockIdx.y * tiles_x + blockIdx.x] = s;
    }
    if (bad) atomicAdd(P.nonfinite, bad);
}

// ---------------------------------------------------------------------------
// Importance weights of §2.5: h~_j = h_j / max(h) + lambda, computed in fp64 and
// held in fp32.  h must be finite and non-negative with a positive maximum; a
// violation raises *bad (the factorization then reports EXTERND_EINVAL).
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(1024) weights_kernel(const float* __restrict__ h, int64_t n, double lambda,
                                                       float* __restrict__ hw, unsigned* bad) {
    __shared__ float smax[32];
    __shared__ int sbad[32];
    float mx = 0.f;
    int b = 0;
    for (int64_t j = threadIdx.x; j < n; j += 1024) {
        const float v = h[j];
        if (!(v >= 0.f) || !isfinite(v)) b = 1;
        else mx = fmaxf(mx, v);
    }
    #pragma unroll
    for (int o = 16; o; o >>= 1) {
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
        b |= __shfl_xor_sync(FULL, b, o);
    }
    if ((threadIdx.x & 31) == 0) { smax[threadIdx.x >> 5] = mx; sbad[threadIdx.x >> 5] = b; }
    __syncthreads();
    float M = 0.f;
    int B = 0;
    for (int w = 0; w < 32; ++w) { M = fmaxf(M, smax[w]); B |= sbad[w]; }
    if (B || !(M > 0.f) || !isfinite(lambda) || lambda < 0.0) {
        if (threadIdx.x == 0) *bad = 1u;
        return;
    }
    for (int64_t j = threadIdx.x; j < n; j += 1024) hw[j] = (float)((double)h[j] / (double)M + lambda);
}

// ---------------------------------------------------------------------------
// Start trits u0_i = T_tau(z_i) for every component (reading of §2.3: the pages
// start from an unspecified u; here a seeded Gaussian vector).
// ---------------------------------------------------------------------------

constexpr int NTI = 256;

__global__ void __launch_bounds__(NTI) init_kernel(const Prob* __restrict__ probs) {
    const Prob& P = probs[blockIdx.y];
    if (P.mode != MODE_FACTOR || P.start_given) return;
    const int64_t m = P.m;
    __shared__ double shd[NTI / 32 + 1];
    __shared__ double shm[NTI / 32 + 1];
    __shared__ long long shj[NTI / 32 + 1];
    uint32_t* start = const_cast<uint32_t*>(P.start);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t i = blockIdx.x; i < P.k; i += gridDim.x) {
        double s = 0.0, mx = -1.0;
        long long jx = LLONG_MAX;
        for (int64_t j = threadIdx.x; j < m; j += NTI) {
            const double a = fabs(start_normal(P.seed, (uint32_t)i, (uint32_t)j));
            s += a;
            if (a > mx) { mx = a; jx = j; }
        }
        #pragma unroll
        for (int o = 16; o; o >>= 1) {
            s += __shfl_xor_sync(FULL, s, o);
            const double m2 = __shfl_xor_sync(FULL, mx, o);
            const long long j2 = __shfl_xor_sync(FULL, jx, o);
            maxloc_merge(mx, jx, m2, j2);
        }
        if (lane == 0) { shd[warp] = s; shm[warp] = mx; shj[warp] = jx; }
        __syncthreads();
        if (threadIdx.x == 0) {
            double S = 0.0, M = -1.0;
            long long J = LLONG_MAX;
            for (int w = 0; w < NTI / 32; ++w) { S += shd[w]; maxloc_merge(M, J, shm[w], shj[w]); }
            shd[NTI / 32] = S;
            shj[NTI / 32] = J;
        }
        __syncthreads();
        const double thr = P.tau * shd[NTI / 32] / (double)m;
        const long long Jmax = shj[NTI / 32];
        int any = 0;
        uint32_t* row = start + i * P.start_words;
        for (int64_t w = threadIdx.x; w < P.start_words; w += NTI) {
            uint32_t word = 0;
            for (int e = 0; e < 16; ++e) {
                const int64_t j = w * 16 + e;
                if (j < m) {
                    const double z = start_normal(P.seed, (uint32_t)i, (uint32_t)j);
                    if (fabs(z) > thr) word |= (z < 0.0 ? 3u : 1u) << (2 * e);
                }
            }
            row[w] = word;
            any |= (word != 0u);
        }
        any = __syncthreads_or(any);
        if (!any && threadIdx.x == 0) {
            const double z = start_normal(P.seed, (uint32_t)i, (uint32_t)Jmax);
            row[Jmax >> 4] |= (z < 0.0 ? 3u : 1u) << (2 * (Jmax & 15));
        }
        __syncthreads();
    }
}

// ---------------------------------------------------------------------------
// ALS kernel pieces
// ---------------------------------------------------------------------------

// Stride of the per-warp partial dot products, [l * DSTR + warp]: odd, so a warp's
// lanes (l = lane) write and read distinct banks.
constexpr int DSTR = NWARP + 1;

// Shared-memory carve of the ALS kernel (host and device use the same layout).
struct SmemLayout {
    size_t red, pd, coef, coefV, dotU, dotV, scal, wS, wM, wp, gS, gM, wJ, gJ, wc, dotp, sflag, clk, nzU, sgU, nzV, sgV, pnzU, psgU, pnzV,
        psgV, cnzV, csgV, cnzU, csgU, ulist, vlist, vwl, wd, onzU, osgU, onzV, osgV, dotVw, dotpw, gV, gU, corr, total;
    __host__ __device__ SmemLayout(int64_t m_max, int64_t n_max, int Lc, int pv_max, int pu_max, int weighted) {
        const size_t Wm = (size_t)((m_max + 31) / 32), Wn = (size_t)((n_max + 31) / 32);
        size_t o = 0;
        red = o;  o += 8 * (size_t)NT * 5;   // lanes * (pitch + 1) <= NT * (VEC + 1)
        pd = o;   o += 8 * (size_t)Lc;
        coef = o; o += 8 * (size_t)Lc;
        coefV = o; o += 8 * (size_t)Lc;
        dotU = o; o += 4 * (size_t)Lc;
        dotV = o; o += 4 * (size_t)Lc;
        o = (o + 7) & ~(size_t)7;
        scal = o; o += 8 * 16;
        wS = o;   o += 8 * NWARP;
        wM = o;   o += 8 * NWARP;
        wp = o;   o += 8 * NWARP;
        gS = o;   o += 8 * NWARP;
        gM = o;   o += 8 * NWARP;
        wJ = o;   o += 8 * NWARP;
        gJ = o;   o += 8 * NWARP;
        wc = o;   o += 4 * NWARP;
        dotp = o; o += 4 * DSTR * MAX_PENDING;
        sflag = o; o += 16;
        clk = o;  o += 8 * 12;
        nzU = o;  o += 4 * Wm;
        sgU = o;  o += 4 * Wm;
        nzV = o;  o += 4 * Wn;
        sgV = o;  o += 4 * Wn;
        pnzU = o; o += 4 * Wm * Lc;
        psgU = o; o += 4 * Wm * Lc;
        pnzV = o; o += 4 * Wn * Lc;
        psgV = o; o += 4 * Wn * Lc;
        cnzV = o; o += 4 * (size_t)pv_max;
        csgV = o; o += 4 * (size_t)pv_max;
        cnzU = o; o += 4 * (size_t)pu_max;
        csgU = o; o += 4 * (size_t)pu_max;
        ulist = o; o += 4 * (size_t)m_max;
        vlist = o; o += 4 * (size_t)n_max;
        vwl = o;  o += weighted ? 4 * (size_t)n_max : 0;   // weighted list coefficients of the U-step
        wd = o;   o += 4 * NWARP;
        onzU = o; o += 4 * Wm;
        osgU = o; o += 4 * Wm;
        onzV = o; o += 4 * Wn;
        osgV = o; o += 4 * Wn;
        o = (o + 7) & ~(size_t)7;
        dotVw = o; o += weighted ? 8 * (size_t)MAX_PENDING : 0;
        dotpw = o; o += weighted ? 8 * (size_t)DSTR * MAX_PENDING : 0;
        gV = o;   o += 8 * (size_t)pv_max;
        gU = o;   o += 8 * (size_t)pu_max;
        corr = o; o += 8 * (size_t)(pv_max > pu_max ? pv_max : pu_max);
        total = (o + 15) & ~(size_t)15;
    }
};

struct Smem {
    double *red, *pd, *scal, *wS, *wM, *wp, *gS, *gM;          // red: NT*5
    double *coef, *coefV;                    // d_l (t_l . u) and d_l (t_l . v) for the pending components
    int *dotU, *dotV;                        // the integer dot products t_l . u and t_l . v
    long long *wJ, *gJ;
    int *wc, *dotp, *sflag;
    unsigned long long* clk;                 // [0..9] phase cycles, [11] last stamp (thread 0 of CTA 0)
    uint32_t *nzU, *sgU, *nzV, *sgV;         // current u, v
    uint32_t *pnzU, *psgU, *pnzV, *psgV;     // pending components (full length, stride W)
    uint32_t *cnzV, *csgV, *cnzU, *csgU;     // pending trits at this CTA's outputs, bit l = component l
    int *ulist, *vlist;                      // compacted trit changes: element offset (index * block pitch) | sign << 31 | (|delta| == 2) << 30
    float* vwl;                              // weighted objective: coefficient of each vlist entry, delta * h~_c
    double *dotVw, *dotpw;                   // weighted objective: sum_c h~_c t_l(c) v(c) per pending l; per-warp partials
    int* wd;                                 // per-warp count of changed trits
    uint32_t *onzU, *osgU, *onzV, *osgV;     // masks of the previous u and v of this component
    double *gV, *gU;                         // running GEMV sums R^T u, R v of this CTA's outputs (before lazy-deflation correction)
    double* corr;                            // lazy-deflation correction per output of this CTA
};

// Phase clock (diagnostics): thread 0 of the first CTA adds the cycles since its
// previous stamp to phase k.  A clock read and two shared-memory accesses.
__device__ __forceinline__ void phase_mark(unsigned long long* clk, int k) {
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        const unsigned long long t = (unsigned long long)clock64();
        clk[k] += t - clk[11];
        clk[11] = t;
    }
}
__device__ __forceinline__ void phase_mark(const Smem& s, int k) { phase_mark(s.clk, k); }

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// fp64 value with its 8 low mantissa bits replaced by a half-step tag (see the exchange below)
__device__ __forceinline__ unsigned long long tag_value(double v, unsigned tag) {
    return ((unsigned long long)__double_as_longlong(v) & ~0xFFull) | (unsigned long long)tag;
}

template <int VEC>
__device__ __forceinline__ void load_vec(const float* p, float* v) {
    if constexpr (VEC == 4) {
        const float4 t = __ldcg(reinterpret_cast<const float4*>(p));
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
    } else if constexpr (VEC == 2) {
        const float2 t = __ldcg(reinterpret_cast<const float2*>(p));
        v[0] = t.x; v[1] = t.y;
    } else {
        v[0] = __ldcg(p);
    }
}

// Coefficient of a list entry: -1/+1 from bit 31, doubled by bit 30 (a trit that
// flipped sign); with importance weights the list carries the coefficients itself.
__device__ __forceinline__ float entry_coef(int ent) {
    return (ent < 0 ? -1.f : 1.f) * ((ent & 0x40000000) ? 2.f : 1.f);
}

// Lazy-deflation correction at one of this CTA's outputs: sum_l coef_l t_l(c),
// t_l from the per-output pending bit masks, in increasing l.
struct HalfCorr {
    const double* coef;
    const uint32_t* cnz;
    const uint32_t* csg;
    double* corr;     // out: correction per output of this CTA (filled by the GEMV)
    double* g;        // running sum of the GEMV over this component's trit changes, per output
    int L;
};

// corr[c] = sum_l coef_l t_l(c) for this CTA's outputs.  Few outputs (a CTA of a large
// group): one warp per output, lane l taking pending component l, summed by a fixed
// butterfly.  Many outputs (a small group): one thread per output, the components that
// touch it added in increasing l.
__device__ __forceinline__ void corrections(int valid, const HalfCorr& hc) {
    if (hc.L <= 0) return;
    if (valid <= 2 * NWARP) {
        const int lane = lane_id();
        const double cl = lane < hc.L ? hc.coef[lane] : 0.0;
        for (int c = warp_id(); c < valid; c += NWARP) {
            const uint32_t z = hc.cnz[c], g = hc.csg[c];
            double t = ((z >> lane) & 1u) ? (((g >> lane) & 1u) ? -cl : cl) : 0.0;
            #pragma unroll
            for (int o = 16; o; o >>= 1) t += __shfl_xor_sync(FULL, t, o);
            if (lane == 0) hc.corr[c] = t;
        }
    } else {
        for (int c = threadIdx.x; c < valid; c += NT) {
            uint32_t z = hc.cnz[c];
            const uint32_t g = hc.csg[c];
            double t = 0.0;
            while (z) {
                const int l = __ffs(z) - 1;
                z &= z - 1u;
                t += ((g >> l) & 1u) ? -hc.coef[l] : hc.coef[l];
            }
            hc.corr[c] = t;
        }
    }
}

// Publish one output word and add its (published, 44-bit) magnitude to this thread's
// partial sum of |out|.
__device__ __forceinline__ void emit_tagged(double v, int64_t gi, unsigned long long* gout, unsigned tag, bool skip,
                                            double& S) {
    const unsigned long long w = tag_value(v, tag);
    if (!skip) st_relaxed_u64(gout + gi, w);
    S += fabs(__longlong_as_double((long long)(w & ~0xFFull)));
}

// acc += sum_u c_u v_u for one batch of loaded rows, in fp64: every term c_u v_u is
// exact in fp64 (c_u is +-1, +-2, or an fp32 weight times that; v_u is fp32, so the
// product has at most 48 significant bits) and each fused multiply-add rounds once,
// so a running sum of N terms is within (N - 1) 2^-53 sum|terms| of the exact sum.
template <int VEC, int U>
__device__ __forceinline__ void accumulate_batch(double* acc, const float* cf, float (*v)[VEC]) {
    #pragma unroll
    for (int u = 0; u < U; ++u) {
        const double c = (double)cf[u];
        #pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = fma(c, (double)v[u][e], acc[e]);   // inactive slots hold v = 0
    }
}

// Rows per batch of the GEMV: enough loads in flight per thread within the register budget.
template <int VEC>
__host__ __device__ constexpr int GEMV_U() {
    return (NT >= 1024) ? ((VEC == 4) ? 8 : (VEC == 2 ? 12 : 16)) : ((VEC == 4) ? 16 : (VEC == 2 ? 24 : 32));
}

// acc += sum over the list entries g, g + lanes, g + 2 lanes, ... of this thread's VEC
// columns, U entries per batch (every batch issues all its loads before using any).

template <int VEC, int U, bool WL>
__device__ __forceinline__ void gemv_rows(double* acc, const float* base, const int* __restrict__ list,
                                          const float* __restrict__ wl, int nlist, int g, int lanes) {
    for (int idx = g; idx < nlist; idx += U * lanes) {
        float cf[U];
        float v[U][VEC];
        #pragma unroll
        for (int u = 0; u < U; ++u) {
            const int ii = idx + u * lanes;
            const int ent = ii < nlist ? list[ii] : 0;
            if constexpr (WL) cf[u] = ii < nlist ? wl[ii] : 0.f;
            else cf[u] = entry_coef(ent);
            if (ii < nlist) {
                load_vec<VEC>(base + (ent & 0x3fffffff), v[u]);
            } else {
                #pragma unroll
                for (int e = 0; e < VEC; ++e) v[u][e] = 0.f;
            }
        }
        accumulate_batch<VEC, U>(acc, cf, v);
    }
}

// One half-step GEMV over this CTA's private block.  The list holds the trits that
// changed since the previous half-step of the same kind in this component (all of
// them in the first one, where g starts at 0), so g[c] += sum_{e in list} s_e blk[r_e][c]
// keeps g = R^T t (or R t) for the current input trits t; out[c] = g[c] minus the
// lazy-deflation correction is written to gout[out0 + c].  fp64 accumulation of exact fp32 terms, fixed summation order.
// S returns this warp's sum of the published |out| in lane 0 (a fixed butterfly).
template <int VEC, bool WL>
__device__ void gemv_emit(const float* __restrict__ blk, int pitch, int valid, int64_t out0,
                          const int* __restrict__ list, const float* __restrict__ wl, int nlist, double* red,
                          unsigned long long* gout, const HalfCorr& hc, unsigned tag, bool skip, double& S,
                          unsigned long long* clk) {
    S = 0.0;
    const int nvec = pitch / VEC;
    if (nvec <= 0) return;
    corrections(valid, hc);   // read after the CTA barrier below
    if (nvec <= NT) {
        const int lanes = NT / nvec;
        const int act = min(lanes, nlist);   // row groups that get at least one entry
        const int j = threadIdx.x % nvec;
        const int g = threadIdx.x / nvec;
        const int rs = pitch | 1;   // odd row stride (in doubles): the column sums below are bank-conflict free
        if (g < act) {
            double acc[VEC];
            #pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = 0.0;
            const float* base = blk + j * VEC;
            // batch width from the longest group (uniform over the CTA): short change
            // lists issue few predicated slots
            const int per = (nlist + lanes - 1) / lanes;
            if (per <= 1) gemv_rows<VEC, 1, WL>(acc, base, list, wl, nlist, g, lanes);
            else if (per <= 2) gemv_rows<VEC, 2, WL>(acc, base, list, wl, nlist, g, lanes);
            else if (per <= 4) gemv_rows<VEC, 4, WL>(acc, base, list, wl, nlist, g, lanes);
            else gemv_rows<VEC, GEMV_U<VEC>(), WL>(acc, base, list, wl, nlist, g, lanes);
            #pragma unroll
            for (int e = 0; e < VEC; ++e) red[g * rs + j * VEC + e] = acc[e];
        }
        __syncthreads();
        phase_mark(clk, 0);
        int tpc = 1;
        while (tpc < 32 && tpc * 2 * pitch <= NT) tpc *= 2;
        const int cpr = NT / tpc;
        for (int cb = 0; cb < pitch; cb += cpr) {
            const int c = cb + (int)threadIdx.x / tpc;
            const int s = (int)threadIdx.x % tpc;
            double v = 0.0;
            if (c < pitch)
                for (int gg = s; gg < act; gg += tpc) v += red[gg * rs + c];
            for (int o = tpc >> 1; o; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
            if (s == 0 && c < valid) {
                const double gc = hc.g[c] + v;
                hc.g[c] = gc;
                emit_tagged(hc.L > 0 ? gc - hc.corr[c] : gc, out0 + c, gout, tag, skip, S);
            }
        }
        // this warp's sum of |out| into lane 0: only lanes that are multiples of tpc emitted,
        // so the butterfly rounds below tpc would add exact zeros
        for (int o = 16; o >= tpc; o >>= 1) S += __shfl_xor_sync(FULL, S, o);
    } else {
        constexpr int U = GEMV_U<VEC>();
        __syncthreads();   // corrections
        for (int j = threadIdx.x; j < nvec; j += NT) {
            double acc[VEC];
            #pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = 0.0;
            const float* base = blk + j * VEC;
            for (int idx = 0; idx < nlist; idx += U) {
                float cf[U];
                float v[U][VEC];
                #pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int ii = idx + u;
                    const int ent = ii < nlist ? list[ii] : 0;
                    if constexpr (WL) cf[u] = ii < nlist ? wl[ii] : 0.f;
                    else cf[u] = entry_coef(ent);
                    if (ii < nlist) {
                        load_vec<VEC>(base + (ent & 0x3fffffff), v[u]);
                    } else {
                        #pragma unroll
                        for (int e = 0; e < VEC; ++e) v[u][e] = 0.f;
                    }
                }
                accumulate_batch<VEC, U>(acc, cf, v);
            }
            #pragma unroll
            for (int e = 0; e < VEC; ++e) {
                const int c = j * VEC + e;
                if (c < valid) {
                    const double gc = hc.g[c] + acc[e];
                    hc.g[c] = gc;
                    emit_tagged(hc.L > 0 ? gc - hc.corr[c] : gc, out0 + c, gout, tag, skip, S);
                }
            }
        }
        #pragma unroll
        for (int o = 16; o; o >>= 1) S += __shfl_xor_sync(FULL, S, o);   // this warp's sum into lane 0
    }
}

template <bool WL>
__device__ __forceinline__ void gemv_dispatch(int vec, const float* blk, int pitch, int valid, int64_t out0,
                                              const int* list, const float* wl, int nlist, double* red,
                                              unsigned long long* gout, const HalfCorr& hc, unsigned tag, bool skip,
                                              double& S, unsigned long long* clk) {
    if (vec == 4) gemv_emit<4, WL>(blk, pitch, valid, out0, list, wl, nlist, red, gout, hc, tag, skip, S, clk);
    else if (vec == 2) gemv_emit<2, WL>(blk, pitch, valid, out0, list, wl, nlist, red, gout, hc, tag, skip, S, clk);
    else gemv_emit<1, WL>(blk, pitch, valid, out0, list, wl, nlist, red, gout, hc, tag, skip, S, clk);
}

// Fold the L pending components into this CTA's block:
// blk[r][c] -= sum_l d_l * tR_l(r) * tC_l(c), fp64 sum in increasing l, one fp32 rounding.
// A warp takes 32 block rows at a time: the word-major pending masks of those rows
// (lane l holds component l's 32 row bits) are bit-transposed with ballots so that
// lane b holds row b's mask over the components; tC_l(c) comes from the
// per-output masks cnz/csg.  scratch: 64 words per warp.
template <int VEC>
__device__ void flush_block(float* blk, float* blo, int pitch, int64_t rows, int valid, int L, int Ls, const double* pd,
                            const uint32_t* pnzR, const uint32_t* psgR, const uint32_t* cnz, const uint32_t* csg,
                            uint32_t* scratch) {
    const int nvec = pitch / VEC;
    if (nvec <= 0 || L <= 0) return;
    const int lane = lane_id();
    uint32_t* my = scratch + warp_id() * 64;
    const int64_t WR = (rows + 31) >> 5;
    for (int64_t wr = warp_id(); wr < WR; wr += NWARP) {
        const uint32_t pz = lane < L ? pnzR[wr * Ls + lane] : 0u;
        const uint32_t ps = lane < L ? psgR[wr * Ls + lane] : 0u;
        uint32_t rz = 0u, rsg = 0u;
        #pragma unroll
        for (int b = 0; b < 32; ++b) {
            const uint32_t z = __ballot_sync(FULL, (pz >> b) & 1u);
            const uint32_t g = __ballot_sync(FULL, (ps >> b) & 1u);
            if (lane == b) { rz = z; rsg = g; }
        }
        my[lane] = rz;
        my[32 + lane] = rsg;
        __syncwarp();
        const int nrows = (int)min((int64_t)32, rows - (wr << 5));
        const int pairs = nrows * nvec;
        for (int t = lane; t < pairs; t += 32) {
            const int b = t / nvec;
            const int j = t - b * nvec;
            const uint32_t rnz = my[b];
            if (!rnz) continue;
            const uint32_t rsn = my[32 + b];
            float* p = blk + ((wr << 5) + b) * pitch + j * VEC;
            float* plo = blo + ((wr << 5) + b) * pitch + j * VEC;
            #pragma unroll
            for (int e = 0; e < VEC; ++e) {
                const int c = j * VEC + e;
                if (c >= valid) continue;
                uint32_t bits = rnz & cnz[c];
                if (!bits) continue;
                const uint32_t neg = rsn ^ csg[c];
                double corr = 0.0;
                while (bits) {
                    const int l = __ffs(bits) - 1;
                    bits &= bits - 1u;
                    corr += ((neg >> l) & 1u) ? -pd[l] : pd[l];
                }
                // hi + lo is exact in fp64; the new value rounds once in fp64, then splits
                // into its nearest fp32 (hi) and the fp32 rounding of the rest (lo)
                const double nv = ((double)__ldcg(p + e) + (double)__ldcg(plo + e)) - corr;
                const float hi = (float)nv;
                p[e] = hi;
                plo[e] = (float)(nv - (double)hi);
            }
        }
        __syncwarp();
    }
}

__device__ __forceinline__ void flush_dispatch(int vec, float* blk, float* blo, int pitch, int64_t rows, int valid, int L,
                                               int Ls, const double* pd, const uint32_t* pnzR, const uint32_t* psgR,
                                               const uint32_t* cnz, const uint32_t* csg, uint32_t* scratch) {
    if (vec == 4) flush_block<4>(blk, blo, pitch, rows, valid, L, Ls, pd, pnzR, psgR, cnz, csg, scratch);
    else if (vec == 2) flush_block<2>(blk, blo, pitch, rows, valid, L, Ls, pd, pnzR, psgR, cnz, csg, scratch);
    else flush_block<1>(blk, blo, pitch, rows, valid, L, Ls, pd, pnzR, psgR, cnz, csg, scratch);
}

// Start trits (2-bit packed words) -> masks and list; returns nnz.
__device__ int build_from_trits(const uint32_t* words, int64_t nwords, int64_t len, uint32_t* nz, uint32_t* sg,
                                int* list, int rowpitch, const Smem& s) {
    const int W = (int)((len + 31) >> 5);
    const int wpw = (W + NWARP - 1) / NWARP;
    const int w0 = min(W, warp_id() * wpw), w1 = min(W, w0 + wpw);
    int cnt = 0;
    for (int w = w0 + lane_id(); w < w1; w += 32) {
        const int64_t a = 2 * (int64_t)w, b = a + 1;
        const uint32_t lo = a < nwords ? __ldcg(words + a) : 0u;
        const uint32_t hi = b < nwords ? __ldcg(words + b) : 0u;
        uint32_t z = compact_even(lo) | (compact_even(hi) << 16);
        uint32_t sb = compact_even(lo >> 1) | (compact_even(hi >> 1) << 16);
        const int64_t rem = len - ((int64_t)w << 5);
        if (rem < 32) z &= (1u << rem) - 1u;
        sb &= z;
        nz[w] = z;
        sg[w] = sb;
        cnt += __popc(z);
    }
    #pragma unroll
    for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(FULL, cnt, o);
    if (lane_id() == 0) s.wc[warp_id()] = cnt;
    __syncthreads();
    int off = 0, total = 0;
    for (int w = 0; w < NWARP; ++w) {
        const int c = s.wc[w];
        off += (w < warp_id()) ? c : 0;
        total += c;
    }
    int run = off;
    for (int w = w0; w < w1; ++w) {
        const uint32_t bz = nz[w];
        if ((bz >> lane_id()) & 1u)
            list[run + __popc(bz & ((1u << lane_id()) - 1u))] =
                (int)((((unsigned)w << 5) + lane_id()) * (unsigned)rowpitch) | (int)(((sg[w] >> lane_id()) & 1u) << 31);
        run += __popc(bz);
    }
    __syncthreads();
    return total;
}

// dot_l = t_l . t and coef_l = d_l dot_l for every pending component (integer dot
// product of trit masks)
__device__ void pending_coef(int L, int Ls, int W, const uint32_t* pnz, const uint32_t* psg, const uint32_t* nz,
                             const uint32_t* sg, const double* pd, int* dots, double* coef) {
    for (int l = warp_id(); l < L; l += NWARP) {
        int acc = 0;
        for (int w = lane_id(); w < W; w += 32) {
            const uint32_t both = pnz[w * Ls + l] & nz[w];
            const uint32_t diff = psg[w * Ls + l] ^ sg[w];
            acc += __popc(both & ~diff) - __popc(both & diff);
        }
        #pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
        if (lane_id() == 0) { dots[l] = acc; coef[l] = pd[l] * (double)acc; }
    }
    __syncthreads();
}

// dotw_l = sum_c h~_c t_l(c) t(c) and coef_l = d_l dotw_l for every pending component
// (weighted objective), fixed order: words by lane, bits in increasing order.
__device__ void pending_coef_w(int L, int Ls, int W, const uint32_t* pnz, const uint32_t* psg, const uint32_t* nz,
                               const uint32_t* sg, const double* pd, const float* hw, double* dotw, double* coef) {
    for (int l = warp_id(); l < L; l += NWARP) {
        double acc = 0.0;
        for (int w = lane_id(); w < W; w += 32) {
            const uint32_t both = pnz[w * Ls + l] & nz[w];
            const uint32_t neg = psg[w * Ls + l] ^ sg[w];
            for (uint32_t mk = both; mk; mk &= mk - 1u) {
                const int b = __ffs(mk) - 1;
                const double hv = (double)__ldg(hw + ((int64_t)w << 5) + b);
                acc += ((neg >> b) & 1u) ? -hv : hv;
            }
        }
        #pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
        if (lane_id() == 0) { dotw[l] = acc; coef[l] = pd[l] * acc; }
    }
    __syncthreads();
}

__device__ void pack_row(const uint32_t* nz, const uint32_t* sg, int W, uint32_t* out, int64_t out_words) {
    for (int64_t w = threadIdx.x; w < out_words; w += NT) {
        const int64_t mw = w >> 1;
        uint32_t z = 0, s = 0;
        if (mw < W) {
            z = nz[mw]; s = sg[mw];
            if (w & 1) { z >>= 16; s >>= 16; }
        }
        out[w] = spread_even(z) | (spread_even(s & z) << 1);
    }
}

// ---------------------------------------------------------------------------
// Exchange of the half-step outputs between the CTAs of a group.
//
// Each output value is published as one 8-byte word: the fp64 value with its 8
// low mantissa bits replaced by a tag that names the half-step (1..255).  An
// 8-byte relaxed store/load at gpu scope is single-copy atomic, so a reader that
// sees the expected tag sees the value of that half-step, with no flag, fence or
// counter.  The value keeps 44 mantissa bits (relative change < 2^-44); every CTA
// reads the same words, so all of them derive the same threshold and trits.  A
// buffer is rewritten only two half-steps later, after every CTA has read it, so a
// stale word always carries the tag of two half-steps before.
// ---------------------------------------------------------------------------

// Positions where the trit vector changed from (oz, os) to (bz, bs) (nonzero mask,
// negative mask), the sign of the change new - old, and whether it is +-2 (a flip).
__device__ __forceinline__ uint32_t delta_mask(uint32_t oz, uint32_t os, uint32_t bz, uint32_t bs, uint32_t& neg,
                                               uint32_t& two) {
    two = oz & bz & (os ^ bs);
    neg = (bz & bs) | (~bz & oz & ~os);
    return (oz ^ bz) | two;
}

// List entry of one changed trit: element offset | negative << 31 | (|change| == 2) << 30.
__device__ __forceinline__ int delta_entry(unsigned idx, int rowpitch, uint32_t neg, uint32_t two, int bit) {
    return (int)(idx * (unsigned)rowpitch) | (int)(((neg >> bit) & 1u) << 31) | (int)(((two >> bit) & 1u) << 30);
}

// Block-wide: compacted list of the changes (onz, osg) -> (nz, sg) over W mask words,
// in index order.  Returns the count.
template <bool WL>
__device__ int build_delta_list(int W, const uint32_t* onz, const uint32_t* osg, const uint32_t* nz,
                                const uint32_t* sg, int* list, int rowpitch, const Smem& s,
                                const float* hw = nullptr, float* wl = nullptr) {
    const int lane = lane_id(), warp = warp_id();
    const int wpw = (W + NWARP - 1) / NWARP;
    const int w0 = min(W, warp * wpw), w1 = min(W, w0 + wpw);
    int cnt = 0;
    for (int w = w0 + lane; w < w1; w += 32) {
        uint32_t ng, tw;
        cnt += __popc(delta_mask(onz[w], osg[w], nz[w], sg[w], ng, tw));
    }
    #pragma unroll
    for (int o = 16; o; o >>= 1) cnt += __shfl_xor_sync(FULL, cnt, o);
    if (lane == 0) s.wd[warp] = cnt;
    __syncthreads();
    int off = 0, total = 0;
    for (int w = 0; w < NWARP; ++w) {
        const int c = s.wd[w];
        off += (w < warp) ? c : 0;
        total += c;
    }
    int run = off;
    for (int w = w0; w < w1; ++w) {
        uint32_t ng, tw;
        const uint32_t ch = delta_mask(onz[w], osg[w], nz[w], sg[w], ng, tw);
        if ((ch >> lane) & 1u) {
            const int at = run + __popc(ch & ((1u << lane) - 1u));
            const int e = delta_entry(((unsigned)w << 5) + lane, rowpitch, ng, tw, lane);
            list[at] = e;
            if constexpr (WL) wl[at] = entry_coef(e) * __ldg(hw + ((int64_t)w << 5) + lane);
        }
        run += __popc(ch);
    }
    __syncthreads();
    return total;
}

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ double untag(unsigned long long b) { return __longlong_as_double((long long)(b & ~0xFFull)); }

// half-step counter -> tag in 1..255 (0 is the zero-initialised buffer)
__device__ __forceinline__ unsigned gen_tag(unsigned gen) { return (gen % 255u) + 1u; }

// Bounded spin until *p carries `tag`; returns the word, or sets ok = 0 on timeout/abort.
__device__ __forceinline__ unsigned long long wait_tagged(const unsigned long long* p, unsigned tag, GroupSync* gs,
                                                          uint64_t limit_ns, int* status, int& ok,
                                                          unsigned long long* stale_ctr = nullptr) {
    unsigned long long b = ld_relaxed_u64(p);
    if ((unsigned)(b & 0xFFull) == tag) return b;
    if (stale_ctr && blockIdx.x == 0) atomicAdd(stale_ctr, 1ull);
    const uint64_t t0 = gtimer();
    unsigned spins = 0;
    while (true) {
        b = ld_relaxed_u64(p);
        if ((unsigned)(b & 0xFFull) == tag) return b;
        if ((++spins & 15u) == 0u) {
            if (ld_relaxed_s32(&gs->abort)) { ok = 0; return 0ull; }
            if (gtimer() - t0 > limit_ns) {
                atomicExch(&gs->abort, 1);
                atomicCAS(status, ST_RUNNING, ST_ETIMEOUT);
                ok = 0;
                return 0ull;
            }
        }
    }
}

__device__ __forceinline__ void red_relaxed_add(unsigned* p, unsigned v) {
    asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Publish this CTA's partial sum |out| of the half-step as a tagged word
// partials[q] and count its arrival on counter q % NCTR; wait until every CTA of
// the group has arrived (NCTR threads poll one counter each, bounded), read all
// partials (tag-checked), read the whole output vector (tag-checked, re-polling any
// word not yet visible), threshold it (T_tau of §2.2 with the all-zero fallback;
// tau_len = tau / len, so the threshold is tau_len * sum |out|),
// write its masks and compacted support list, the coefficients d_l (t_l . t) of the
// pending components for the next half-step, and p = sum over the support of |x|
// into s.scal[0] (s.scal[1] = 1 if the fallback was taken).  Sums are combined in
// one fixed order, so every CTA of the group derives identical results.  Arrival
// needs no fence: the tags validate every word that is read.
// Returns nnz; ok = false if a wait ran out.
template <bool WTD>
__device__ int exchange_threshold(unsigned long long* partials, int q, int Gg, unsigned tag, unsigned& arrivals,
                                  bool skip, double S, const unsigned long long* gvec, int64_t len, double tau_len,
                                  uint32_t* nz, uint32_t* sg, uint32_t* onz, uint32_t* osg, int* list, int rowpitch,
                                  const Smem& s, int L, int Ls, const uint32_t* pnz, const uint32_t* psg, int* dots,
                                  double* coef, bool want_p, double& thr_out, int& ndelta, GroupSync* gs,
                                  uint64_t limit_ns, int* status, bool& ok_out, const float* hw = nullptr,
                                  float* wl = nullptr, double* dotw = nullptr, double* hsum_out = nullptr) {
    const int lane = lane_id(), warp = warp_id();
    // ---- this CTA's partial: S holds each warp's sum in lane 0 (summed by the GEMV's
    //      fixed butterfly), combined across warps in a fixed order
    if (lane == 0) s.wS[warp] = S;
    __syncthreads();
    if (warp == 0) {
        double S2 = lane < NWARP ? s.wS[lane] : 0.0;
        #pragma unroll
        for (int o = 16; o; o >>= 1) S2 += __shfl_xor_sync(FULL, S2, o);
        if (lane == 0) {
            if (Gg > 1) {
                if (!skip) {
                    st_relaxed_u64(partials + q, tag_value(S2, tag));
                    red_relaxed_add(&gs->ctr[q % NCTR][0], 1u);
                }
            } else {
                // a group of one CTA: its own partial, rounded as a published word would be, is
                // the total; there is nothing to wait for
                s.gS[0] = untag(tag_value(S2, tag));
            }
        }
    }
    ++arrivals;
    phase_mark(s, 2);
    // ---- wait for all arrivals (NCTR threads poll one counter each, bounded), then
    //      everyone's partials
    int ok = 1;
    if (Gg > 1 && (int)threadIdx.x < NCTR && (int)threadIdx.x < Gg) {
        const int c = threadIdx.x;
        const unsigned want = arrivals * (unsigned)((Gg - c + NCTR - 1) / NCTR);
        const unsigned* ctr = &gs->ctr[c][0];
        if ((int)(ld_relaxed_u32(ctr) - want) < 0) {
            const uint64_t t0 = gtimer();
            unsigned spins = 0;
            while ((int)(ld_relaxed_u32(ctr) - want) < 0) {
                if ((++spins & 15u) == 0u) {
                    if (ld_relaxed_s32(&gs->abort)) { ok = 0; break; }
                    if (gtimer() - t0 > limit_ns) {
                        atomicExch(&gs->abort, 1);
                        atomicCAS(status, ST_RUNNING, ST_ETIMEOUT);
                        ok = 0;
                        break;
                    }
                }
            }
        }
    }
    ok = __syncthreads_and(ok);
    phase_mark(s, 3);
    if (!ok) { ok_out = false; return 0; }
    // the first chunk of this warp's words is loaded together with the partials
    const int W = (int)((len + 31) >> 5);
    const int wpw = (W + NWARP - 1) / NWARP;
    const int w0 = min(W, warp * wpw), w1 = min(W, w0 + wpw);
    constexpr int CH = (NT >= 1024) ? 8 : 16;
    unsigned long long wb[CH];
    #pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int w = w0 + i;
        const int64_t idx = ((int64_t)w << 5) + lane;
        wb[i] = (w < w1 && idx < len) ? ld_relaxed_u64(gvec + idx) : (unsigned long long)tag;
    }
    if (Gg > 1 && warp * 32 < Gg) {   // the warps that hold partials
        double Sq = 0.0;
        if ((int)threadIdx.x < Gg) Sq = untag(wait_tagged(partials + threadIdx.x, tag, gs, limit_ns, status, ok));
        #pragma unroll
        for (int o = 16; o; o >>= 1) Sq += __shfl_xor_sync(FULL, Sq, o);
        if (lane == 0) s.gS[warp] = Sq;
    }
    if (Gg > 1) ok = __syncthreads_and(ok);   // (one CTA: gS[0] was written before the barrier above)
    phase_mark(s, 4);
    if (!ok) { ok_out = false; return 0; }
    double St = 0.0;   // the same fixed order in every thread
    for (int w = 0; w < Gg; w += 32) St += s.gS[w >> 5];
    const double thr = St * tau_len;   // tau * mean |x|, with tau / len computed once per matrix
    thr_out = thr;

    // ---- one pass over the vector: threshold, masks, counts, pending dots.  The warp
    //      takes its words in groups of up to 32: first every ballot (registers only),
    //      then lane i handles word base + i (old masks, changes, stores) in parallel.
    int cnt = 0, dcnt = 0, dot = 0;
    double ps = 0.0, hsum = 0.0, dotw_acc = 0.0;
    for (int base = w0; base < w1; base += 32) {
        const int K = min(32, w1 - base);
        uint32_t my_bz = 0u, my_bs = 0u;
        for (int c0 = 0; c0 < K; c0 += CH) {
            if (base != w0 || c0 != 0) {
                #pragma unroll
                for (int i = 0; i < CH; ++i) {
                    const int w = base + c0 + i;
                    const int64_t idx = ((int64_t)w << 5) + lane;
                    wb[i] = (c0 + i < K && idx < len) ? ld_relaxed_u64(gvec + idx) : (unsigned long long)tag;
                }
            }
            bool stale = false;
            #pragma unroll
            for (int i = 0; i < CH; ++i) stale |= (unsigned)(wb[i] & 0xFFull) != tag;
            if (__any_sync(FULL, stale)) {   // rare: a word not yet visible here, re-poll it
                #pragma unroll
                for (int i = 0; i < CH; ++i) {
                    if ((unsigned)(wb[i] & 0xFFull) != tag)
                        wb[i] = wait_tagged(gvec + ((int64_t)(base + c0 + i) << 5) + lane, tag, gs, limit_ns, status,
                                            ok, s.clk + 10);
                }
            }
            #pragma unroll
            for (int i = 0; i < CH; ++i) {
                if (c0 + i >= K) break;   // K is the same in every lane: skip the unused slots
                {
                    const double x = untag(wb[i]);           // padding words untag to 0
                    const bool z = fabs(x) > thr;
                    const unsigned bz = __ballot_sync(FULL, z);
                    const unsigned bs = __ballot_sync(FULL, z && (x < 0.0));
                    if (lane == c0 + i) { my_bz = bz; my_bs = bs; }
                    if (want_p && z) ps += fabs(x);
                }
            }
        }
        const int w = base + lane;
        uint32_t oz = 0u, os = 0u, ch = 0u, dn = 0u, dt = 0u;
        if (lane < K) {
            oz = nz[w];
            os = sg[w];
            ch = delta_mask(oz, os, my_bz, my_bs, dn, dt);
        }
        __syncwarp();
        if (lane < K) { nz[w] = my_bz; sg[w] = my_bs; onz[w] = oz; osg[w] = os; }
        cnt += __popc(my_bz);
        dcnt += __popc(ch);
        if constexpr (WTD) {   // sum of h~ over the new support: lane b takes bit b of each word, in word order
            for (int i = 0; i < K; ++i) {
                const uint32_t zi = __shfl_sync(FULL, my_bz, i);
                const int64_t c = ((int64_t)(base + i) << 5) + lane;
                if ((zi >> lane) & 1u) hsum += (double)__ldg(hw + c);
            }
        }
        // change of t_l . t (weighted: sum h~_c t_l(c) t(c)) over the words that changed
        // (lane l = pending component l)
        unsigned chw = __ballot_sync(FULL, ch != 0u);
        while (chw) {
            const int i = __ffs(chw) - 1;
            chw &= chw - 1u;
            const uint32_t zi = __shfl_sync(FULL, my_bz, i), si = __shfl_sync(FULL, my_bs, i);
            const uint32_t ozi = __shfl_sync(FULL, oz, i), osi = __shfl_sync(FULL, os, i);
            const uint32_t chi = __shfl_sync(FULL, ch, i);
            if constexpr (WTD) {
                // sum over the changed bits b of h~_b t_l(b) (new - old trit), lane l = component l;
                // the word's 32 weights are loaded once (lane b: bit b) and broadcast per bit
                const uint32_t dni = __shfl_sync(FULL, dn, i), dti = __shfl_sync(FULL, dt, i);
                const int64_t cb = ((int64_t)(base + i) << 5) + lane;
                const float hword = cb < len ? __ldg(hw + cb) : 0.f;
                const uint32_t pz = lane < L ? pnz[(base + i) * Ls + lane] : 0u;
                const uint32_t pg = lane < L ? psg[(base + i) * Ls + lane] : 0u;
                // each lane walks its own bits (pz & chi) in increasing order; every lane takes
                // part in each shuffle, so the loop runs the warp's largest count
                uint32_t mine = pz & chi;
                const int rounds = (int)__reduce_max_sync(FULL, (unsigned)__popc(mine));
                for (int t = 0; t < rounds; ++t) {
                    const int b = mine ? __ffs(mine) - 1 : 0;
                    const double hv = (double)__shfl_sync(FULL, hword, b);
                    if (mine) {
                        const double dv = (((dni >> b) & 1u) ? -1.0 : 1.0) * (((dti >> b) & 1u) ? 2.0 : 1.0);
                        dotw_acc += ((pg >> b) & 1u) ? -hv * dv : hv * dv;
                        mine &= mine - 1u;
                    }
                }
            } else if (lane < L) {
                const uint32_t pz = pnz[(base + i) * Ls + lane], pg = psg[(base + i) * Ls + lane];
                {
                    const uint32_t zn = pz & zi & chi, zo = pz & ozi & chi;
                    const uint32_t sn = pg ^ si, so = pg ^ osi;
                    dot += (__popc(zn & ~sn) - __popc(zn & sn)) - (__popc(zo & ~so) - __popc(zo & so));
                }
            }
        }
    }
    cnt = __reduce_add_sync(FULL, cnt);
    dcnt = __reduce_add_sync(FULL, dcnt);
    if (want_p) {
        #pragma unroll
        for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(FULL, ps, o);
    }
    if constexpr (WTD) {
        #pragma unroll
        for (int o = 16; o; o >>= 1) hsum += __shfl_xor_sync(FULL, hsum, o);
        if (lane == 0) s.wM[warp] = hsum;
        if (lane < L) s.dotpw[lane * DSTR + warp] = dotw_acc;
    }
    if (lane == 0) { s.wc[warp] = cnt; s.wd[warp] = dcnt; s.wp[warp] = ps; }
    if (lane < L) s.dotp[lane * DSTR + warp] = dot;
    ok = __syncthreads_and(ok);
    phase_mark(s, 5);
    if (!ok) { ok_out = false; return 0; }
    const int dw = lane < NWARP ? s.wd[lane] : 0;
    const int total = __reduce_add_sync(FULL, lane < NWARP ? s.wc[lane] : 0);
    const int off = __reduce_add_sync(FULL, lane < warp ? dw : 0);   // this warp's place in the list
    const int dtotal = __reduce_add_sync(FULL, dw);
    double p = 0.0;   // needed by thread 0 only
    if (warp == 0 && want_p) {
        p = lane < NWARP ? s.wp[lane] : 0.0;
        #pragma unroll
        for (int o = 16; o; o >>= 1) p += __shfl_xor_sync(FULL, p, o);
    }
    if constexpr (WTD) {
        double hs = lane < NWARP ? s.wM[lane] : 0.0;
        #pragma unroll
        for (int o = 16; o; o >>= 1) hs += __shfl_xor_sync(FULL, hs, o);
        *hsum_out = hs;
    }
    if (total > 0) {
        for (int l = warp; l < L; l += NWARP) {
            if constexpr (WTD) {
                double d = lane < NWARP ? s.dotpw[l * DSTR + lane] : 0.0;
                #pragma unroll
                for (int o = 16; o; o >>= 1) d += __shfl_xor_sync(FULL, d, o);
                if (lane == 0) {
                    d += dotw[l];
                    dotw[l] = d;
                    coef[l] = s.pd[l] * d;
                }
            } else {
                int d = lane < NWARP ? s.dotp[l * DSTR + lane] : 0;
                d = __reduce_add_sync(FULL, d);
                if (lane == 0) {
                    d += dots[l];
                    dots[l] = d;
                    coef[l] = s.pd[l] * (double)d;
                }
            }
        }
        int run = off;
        if constexpr (WTD) {   // one word at a time across the lanes (lane b: bit b), in index order
            for (int w = w0; w < w1; ++w) {
                uint32_t ng, tw;
                const uint32_t ch = delta_mask(onz[w], osg[w], nz[w], sg[w], ng, tw);
                if ((ch >> lane) & 1u) {
                    const int at = run + __popc(ch & ((1u << lane) - 1u));
                    const int e = delta_entry(((unsigned)w << 5) + lane, rowpitch, ng, tw, lane);
                    wl[at] = entry_coef(e) * __ldg(hw + ((int64_t)w << 5) + lane);
                    list[at] = e;
                }
                run += __popc(ch);
            }
        } else for (int base = w0; base < w1; base += 32) {
            const int w = base + lane;
            uint32_t ch = 0u, ng = 0u, tw = 0u;
            if (w < w1) ch = delta_mask(onz[w], osg[w], nz[w], sg[w], ng, tw);
            const int c = __popc(ch);
            int incl = c;
            #pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(FULL, incl, o);
                if (lane >= o) incl += t;
            }
            int at = run + incl - c;
            for (uint32_t mk = ch; mk; mk &= mk - 1u) {
                const int b = __ffs(mk) - 1;
                const int e = delta_entry(((unsigned)w << 5) + b, rowpitch, ng, tw, b);
                list[at++] = e;
            }
            run += __shfl_sync(FULL, incl, 31);
        }
        ndelta = dtotal;
        if (threadIdx.x == 0) { s.scal[0] = p; s.scal[1] = 0.0; }
    } else {
        // all-zero fallback: keep the lowest index among the largest magnitudes
        // (every CTA scans the same vector in the same order)
        double Mx = -1.0;
        long long Jx = LLONG_MAX;
        for (int64_t i = threadIdx.x; i < len; i += NT) {
            const double a = fabs(untag(ld_relaxed_u64(gvec + i)));
            if (a > Mx) { Mx = a; Jx = i; }
        }
        long long Jt = Jx;
        block_maxloc(Mx, Jt, s.red, reinterpret_cast<long long*>(s.red + 64));   // red is free here
        const long long Jc = (Jt >= 0 && Jt < len) ? Jt : 0;   // out of range only with non-finite data
        const double x = untag(ld_relaxed_u64(gvec + Jc));
        const bool neg = x < 0.0;
        const int wj = (int)(Jc >> 5);
        const uint32_t bj = 1u << (Jc & 31);
        if (threadIdx.x == 0) {
            nz[wj] |= bj;
            if (neg) sg[wj] |= bj;
            s.scal[0] = fabs(x);
            s.scal[1] = 1.0;
        }
        __syncthreads();
        ndelta = build_delta_list<WTD>((int)((len + 31) >> 5), onz, osg, nz, sg, list, rowpitch, s, hw, wl);
        if (L > 0) {
            if constexpr (WTD) pending_coef_w(L, Ls, (int)((len + 31) >> 5), pnz, psg, nz, sg, s.pd, hw, dotw, coef);
            else pending_coef(L, Ls, (int)((len + 31) >> 5), pnz, psg, nz, sg, s.pd, dots, coef);
        }
        if constexpr (WTD) *hsum_out = (double)__ldg(hw + Jc);
    }
    __syncthreads();
    phase_mark(s, 6);
    ok_out = true;
    return total > 0 ? total : 1;
}

// Sum of one fp64 value per CTA of the group (fixed order), exchanged as tagged words.
// `use` numbers the calls of this group from 1: consecutive calls alternate between
// two buffers of Gg words and carry different tags, so a CTA that is already in call
// j + 1 cannot overwrite a word another CTA still waits for in call j.  Every
// exchange also orders: a CTA leaves it only after every CTA has entered it.
__device__ bool exchange_sum(unsigned long long* sums, int q, int Gg, double v, double* red, GroupSync* gs,
                             uint64_t limit_ns, int* status, bool skip, unsigned use, double& out) {
    const unsigned tag = gen_tag(use);
    unsigned long long* buf = sums + (size_t)(use & 1u) * Gg;
    const double t = block_sum(v, red);
    if (threadIdx.x == 0 && !skip) st_relaxed_u64(buf + q, tag_value(t, tag));
    int ok = 1;
    double x = 0.0;
    if ((int)threadIdx.x < Gg) x = untag(wait_tagged(buf + threadIdx.x, tag, gs, limit_ns, status, ok));
    ok = __syncthreads_and(ok);
    if (!ok) return false;
    out = block_sum(x, red);
    return true;
}

// Append the rank-1 term d u v^T (u, v: the masks nzU/sgU, nzV/sgV) as pending
// lazy-deflation component L: full-length word-major masks for the dot products and
// per-output bits for the corrections of this CTA's columns and rows.
__device__ void push_pending(const Smem& s, int L, int Ls, double d, int Wm, int Wn, int64_t c0, int validV,
                             int64_t r0, int validU) {
    const int tid = threadIdx.x;
    if (tid == 0) s.pd[L] = d;
    for (int w = tid; w < Wm; w += NT) { s.pnzU[w * Ls + L] = s.nzU[w]; s.psgU[w * Ls + L] = s.sgU[w]; }
    for (int w = tid; w < Wn; w += NT) { s.pnzV[w * Ls + L] = s.nzV[w]; s.psgV[w * Ls + L] = s.sgV[w]; }
    for (int c = tid; c < validV; c += NT) {
        const int64_t gc = c0 + c;
        const uint32_t b = 1u << (gc & 31);
        if (s.nzV[gc >> 5] & b) {
            s.cnzV[c] |= 1u << L;
            if (s.sgV[gc >> 5] & b) s.csgV[c] |= 1u << L;
        }
    }
    for (int r = tid; r < validU; r += NT) {
        const int64_t gr = r0 + r;
        const uint32_t b = 1u << (gr & 31);
        if (s.nzU[gr >> 5] & b) {
            s.cnzU[r] |= 1u << L;
            if (s.sgU[gr >> 5] & b) s.csgU[r] |= 1u << L;
        }
    }
    __syncthreads();
}

// Calls of exchange_sum during refinement, numbered from 1 by visit: per refinement
// visit r = 0, 1, ... one at its end (p_old) and, with k = 1, one at its start.
__device__ __forceinline__ unsigned sum_use_start(int64_t r) { return (unsigned)(2 * r + 1); }
__device__ __forceinline__ unsigned sum_use_end(int64_t r, int64_t kk) { return (unsigned)(kk == 1 ? 2 * r + 2 : r + 1); }

// Start of a refinement visit of component i (§2.4, "Refinement sweeps"): load the
// stored u_i, v_i (packed rows of B and C) and d_i, record d_i, n_old and the pending
// slot in s.scal[8], [9], [11], and append the added-back term d_i u_i v_i^T as pending
// component L with coefficient -d_i.  Leaves u = u_i in nzU/sgU/ulist and v = 0.
// Returns nnz(u_i), or -1 if the group aborted.  (Inlined: as a call, the registers
// the half-step loop keeps live across it spilled more than the inlined code does.)
__device__ __forceinline__ int refine_begin(const Prob& P, int64_t i, int q, int Gg, const KCfg& cfg, const Smem& s,
                                         GroupSync* gs, bool skip, unsigned sum_use, int L, int Ls, int Wm, int Wn,
                                         int64_t c0, int validV, int64_t r0, int validU, int pitchU, int pitchV,
                                         bool wtd) {
    const int tid = threadIdx.x;
    const int64_t m = P.m, n = P.n;
    const int64_t kk = P.k;
    // the stored component (written by the lead CTA at least one exchange ago;
    // with k = 1 one more exchange orders it), read through L2
    if (kk == 1) {
        double unused;
        if (!exchange_sum(P.sums, q, Gg, 0.0, s.red, gs, cfg.limit_ns, P.status, skip, sum_use, unused))
            return -1;
    }
    __threadfence();
    const int nV0 = build_from_trits(reinterpret_cast<const uint32_t*>(P.C + i * P.c_bytes), P.c_bytes / 4, n, s.nzV,
                                     s.sgV, s.vlist, pitchU, s);
    const int nU0 = build_from_trits(reinterpret_cast<const uint32_t*>(P.B + i * P.b_bytes), P.b_bytes / 4, m, s.nzU,
                                     s.sgU, s.ulist, pitchV, s);
    double hv0 = (double)nV0;   // v_i^T diag(h~) v_i (nnz(v_i) for the plain objective)
    if (wtd) {
        double acc = 0.0;
        for (int w = tid; w < Wn; w += NT)
            for (uint32_t mk = s.nzV[w]; mk; mk &= mk - 1u)
                acc += (double)__ldg(P.hw + ((int64_t)w << 5) + __ffs(mk) - 1);
        hv0 = block_sum(acc, s.red);
    }
    const double di = __ldcg(P.dk + i);
    if (tid == 0) {
        s.scal[8] = di;
        s.scal[9] = (double)nU0 * hv0;
        s.scal[11] = (double)L;
    }
    // add d_i u_i v_i^T back: a pending term with coefficient -d_i
    push_pending(s, L, Ls, -di, Wm, Wn, c0, validV, r0, validU);
    for (int w = tid; w < Wn; w += NT) { s.nzV[w] = 0u; s.sgV[w] = 0u; }
    __syncthreads();
    return nU0;
}

// Test-hook trace of one half-step (lead CTA): the published output vector (the
// values the threshold saw), the threshold and the resulting trits.
// (Kept out of line: inlined at its two call sites it made the half-step loop spill
// several times more.)
__device__ __noinline__ void trace_halfstep(const unsigned long long* gvec, int64_t len, double thr, const uint32_t* nz,
                                            const uint32_t* sg, double* pre, double* thr_out, uint8_t* trits,
                                            int64_t row_bytes) {
    for (int64_t t = threadIdx.x; t < len; t += NT) pre[t] = untag(ld_relaxed_u64(gvec + t));
    if (threadIdx.x == 0) *thr_out = thr;
    pack_row(nz, sg, (int)((len + 31) >> 5), reinterpret_cast<uint32_t*>(trits), row_bytes / 4);
}

// Factor (or run one debug half-step of) one matrix with this CTA group.
// Returns false if the group aborted.
template <bool WTD, bool SWP>
__device__ bool run_problem(const Prob& P, int q, const KCfg& cfg, const Smem& s, GroupSync* gs, unsigned& arrivals) {
    const int64_t m = P.m, n = P.n;
    const int Wm = (int)((m + 31) >> 5), Wn = (int)((n + 31) >> 5);
    const int mode = P.mode;
    const int Gg = cfg.Gg;
    const int tid = threadIdx.x;
    const bool lead = (q == 0);
    const bool skip = (cfg.fault_skip == q);
    constexpr bool wtd = WTD;   // §2.5 importance-weighted objective (P.hw set)
    const double tauV = P.tau / (double)n, tauU = P.tau / (double)m;   // T_tau: tau / length, times sum |x|
    const int Ls = cfg.Lcap > 0 ? cfg.Lcap : 1;   // stride of the word-major pending masks

    float* blkV = P.Rv + P.pv.block_offset(q, m);
    const int pitchV = P.pv.pitch(q);
    const int64_t c0 = P.pv.start(q);
    const int validV = (int)(P.pv.end(q) - c0);
    float* blkU = P.Ru + P.pu.block_offset(q, n);
    const int pitchU = P.pu.pitch(q);
    const int64_t r0 = P.pu.start(q);
    const int validU = (int)(P.pu.end(q) - r0);

    if (__ldcg(P.nonfinite) != 0u) {
        if (lead && tid == 0) atomicExch(P.status, ST_ENONFINITE);
        return true;
    }
    if (__ldcg(P.nonfinite + 1) != 0u) {   // importance weights not finite, negative or all zero
        if (lead && tid == 0) atomicExch(P.status, ST_EINVAL);
        return true;
    }
    double N0 = 1.0;
    if (mode == MODE_FACTOR) {
        double ps = 0.0;
        for (int64_t t = tid; t < P.n_norm_part; t += NT) ps += __ldcg(P.norm_part + t);
        N0 = block_sum(ps, s.red);
        if (!(N0 > 0.0)) {
            if (lead && tid == 0) atomicExch(P.status, ST_EZERO);
            return true;
        }
    }
    for (int c = tid; c < pitchV; c += NT) { s.cnzV[c] = 0u; s.csgV[c] = 0u; }
    for (int c = tid; c < pitchU; c += NT) { s.cnzU[c] = 0u; s.csgU[c] = 0u; }
    __syncthreads();

    double RN2 = N0;
    int L = 0;
    // test hook: rank-1 terms d_j u_j v_j^T supplied by the caller, held pending (not yet
    // folded into R) exactly as the factorization holds its own recent components
    for (int j = 0; j < P.n_pend; ++j) {
        build_from_trits(P.pend_u + j * (P.b_bytes / 4), P.b_bytes / 4, m, s.nzU, s.sgU, s.ulist, pitchV, s);
        build_from_trits(P.pend_v + j * (P.c_bytes / 4), P.c_bytes / 4, n, s.nzV, s.sgV, s.vlist, pitchU, s);
        push_pending(s, L, Ls, P.pend_d[j], Wm, Wn, c0, validV, r0, validU);
        ++L;
    }
    unsigned long long sum_nu = 0, sum_nv = 0, sum_du = 0, sum_dv = 0, sum_nunv = 0, hs = 0, fb = 0, sgh = 0;
    const int64_t kk = (mode == MODE_FACTOR) ? P.k : 1;
    // §2.4 refinement sweeps: visits kk .. nvis-1 revisit components 0 .. kk-1 in order.
    // (Little of this is held in registers across the visit loop: the half-steps already
    // use most of a thread's registers.)  s.scal[12] counts the visits that kept the
    // stored pair.
    const int64_t nvis = kk * (int64_t)(1 + ((SWP && mode == MODE_FACTOR) ? P.sweeps : 0));
    if constexpr (SWP) if (tid == 0) s.scal[12] = 0.0;
    int nU = 0, nV = 0, dU = 0, dV = 0;   // support sizes and list lengths (trit changes)
    double hsv = 0.0;                     // weighted objective: sum of h~ over the support of v
    double p = 0.0, thr;
    unsigned gen = 0;   // half-step counter of this matrix (tags of the exchanged words)
    HalfCorr hcV{s.coef, s.cnzV, s.csgV, s.corr, s.gV, 0};
    HalfCorr hcU{s.coefV, s.cnzU, s.csgU, s.corr, s.gU, 0};
    if (blockIdx.x == 0 && tid == 0) {
        for (int k2 = 0; k2 < 11; ++k2) s.clk[k2] = 0ull;
        s.clk[11] = (unsigned long long)clock64();
    }

    for (int64_t vis = 0; vis < nvis; ++vis) {
        const int64_t i = vis % kk;
        const bool refine = SWP && vis >= kk;   // a refinement visit of component i
        const bool trv = P.tr_pre_v != nullptr && lead && vis >= P.tr_first && vis - P.tr_first < P.tr_count;
        // refinement state in shared memory (s.scal[8..11]): d_i, n_old = nnz(u_i) v_i^T diag(h~) v_i,
        // this CTA's part of p_old, and the pending slot of the added-back term
        // a new component: the GEMV sums restart from zero and the previous trits
        // of the output vectors are zero, so the first lists hold whole supports
        for (int c = tid; c < pitchV; c += NT) s.gV[c] = 0.0;
        for (int c = tid; c < pitchU; c += NT) s.gU[c] = 0.0;
        if (mode != MODE_HALF_U) {
            if constexpr (SWP) if (refine) {
                const int nU0 = refine_begin(P, i, q, Gg, cfg, s, gs, skip, sum_use_start(vis - kk), L, Ls, Wm, Wn, c0, validV, r0,
                                             validU, pitchU, pitchV, wtd);
                if (nU0 < 0) return false;
                ++L;
                nU = nU0;   // the refit starts from the stored u
            }
            if (!refine) {
                for (int w = tid; w < Wn; w += NT) { s.nzV[w] = 0u; s.sgV[w] = 0u; }
                nU = build_from_trits(P.start + i * P.start_words, P.start_words, m, s.nzU, s.sgU, s.ulist, pitchV, s);
            }
            dU = nU;
            if (L > 0) pending_coef(L, Ls, Wm, s.pnzU, s.psgU, s.nzU, s.sgU, s.pd, s.dotU, s.coef);
            for (int l = tid; l < L; l += NT) {
                s.dotV[l] = 0;
                s.coefV[l] = 0.0;
                if (wtd) s.dotVw[l] = 0.0;
            }
        } else {
            for (int w = tid; w < Wm; w += NT) { s.nzU[w] = 0u; s.sgU[w] = 0u; }
            nV = build_from_trits(P.start, P.start_words, n, s.nzV, s.sgV, s.vlist, pitchU, s);
            dV = nV;
        }
        phase_mark(s, 7);
        for (int it = 0; it < P.iters; ++it) {
            if (mode != MODE_HALF_U) {
                // ---- V-step: x = R^T u on this CTA's columns (§2.3 step 1, first half)
                phase_mark(s, 6);
                const unsigned tg = gen_tag(++gen);
                double S;
                hcV.L = L;
                gemv_dispatch<false>(P.pv.vec, blkV, pitchV, validV, c0, s.ulist, nullptr, dU, s.red, P.xbuf, hcV, tg, skip, S, s.clk);
                phase_mark(s, 1);
                bool ok = true;
                const int nv2 = exchange_threshold<WTD>(P.partV, q, Gg, tg, arrivals, skip, S, P.xbuf, n, tauV, s.nzV,
                                                   s.sgV, s.onzV, s.osgV, s.vlist, pitchU, s, L, Ls, s.pnzV, s.psgV,
                                                   s.dotV, s.coefV, false, thr, dV, gs, cfg.limit_ns, P.status, ok,
                                                   wtd ? P.hw : nullptr, wtd ? s.vwl : nullptr, s.dotVw, &hsv);
                if (!ok) return false;
                if constexpr (SWP) if (refine && it == 0) {
                    // u_i^T R (h~ v_i) of the added-back residual: x = R^T u_i at this CTA's columns
                    const int La = (int)s.scal[11];
                    double pold_part = 0.0;
                    for (int c = tid; c < validV; c += NT) {
                        if ((s.cnzV[c] >> La) & 1u) {
                            double x = untag(ld_relaxed_u64(P.xbuf + c0 + c));
                            if (wtd) x *= (double)__ldg(P.hw + c0 + c);
                            pold_part += ((s.csgV[c] >> La) & 1u) ? -x : x;
                        }
                    }
                    pold_part = block_sum(pold_part, s.red);
                    if (tid == 0) s.scal[10] = pold_part;
                }
                if (trv) {
                    const int64_t at = (vis - P.tr_first) * P.iters + it;
                    trace_halfstep(P.xbuf, n, thr, s.nzV, s.sgV, P.tr_pre_v + at * n, P.tr_thr_v + at,
                                   P.tr_trit_v + at * P.c_bytes, P.c_bytes);
                }
                fb += (s.scal[1] != 0.0) ? 1 : 0;
                sum_nu += (unsigned long long)nU;
                sum_du += (unsigned long long)dU;
                nV = nv2;
                ++hs;
                if (mode == MODE_HALF_V) {
                    if (lead) {
                        for (int64_t t = tid; t < n; t += NT) P.pre_out[t] = untag(ld_relaxed_u64(P.xbuf + t));
                        if (tid == 0) *P.thr_out = thr;
                        pack_row(s.nzV, s.sgV, Wn, reinterpret_cast<uint32_t*>(P.trit_out), P.c_bytes / 4);
                        __syncthreads();
                        if (tid == 0) { __threadfence(); atomicExch(P.status, ST_OK); }
                    }
                    return true;
                }
            }
            // ---- U-step: y = R v on this CTA's rows (§2.3 step 1, second half)
            phase_mark(s, 6);
            const unsigned tg = gen_tag(++gen);
            double S;
            hcU.L = L;
            gemv_dispatch<WTD>(P.pu.vec, blkU, pitchU, validU, r0, s.vlist, wtd ? s.vwl : nullptr, dV, s.red, P.ybuf, hcU, tg, skip,
                          S, s.clk);
            phase_mark(s, 1);
            bool ok = true;
            sum_nv += (unsigned long long)nV;
            sum_dv += (unsigned long long)dV;
            nU = exchange_threshold<false>(P.partU, q, Gg, tg, arrivals, skip, S, P.ybuf, m, tauU, s.nzU, s.sgU, s.onzU,
                                    s.osgU, s.ulist, pitchV, s, L, Ls, s.pnzU, s.psgU, s.dotU, s.coef, true, thr, dU,
                                    gs, cfg.limit_ns, P.status, ok);
            if (!ok) return false;
            if (trv) {
                const int64_t at = (vis - P.tr_first) * P.iters + it;
                trace_halfstep(P.ybuf, m, thr, s.nzU, s.sgU, P.tr_pre_u + at * m, P.tr_thr_u + at,
                               P.tr_trit_u + at * P.b_bytes, P.b_bytes);
            }
            p = s.scal[0];
            fb += (s.scal[1] != 0.0) ? 1 : 0;
            ++hs;
            if (mode == MODE_HALF_U) {
                if (lead) {
                    for (int64_t t = tid; t < m; t += NT) P.pre_out[t] = untag(ld_relaxed_u64(P.ybuf + t));
                    if (tid == 0) *P.thr_out = thr;
                    pack_row(s.nzU, s.sgU, Wm, reinterpret_cast<uint32_t*>(P.trit_out), P.b_bytes / 4);
                    __syncthreads();
                    if (tid == 0) { __threadfence(); atomicExch(P.status, ST_OK); }
                }
                return true;
            }
            // A U-step that changed no trit of u ends the alternation: the next V-step would
            // see the same u (an empty change list, unchanged sums and corrections), hence give
            // the same x, v, y and u, and so would every later iteration.  Stopping here yields
            // exactly the factors of all `iters` iterations.  (dU is the same in every CTA.)
            // Refits start next to their fixed point, so this matters in the instantiation with
            // refinement sweeps; first fits rarely settle within 15 iterations, and in the plain
            // instantiations the extra exit costs registers, so they run every iteration.
            if (SWP && dU == 0) break;
        }
        // ---- scale (§2.3 step 2): d = u^T R v / (nnz(u) nnz(v)), with u^T R v = u^T y = p;
        //      weighted (§2.5): d = u^T R (h~ v) / (nnz(u) sum_{v != 0} h~), the decrease p d
        const double dnew = (p == 0.0) ? 0.0 : p / ((double)nU * (wtd ? hsv : (double)nV));
        double d = dnew;
        bool take = true;   // store the refit (always, outside refinement)
        if constexpr (SWP) if (refine) {
            // §2.4 refinement: the residual grew by the added-back term,
            // ||R + d_i u_i v_i^T||^2 = ||R||^2 + 2 d_i p_old - d_i^2 n_old with p_old = u_i^T R_added (h~ v_i);
            // keep the refit if its decrease p dnew is at least the stored pair's p_old^2 / n_old
            const double di = s.scal[8], n_old = s.scal[9];
            const int La = (int)s.scal[11];
            double pold = 0.0;
            if (!exchange_sum(P.sums, q, Gg, tid == 0 ? s.scal[10] : 0.0, s.red, gs, cfg.limit_ns, P.status, skip,
                              sum_use_end(vis - kk, kk),
                              pold))
                return false;
            RN2 += 2.0 * di * pold - di * di * n_old;
            const double dold = (pold == 0.0 || n_old == 0.0) ? 0.0 : pold / n_old;
            take = (p * dnew >= pold * dold);
            RN2 -= take ? p * dnew : pold * dold;
            d = take ? dnew : dold;
            if (tid == 0 && !take) {
                s.scal[12] += 1.0;
                s.pd[La] = dold - di;   // net pending term of the stored pair
            }
        }
        // §7 safeguard condition: the ALS decrease p d below the single-entry bound ||R||^2 / (m n)
        // (counted, not substituted; RN2 is ||R||^2 before this component)
        if (!refine) {
            sgh += (p * dnew < RN2 / ((double)m * (double)n)) ? 1ull : 0ull;
            RN2 -= p * dnew;
        }
        sum_nunv += (unsigned long long)nU * (unsigned long long)nV;
        if (lead) {
            // (selects rather than branches on `take` keep the half-step loop's register allocation)
            pack_row(s.nzU, s.sgU, Wm, reinterpret_cast<uint32_t*>(P.B + i * P.b_bytes), take ? P.b_bytes / 4 : 0);
            pack_row(s.nzV, s.sgV, Wn, reinterpret_cast<uint32_t*>(P.C + i * P.c_bytes), take ? P.c_bytes / 4 : 0);
            if (tid == 0) {
                P.D[i] = (float)d;
                if (P.energy && !refine) P.energy[i] = 1.0 - RN2 / N0;
                if (P.d64) P.d64[i] = d;
                if (P.dk) P.dk[i] = d;
                if (refine && i == kk - 1 && P.sweep_energy) P.sweep_energy[vis / kk - 1] = 1.0 - RN2 / N0;
            }
            if (SWP) __threadfence();   // the other CTAs re-read this component in the next sweep
        }
        // ---- deflation (§2.3 step 3), held lazily as a pending rank-1 term; a refinement
        //      visit that kept the stored pair pushes the refit with coefficient 0 (the
        //      pair's new scale sits in its added-back slot)
        push_pending(s, L, Ls, take ? d : 0.0, Wm, Wn, c0, validV, r0, validU);
        ++L;
        phase_mark(s, 8);
        // room for the next visit's terms (two during refinement; extraction folds on the
        // plain schedule, so its rounding is that of a run without sweeps), and R folded
        // at the end of the extraction and of the run
        if (L + (vis + 1 >= kk ? 2 : 1) > cfg.Lcap || vis == kk - 1 || vis == nvis - 1) {
            uint32_t* scratch = reinterpret_cast<uint32_t*>(s.red);
            flush_dispatch(P.pv.vec, blkV, P.Rv_lo + P.pv.block_offset(q, m), pitchV, m, validV, L, Ls, s.pd, s.pnzU,
                           s.psgU, s.cnzV, s.csgV, scratch);
            flush_dispatch(P.pu.vec, blkU, P.Ru_lo + P.pu.block_offset(q, n), pitchU, n, validU, L, Ls, s.pd, s.pnzV,
                           s.psgV, s.cnzU, s.csgU, scratch);
            __syncthreads();
            for (int c = tid; c < pitchV; c += NT) { s.cnzV[c] = 0u; s.csgV[c] = 0u; }
            for (int c = tid; c < pitchU; c += NT) { s.cnzU[c] = 0u; s.csgU[c] = 0u; }
            L = 0;
            __syncthreads();
        }
        phase_mark(s, 9);
    }

    // ---- explicit ||R_k||^2 from the folded residual hi + lo (V-layout covers all of R)
    double rs = 0.0;
    if (validV > 0) {
        const float* bloV = P.Rv_lo + P.pv.block_offset(q, m);
        const int64_t tot = m * (int64_t)validV;
        for (int64_t t = tid; t < tot; t += NT) {
            const int64_t r = t / validV;
            const int c = (int)(t - r * validV);
            const double v = (double)__ldcg(blkV + r * pitchV + c) + (double)__ldcg(bloV + r * pitchV + c);
            rs += v * v * (wtd ? (double)__ldg(P.hw + c0 + c) : 1.0);
        }
    }
    double R2 = 0.0;
    // the final sum follows the refinement visits' calls
    const unsigned last_use = (nvis > kk) ? sum_use_end(nvis - kk - 1, kk) : 0u;
    if (!exchange_sum(P.sums, q, Gg, rs, s.red, gs, cfg.limit_ns, P.status, skip, last_use + 1u, R2)) return false;
    if (lead && tid == 0) {
        P.stats->sum_nu = sum_nu;
        P.stats->sum_nv = sum_nv;
        P.stats->sum_du = sum_du;
        P.stats->sum_dv = sum_dv;
        P.stats->sum_nunv = sum_nunv;
        P.stats->half_steps = hs;
        P.stats->fallbacks = fb;
        P.stats->residual2 = R2;
        P.stats->norm_a2 = N0;
        P.stats->sweep_kept = SWP ? (unsigned long long)s.scal[12] : 0ull;
        P.stats->safeguard = sgh;
        phase_mark(s, 7);
        for (int k2 = 0; k2 < 11; ++k2) P.stats->phase[k2] = s.clk[k2];
        __threadfence();
        atomicExch(P.status, ST_OK);
    }
    __syncthreads();
    return true;
}

template <bool WTD, bool SWP>
__global__ void __launch_bounds__(NT, 1) als_kernel(const KCfg cfg) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int grp = blockIdx.x / cfg.Gg;
    const int q = blockIdx.x - grp * cfg.Gg;
    const int Lc = cfg.Lcap > 0 ? cfg.Lcap : 1;
    const SmemLayout lay(cfg.m_max, cfg.n_max, Lc, cfg.pv_max, cfg.pu_max, cfg.weighted);
    Smem s;
    s.red = reinterpret_cast<double*>(smem_raw + lay.red);
    s.pd = reinterpret_cast<double*>(smem_raw + lay.pd);
    s.coef = reinterpret_cast<double*>(smem_raw + lay.coef);
    s.coefV = reinterpret_cast<double*>(smem_raw + lay.coefV);
    s.dotU = reinterpret_cast<int*>(smem_raw + lay.dotU);
    s.dotV = reinterpret_cast<int*>(smem_raw + lay.dotV);
    s.scal = reinterpret_cast<double*>(smem_raw + lay.scal);
    s.wS = reinterpret_cast<double*>(smem_raw + lay.wS);
    s.wM = reinterpret_cast<double*>(smem_raw + lay.wM);
    s.wp = reinterpret_cast<double*>(smem_raw + lay.wp);
    s.gS = reinterpret_cast<double*>(smem_raw + lay.gS);
    s.gM = reinterpret_cast<double*>(smem_raw + lay.gM);
    s.wJ = reinterpret_cast<long long*>(smem_raw + lay.wJ);
    s.gJ = reinterpret_cast<long long*>(smem_raw + lay.gJ);
    s.wc = reinterpret_cast<int*>(smem_raw + lay.wc);
    s.dotp = reinterpret_cast<int*>(smem_raw + lay.dotp);
    s.sflag = reinterpret_cast<int*>(smem_raw + lay.sflag);
    s.clk = reinterpret_cast<unsigned long long*>(smem_raw + lay.clk);
    s.nzU = reinterpret_cast<uint32_t*>(smem_raw + lay.nzU);
    s.sgU = reinterpret_cast<uint32_t*>(smem_raw + lay.sgU);
    s.nzV = reinterpret_cast<uint32_t*>(smem_raw + lay.nzV);
    s.sgV = reinterpret_cast<uint32_t*>(smem_raw + lay.sgV);
    s.pnzU = reinterpret_cast<uint32_t*>(smem_raw + lay.pnzU);
    s.psgU = reinterpret_cast<uint32_t*>(smem_raw + lay.psgU);
    s.pnzV = reinterpret_cast<uint32_t*>(smem_raw + lay.pnzV);
    s.psgV = reinterpret_cast<uint32_t*>(smem_raw + lay.psgV);
    s.cnzV = reinterpret_cast<uint32_t*>(smem_raw + lay.cnzV);
    s.csgV = reinterpret_cast<uint32_t*>(smem_raw + lay.csgV);
    s.cnzU = reinterpret_cast<uint32_t*>(smem_raw + lay.cnzU);
    s.csgU = reinterpret_cast<uint32_t*>(smem_raw + lay.csgU);
    s.ulist = reinterpret_cast<int*>(smem_raw + lay.ulist);
    s.vlist = reinterpret_cast<int*>(smem_raw + lay.vlist);
    s.wd = reinterpret_cast<int*>(smem_raw + lay.wd);
    s.onzU = reinterpret_cast<uint32_t*>(smem_raw + lay.onzU);
    s.osgU = reinterpret_cast<uint32_t*>(smem_raw + lay.osgU);
    s.onzV = reinterpret_cast<uint32_t*>(smem_raw + lay.onzV);
    s.osgV = reinterpret_cast<uint32_t*>(smem_raw + lay.osgV);
    s.vwl = reinterpret_cast<float*>(smem_raw + lay.vwl);
    s.dotVw = reinterpret_cast<double*>(smem_raw + lay.dotVw);
    s.dotpw = reinterpret_cast<double*>(smem_raw + lay.dotpw);
    s.gV = reinterpret_cast<double*>(smem_raw + lay.gV);
    s.gU = reinterpret_cast<double*>(smem_raw + lay.gU);
    s.corr = reinterpret_cast<double*>(smem_raw + lay.corr);

    GroupSync* gs = cfg.gsync + grp;
    unsigned arrivals = 0;   // exchanges this CTA took part in (counter targets)
    for (int pi = grp; pi < cfg.nprob; pi += cfg.NG) {
        if (!run_problem<WTD, SWP>(cfg.probs[pi], q, cfg, s, gs, arrivals)) return;
    }
}

}  // namespace externd

#include "als_cluster.cuh"
#ifndef EXTERND_SECONDARY
#include "block_als.cuh"
#endif

namespace externd {

// Writes one problem descriptor and its running status into a caller-fixed workspace.
// The four instantiations: importance weights (§2.5) x refinement sweeps (§2.4).
static const void* als2_fn(int weighted) {
    return weighted ? (const void*)als2_kernel<true> : (const void*)als2_kernel<false>;
}

static const void* als_fn(int weighted, int sweeping) {
    if (weighted) return sweeping ? (const void*)als_kernel<true, true> : (const void*)als_kernel<true, false>;
    return sweeping ? (const void*)als_kernel<false, true> : (const void*)als_kernel<false, false>;
}

__global__ void init_control_kernel(const Prob p, Prob* dst, int* status) {
    if (threadIdx.x == 0) {
        *dst = p;
        *status = ST_RUNNING;
    }
}

// ---------------------------------------------------------------------------
// Reconstruction Ahat = B diag(D) C (§2.1), fp64 accumulation
// ---------------------------------------------------------------------------

constexpr int RKC = 64;

__device__ __forceinline__ int trit_at(const uint8_t* row, int64_t x) {
    const int code = (row[x >> 2] >> (2 * (x & 3))) & 3;
    return code == 1 ? 1 : (code == 3 ? -1 : 0);
}

__global__ void __launch_bounds__(256) reconstruct_kernel(const uint8_t* __restrict__ B, const float* __restrict__ D,
                                                          const uint8_t* __restrict__ C, int64_t m, int64_t n,
                                                          int64_t k, int64_t bb, int64_t cb, float* __restrict__ out) {
    __shared__ signed char sb[RKC][32];
    __shared__ signed char sc[RKC][32];
    __shared__ double sd[RKC];
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int tid = ty * 32 + tx;
    const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int64_t i0 = 0; i0 < k; i0 += RKC) {
        for (int t = tid; t < RKC * 32; t += 256) {
            const int ii = t >> 5, x = t & 31;
            const int64_t i = i0 + ii;
            int b = 0, c = 0;
            if (i < k) {
                if (r0 + x < m) b = trit_at(B + i * bb, r0 + x);
                if (c0 + x < n) c = trit_at(C + i * cb, c0 + x);
            }
            sb[ii][x] = (signed char)b;
            sc[ii][x] = (signed char)c;
        }
        for (int t = tid; t < RKC; t += 256) sd[t] = (i0 + t < k) ? (double)D[i0 + t] : 0.0;
        __syncthreads();
        for (int ii = 0; ii < RKC; ++ii) {
            const int c = sc[ii][tx];
            if (c) {
                const double dc = c > 0 ? sd[ii] : -sd[ii];
                #pragma unroll
                for (int rr = 0; rr < 4; ++rr) {
                    const int b = sb[ii][ty + 8 * rr];
                    if (b) acc[rr] += b > 0 ? dc : -dc;
                }
            }
        }
        __syncthreads();
    }
    #pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
        const int64_t r = r0 + ty + 8 * rr, c = c0 + tx;
        if (r < m && c < n) out[r * n + c] = (float)acc[rr];
    }
}

}  // namespace externd

// ===========================================================================
// Host side
// ===========================================================================

using namespace externd;

namespace {

struct DevInfo {
    int sms = 0;
    size_t smem_optin = 0;
    int coop = 0;
    bool attr_set = false;
    bool valid = false;
};

std::mutex g_mu;
DevInfo g_dev[64];
thread_local externd_stats g_last = {};

int dev_info(DevInfo& out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return EXTERND_ECUDA; }
    std::lock_guard<std::mutex> lk(g_mu);
    DevInfo& d = g_dev[dev & 63];
    if (!d.valid) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) { cudaGetLastError(); return EXTERND_ECUDA; }
        d.sms = v;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) { cudaGetLastError(); return EXTERND_ECUDA; }
        d.smem_optin = (size_t)v;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess) { cudaGetLastError(); return EXTERND_ECUDA; }
        d.coop = v;
        bool attr_ok = true;
        for (int w = 0; w < 2; ++w)
            for (int sw = 0; sw < 2; ++sw)
                attr_ok = attr_ok && cudaFuncSetAttribute(als_fn(w, sw), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                          (int)d.smem_optin) == cudaSuccess;
        for (int w = 0; w < 2; ++w) {
            attr_ok = attr_ok && cudaFuncSetAttribute(als2_fn(w), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      (int)d.smem_optin) == cudaSuccess;
            // clusters of 16 CTAs need the non-portable size
            if (cudaFuncSetAttribute(als2_fn(w), cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)
                cudaGetLastError();
        }
        if (!attr_ok) {
            cudaGetLastError();
            return EXTERND_ECUDA;
        }
        cudaMemPool_t pool;
        if (cudaDeviceGetDefaultMemPool(&pool, dev) == cudaSuccess) {
            uint64_t thr = UINT64_MAX;
            cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &thr);
        }
        cudaGetLastError();
        d.valid = true;
    }
    out = d;
    return EXTERND_OK;
}

bool is_device_ptr(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) { cudaGetLastError(); return false; }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int64_t rank_of(int64_t m, int64_t n, double mu) {
    if (m < 1 || n < 1 || !std::isfinite(mu)) return -1;
    const double x = mu * (double)(m < n ? m : n);
    if (!(x >= 0.5) || x > 9.0e18) return -1;
    const int64_t k = (int64_t)std::llround(x);
    return k >= 1 ? k : -1;
}

size_t trit_bytes(int64_t len) { return len < 1 ? 0 : round_up((size_t)((len + 3) / 4), 16); }

// Vector width of a stripe layout: minimise the largest stripe's GEMV cost,
// (units per stripe) * width * (instructions per element at that width).
int choose_vec(int64_t len, int G) {
    int best = 4;
    double best_cost = 1e300;
    for (int vec : {4, 2, 1}) {
        const double per_elem = vec == 4 ? 2.25 : (vec == 2 ? 3.5 : 6.0);
        const int64_t units = (len + vec - 1) / vec;
        const int64_t maxu = (units + G - 1) / G;
        const double cost = (double)(maxu * vec) * per_elem;
        if (cost < best_cost * (1.0 - 1e-9)) { best_cost = cost; best = vec; }
    }
    return best;
}

Part make_part(int64_t len, int G, int vec) {
    Part p;
    p.len = len;
    p.vec = vec;
    p.G = G;
    p.units = (len + vec - 1) / vec;
    return p;
}

size_t als_smem_bytes(int64_t m_max, int64_t n_max, int L, int pv_max, int pu_max, int weighted) {
    return SmemLayout(m_max, n_max, L > 0 ? L : 1, pv_max, pu_max, weighted).total;
}

struct ProbIn {
    const float* A;
    const float* h;       // §2.5 per-column second moments (n), or null for the plain objective
    double lambda;
    int64_t m, n, k;
    double tau;
    int iters;
    uint64_t seed;
    uint8_t* B;
    float* D;
    uint8_t* C;
    double* energy;
    double* d64;
    int sweeps;           // §2.4 refinement sweeps (MODE_FACTOR only)
    double* sweep_energy; // nullable, sweeps values
    int mode;
    const uint8_t* dbg_in;
    double* pre_out;
    double* thr_out;
    uint8_t* trit_out;
    // test hooks (device pointers)
    const uint8_t* start_in;  // caller-given start trits of component 0 (k = 1), or null
    int n_pend;
    const double* pend_d;
    const uint8_t* pend_u;
    const uint8_t* pend_v;
    int64_t tr_first, tr_count;
    double *tr_pre_v, *tr_thr_v, *tr_pre_u, *tr_thr_u;
    uint8_t *tr_trit_v, *tr_trit_u;
};

struct RunOpts {
    int grid = 0;
    int pending = 0;
    double wait_limit_s = 2.0;
    int fault_skip = -1;
    bool init_only = false;
    bool plan_only = false;   // fill the stats with the launch plan and return (no device work)
    int cluster = 0;          // 0: automatic; 1: the one-CTA-per-stripe kernel; 2, 4, 8, 16: clusters of that size
    int* async_status = nullptr;   // device int: queue everything, write the status there, do not wait
    int block = 0;            // threads per CTA: 0 automatic, else 256, 512 or 1024
};

// Status of an asynchronous call: the first matrix's failure (a group that stopped before a
// matrix finished counts as a timeout), else EXTERND_OK.
__global__ void async_status_kernel(const int* __restrict__ status, int np, int* out) {
    if (threadIdx.x != 0) return;
    int r = EXTERND_OK;
    for (int b = 0; b < np && r == EXTERND_OK; ++b) {
        const int s = status[b];
        r = (s == ST_RUNNING) ? EXTERND_ETIMEOUT : s;
    }
    *out = r;
}

// Plan of the clustered kernel for one launch (see als_cluster.cuh).
struct Plan2 {
    bool ok = false;
    int c = 0, Gg = 0, Lcap = 0, ncl = 0;
    size_t smem = 0;
    int qr_max = 1, qc_max = 1, sv_max = 1, su_max = 1, wpm = 1;
    std::vector<Grid2> g;
    std::vector<int64_t> bsv, bsu;
};

// Try clusters of size c for groups of G CTAs (a multiple of c).  pl.ncl reports how many
// such clusters can be resident at once.
Plan2 plan_cluster(const ProbIn* in, int np, int NG, int G, int c, int Lreq, int weighted, const DevInfo& di) {
    Plan2 pl;
    if (G < c || G % c != 0 || G > NT) return pl;
    const int NC = G / c;
    int64_t m_max = 1, n_max = 1;
    pl.g.resize(np);
    pl.bsv.resize(np);
    pl.bsu.resize(np);
    for (int b = 0; b < np; ++b) {
        Grid2& g = pl.g[b];
        g.m = in[b].m;
        g.n = in[b].n;
        g.c = c;
        g.NC = NC;
        g.vecv = 4;   // the clustered kernel reads its blocks in 16-byte vectors
        g.vecu = 4;
        m_max = in[b].m > m_max ? in[b].m : m_max;
        n_max = in[b].n > n_max ? in[b].n : n_max;
        const Part QR = g.qr(), QC = g.qc();
        int64_t bsv = 1, bsu = 1;
        for (int r = 0; r < c; ++r) {
            pl.qr_max = (int)std::max<int64_t>(pl.qr_max, QR.end(r) - QR.start(r));
            pl.qc_max = (int)std::max<int64_t>(pl.qc_max, QC.end(r) - QC.start(r));
            for (int q = 0; q < NC; ++q) {
                pl.wpm = std::max(pl.wpm, std::max(g.pcol(r).pitch(q), g.prow(r).pitch(q)));
            }
        }
        for (int q = 0; q < NC; ++q) {
            const int pv = g.pitchV(q), pu = g.pitchU(q);
            pl.sv_max = std::max(pl.sv_max, pv);
            pl.su_max = std::max(pl.su_max, pu);
            for (int r = 0; r < c; ++r) {
                bsv = std::max<int64_t>(bsv, (QR.end(r) - QR.start(r)) * (int64_t)pv);
                bsu = std::max<int64_t>(bsu, (QC.end(r) - QC.start(r)) * (int64_t)pu);
            }
        }
        // list entries hold element offsets below 2^30
        if ((double)bsv >= 1073741824.0 || (double)bsu >= 1073741824.0) return pl;
        pl.bsv[b] = (bsv + 63) / 64 * 64;
        pl.bsu[b] = (bsu + 63) / 64 * 64;
    }
    int L = MAX_PENDING;
    auto smem_of = [&](int Lc) {
        return SmemLayout2(m_max, n_max, pl.qr_max, pl.qc_max, pl.sv_max, pl.su_max, pl.wpm, pl.wpm, c, Lc, weighted).total;
    };
    while (L > 1 && smem_of(L) > di.smem_optin) --L;
    if (Lreq > 0 && Lreq < L) L = Lreq;
    if (smem_of(L) > di.smem_optin) return pl;
    pl.smem = smem_of(L);
    // every cluster of the launch must be resident at once
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(NG * G));
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = pl.smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int ncl = 0;
    if (cudaOccupancyMaxActiveClusters(&ncl, als2_fn(weighted), &cfg) != cudaSuccess) {
        cudaGetLastError();
        return pl;
    }
    pl.ncl = ncl;
    if ((int64_t)ncl < (int64_t)NG * NC) return pl;
    pl.ok = true;
    pl.c = c;
    pl.Gg = G;
    pl.Lcap = L;
    return pl;
}

struct Buf {  // device staging for a possibly-host pointer
    void* host = nullptr;
    void* dev = nullptr;
    size_t bytes = 0;
    bool staged = false;
};

#define CK(call)                                                   \
    do {                                                           \
        cudaError_t e_ = (call);                                   \
        if (e_ != cudaSuccess) {                                   \
            cudaGetLastError();                                    \
            rc = (e_ == cudaErrorMemoryAllocation) ? EXTERND_ENOMEM : EXTERND_ECUDA; \
            goto done;                                             \
        }                                                          \
    } while (0)

// Runs setup + init + ALS for `np` problems.  All pointers in `in` may be
// host or device.  statuses[np] receives per-problem status.
// Caller-fixed workspace (no allocation, no host-side copies, no events).
struct FixedWs {
    unsigned char* base = nullptr;
    size_t cap = 0;
};

#ifndef EXTERND_SECONDARY
// Threads per CTA of the one-CTA-per-stripe kernel for a plan of G CTAs per matrix.  A CTA's
// work per half-step grows with its share of the residual (the stripe its GEMV reads, m n / G
// elements) and with the whole vector it thresholds (m or n entries: 8 (m + n) weighs them like
// stripe elements).  Fewer threads shorten the barrier-bound chain of a half-step; more threads
// pay once the share is large.  Measured on B200 (ALS time, 15 iterations): 256 threads are
// fastest below W = 170k -- single matrices of 1024^2 to 2048^2 at 65k elements per CTA run
// 7-20 % faster than at 512, 256^2 on one CTA 23 % -- 512 up to 230k (2560 x 6912 over 148 CTAs,
// W = 196k: 4 % ahead of 256, 3 % of 1024), 1024 above (16 matrices of 1536^2 over 9 CTAs
// each, W = 287k: 12 % ahead of 512; 2560 x 6912 over 74 CTAs, W = 315k: 8 %).  Refinement
// sweeps are the exception below 170k: their refits of stored components ran 18 % slower at 256
// threads than at 512 (1024^2 with ten sweeps: 9636 against 10669 fits/s), so plans with sweeps
// take 512 there.
constexpr int AUTO_MIN_DEPTH = 8;   // a shorter pending list folds the residual every few components
int auto_block(double work_max, int64_t m_max, int64_t n_max, int G, bool sweeping) {
    const double W = work_max / G + 8.0 * (double)(m_max + n_max);
    if (W >= 230000.0) return 1024;
    return (W < 170000.0 && !sweeping) ? 256 : 512;
}
#endif

int run(const ProbIn* in, int np, const RunOpts& opt, cudaStream_t stream, int* statuses,
        const FixedWs* fixed = nullptr) {
    int rc = EXTERND_OK;
    DevInfo di;
    if ((rc = dev_info(di)) != EXTERND_OK) return rc;
    if (!di.coop) return EXTERND_ELAUNCH;

    externd_stats st = {};
    const int sms = di.sms;

    // ---- grouping: NG groups of Gg CTAs; a group factors problems g, g+NG, ...
    int64_t m_max = 1, n_max = 1;
    double work_max = 0;
    for (int b = 0; b < np; ++b) {
        m_max = in[b].m > m_max ? in[b].m : m_max;
        n_max = in[b].n > n_max ? in[b].n : n_max;
        work_max = (double)in[b].m * in[b].n > work_max ? (double)in[b].m * in[b].n : work_max;
    }
    int NG = np < sms ? np : sms;
    int Gg;
    if (opt.grid > 0) {
        Gg = opt.grid;
        if ((int64_t)Gg * NG > sms) NG = sms / Gg > 0 ? sms / Gg : 1;
    } else {
        Gg = sms / NG;
        const int64_t want = (int64_t)std::ceil(work_max / 65536.0);
        if (want < Gg) Gg = (int)(want > 0 ? want : 1);
    }
    // no empty stripes
    for (int b = 0; b < np; ++b) {
        if (Gg > in[b].m) Gg = (int)in[b].m;
        if (Gg > in[b].n) Gg = (int)in[b].n;
    }
    if (Gg < 1) Gg = 1;
#ifndef EXTERND_SECONDARY
    // ---- block size: the caller's, else by the work of one CTA (the clustered kernel: 512)
    if (opt.cluster <= 1) {
        bool sweeps = false;
        for (int b = 0; b < np; ++b) sweeps = sweeps || (in[b].mode == MODE_FACTOR && in[b].sweeps > 0);
        int nt = opt.block > 0 ? opt.block : auto_block(work_max, m_max, n_max, Gg, sweeps);
        if (opt.block == 0 && nt == 1024) {
            // the 1024-thread layout keeps more shared state per CTA, so on the largest shapes it
            // leaves a shorter lazy-deflation depth, or none: below AUTO_MIN_DEPTH the 512-thread plan
            // is kept (every shape the 512-thread build can plan stays plannable)
            RunOpts probe = opt;
            probe.plan_only = true;
            probe.pending = 0;
            externd_stats pst = {};
            std::vector<int> pstat(np, 0);
            if (externd_run_nt1024(in, np, &probe, stream, pstat.data(), &pst, nullptr, 0) != EXTERND_OK ||
                pst.pending < AUTO_MIN_DEPTH)
                nt = 512;
        }
        if (nt != NT) {
            externd_stats st2 = {};
            const int rc2 = (nt == 256 ? externd_run_nt256 : externd_run_nt1024)(
                in, np, &opt, stream, statuses, &st2, fixed ? fixed->base : nullptr, fixed ? fixed->cap : 0);
            if (!fixed) g_last = st2;   // the allocation-free call leaves the stats alone
            return rc2;
        }
    }
#endif

    // ---- lazy deflation depth from the shared-memory budget
    if (Gg > NT) Gg = NT;   // one thread per CTA of the group polls its stripe
    std::vector<int> vecv(np), vecu(np);
    int pv_max = 1, pu_max = 1;
    for (int b = 0; b < np; ++b) {
        vecv[b] = choose_vec(in[b].n, Gg);
        vecu[b] = choose_vec(in[b].m, Gg);
        const int64_t uv = (in[b].n + vecv[b] - 1) / vecv[b], uu = (in[b].m + vecu[b] - 1) / vecu[b];
        const int pv = (int)(((uv + Gg - 1) / Gg) * vecv[b]), pu = (int)(((uu + Gg - 1) / Gg) * vecu[b]);
        pv_max = pv > pv_max ? pv : pv_max;
        pu_max = pu > pu_max ? pu : pu_max;
    }
    for (int b = 0; b < np; ++b)
        if ((double)in[b].m * pv_max >= 1073741824.0 || (double)in[b].n * pu_max >= 1073741824.0) return EXTERND_ELIMIT;
    int Lcap = MAX_PENDING;
    // one launch runs one objective: every problem weighted, or none
    int weighted = 0;
    for (int b = 0; b < np; ++b) weighted += (in[b].h != nullptr);
    if (weighted != 0 && weighted != np) return EXTERND_EINVAL;
    weighted = weighted ? 1 : 0;
    while (Lcap > 1 && als_smem_bytes(m_max, n_max, Lcap, pv_max, pu_max, weighted) > di.smem_optin) --Lcap;
    if (opt.pending > 0 && opt.pending < Lcap) Lcap = opt.pending;
    for (int b = 0; b < np; ++b) {
        if (in[b].mode == MODE_FACTOR && in[b].sweeps > 0 && Lcap < 2) return EXTERND_ELIMIT;   // add-back + refit
        if (in[b].n_pend > 0 && in[b].n_pend + 1 > Lcap) return EXTERND_ELIMIT;   // caller's terms + the component
    }
    size_t smem = als_smem_bytes(m_max, n_max, Lcap, pv_max, pu_max, weighted);
    if (smem > di.smem_optin) return EXTERND_ELIMIT;

    int nb = 0;
    int sweeping = 0;
    for (int b = 0; b < np; ++b) sweeping |= (in[b].mode == MODE_FACTOR && in[b].sweeps > 0);
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, als_fn(weighted, sweeping), NT, smem) != cudaSuccess) {
        cudaGetLastError();
        return EXTERND_ECUDA;
    }
    if ((int64_t)nb * sms < (int64_t)NG * Gg) return EXTERND_ELAUNCH;

    // ---- the clustered kernel (factorizations without refinement sweeps), where its
    //      clusters can all be resident; the largest cluster size that keeps at least 85 %
    //      of the CTAs asked for (small matrices: a group of up to 16 CTAs, one word of
    //      32 indices per quarter at least)
    Plan2 pl;
    if (!opt.init_only && opt.cluster > 1 && !sweeping) {
        bool all_factor = true;
        int64_t mn_min = INT64_MAX;
        for (int b = 0; b < np; ++b) {
            all_factor = all_factor && in[b].mode == MODE_FACTOR;
            mn_min = std::min<int64_t>(mn_min, std::min(in[b].m, in[b].n));
        }
        if (all_factor) {
            int Gt = Gg;
            if (opt.grid <= 0 && Gt < 16) {
                const int64_t want = std::min<int64_t>(16, std::max<int64_t>(2, (mn_min + 31) / 32));
                if ((int64_t)NG * want <= sms) Gt = (int)want;
            }
            for (int c : {16, 8, 4, 2}) {
                if (opt.cluster > 1 && c != opt.cluster) continue;
                if (c > Gt) continue;
                Plan2 t = plan_cluster(in, np, NG, (Gt / c) * c, c, opt.pending, weighted, di);
                if (!t.ok && opt.grid <= 0 && t.ncl >= NG) {   // fewer clusters per matrix, as many as fit
                    const int G1 = (t.ncl / NG) * c;
                    if (G1 >= c && G1 < (Gt / c) * c) t = plan_cluster(in, np, NG, G1, c, opt.pending, weighted, di);
                }
                if (t.ok && (opt.cluster > 1 || opt.grid > 0 || t.Gg * 100 >= Gt * 85)) {
                    pl = t;
                    break;
                }
            }
            if (opt.cluster > 1 && !pl.ok) return EXTERND_ELAUNCH;   // the size asked for does not fit
        }
    }
    const bool clustered = pl.ok;
    if (clustered) {
        Gg = pl.Gg;
        Lcap = pl.Lcap;
        smem = pl.smem;
    }

    if (opt.plan_only) {
        st.grid = NG * Gg;
        st.group = Gg;
        st.block = NT;
        st.pending = Lcap;
        st.cluster = clustered ? pl.c : 1;
        st.smem_bytes = smem;
        g_last = st;
        for (int b = 0; b < np; ++b) statuses[b] = EXTERND_OK;
        return EXTERND_OK;
    }

    // ---- plan the workspace
    std::vector<Prob> probs(np);
    std::vector<size_t> off_rv(np), off_ru(np), off_rvl(np), off_rul(np), off_x(np), off_y(np), off_sums(np), off_start(np), off_norm(np), off_A(np),
        off_B(np), off_C(np), off_D(np), off_E(np), off_d64(np), off_pre(np), off_thr(np), off_tro(np), off_hw(np), off_h(np),
        off_dk(np), off_SE(np);
    size_t ctl = 0;
    const size_t off_gsync = ctl;
    ctl += round_up(sizeof(GroupSync) * NG, 256);
    const size_t off_status = ctl;
    ctl += round_up(sizeof(int) * np, 256);
    const size_t off_nonfin = ctl;
    ctl += round_up(sizeof(unsigned) * 2 * np, 256);
    const size_t off_stats = ctl;
    ctl += round_up(sizeof(DevStats) * np, 256);
    const size_t off_probs = ctl;
    ctl += round_up(sizeof(Prob) * np, 256);
    size_t ws = ctl;
    const size_t zero_from = ws;
    for (int b = 0; b < np; ++b) {
        const ProbIn& I = in[b];
        const int vv = vecv[b], vu = vecu[b];
        Prob& P = probs[b];
        memset(&P, 0, sizeof(P));
        P.m = I.m; P.n = I.n; P.k = I.k; P.tau = I.tau; P.iters = I.iters; P.mode = I.mode; P.seed = I.seed;
        P.pv = make_part(I.n, Gg, vv);
        P.pu = make_part(I.m, Gg, vu);
        P.b_bytes = (int64_t)trit_bytes(I.m);
        P.c_bytes = (int64_t)trit_bytes(I.n);
        P.start_words = (int64_t)trit_bytes(I.mode == MODE_HALF_U ? I.n : I.m) / 4;
        P.start_given = I.start_in != nullptr;
        P.n_pend = I.n_pend;
        P.pend_d = I.pend_d;
        P.pend_u = reinterpret_cast<const uint32_t*>(I.pend_u);
        P.pend_v = reinterpret_cast<const uint32_t*>(I.pend_v);
        P.tr_first = I.tr_first;
        P.tr_count = I.tr_count;
        P.tr_pre_v = I.tr_pre_v; P.tr_thr_v = I.tr_thr_v; P.tr_trit_v = I.tr_trit_v;
        P.tr_pre_u = I.tr_pre_u; P.tr_thr_u = I.tr_thr_u; P.tr_trit_u = I.tr_trit_u;
        P.n_norm_part = ((I.m + 31) / 32) * ((I.n + 31) / 32);
        if (clustered) {
            P.g2 = pl.g[b];
            P.bsv = pl.bsv[b];
            P.bsu = pl.bsu[b];
        }
        const size_t rv_elems = clustered ? (size_t)Gg * (size_t)pl.bsv[b] : (size_t)P.pv.total(I.m);
        const size_t ru_elems = clustered ? (size_t)Gg * (size_t)pl.bsu[b] : (size_t)P.pu.total(I.n);
        off_rv[b] = ws; ws += round_up(sizeof(float) * rv_elems, 256);
        off_ru[b] = ws; ws += round_up(sizeof(float) * ru_elems, 256);
        // low halves of the residual (zero until the first fold)
        off_rvl[b] = ws; ws += round_up(sizeof(float) * rv_elems, 256);
        off_rul[b] = ws; ws += round_up(sizeof(float) * ru_elems, 256);
        // exchange buffers: zero = "no half-step yet" (tags are 1..255)
        off_x[b] = ws; ws += round_up(sizeof(unsigned long long) * (size_t)I.n, 256);
        off_y[b] = ws; ws += round_up(sizeof(unsigned long long) * (size_t)I.m, 256);
        off_sums[b] = ws; ws += round_up(sizeof(unsigned long long) * (size_t)Gg * 4, 256);   // sums x2, partV, partU
    }
    const size_t zero_to = ws;
    for (int b = 0; b < np; ++b) {
        const ProbIn& I = in[b];
        Prob& P = probs[b];
        const int64_t srows = (I.mode == MODE_FACTOR) ? I.k : 1;
        off_start[b] = ws; ws += round_up(sizeof(uint32_t) * (size_t)(P.start_words * srows), 256);
        off_norm[b] = ws; ws += round_up(sizeof(double) * (size_t)P.n_norm_part, 256);
        off_hw[b] = off_h[b] = SIZE_MAX;
        if (I.h) {
            off_hw[b] = ws; ws += round_up(sizeof(float) * (size_t)I.n, 256);
            if (!is_device_ptr(I.h)) { off_h[b] = ws; ws += round_up(sizeof(float) * (size_t)I.n, 256); }
        }
        // staging for host pointers
        off_A[b] = SIZE_MAX;
        if (I.A && !is_device_ptr(I.A)) { off_A[b] = ws; ws += round_up(sizeof(float) * (size_t)(I.m * I.n), 256); }
        off_B[b] = off_C[b] = off_D[b] = off_E[b] = off_d64[b] = off_pre[b] = off_thr[b] = off_tro[b] = SIZE_MAX;
        off_dk[b] = off_SE[b] = SIZE_MAX;
        if (I.mode == MODE_FACTOR && !opt.init_only && I.sweeps > 0) {
            off_dk[b] = ws; ws += round_up(sizeof(double) * (size_t)I.k, 256);
            if (I.sweep_energy && !is_device_ptr(I.sweep_energy)) {
                off_SE[b] = ws; ws += round_up(sizeof(double) * (size_t)I.sweeps, 256);
            }
        }
        if (I.mode == MODE_FACTOR && !opt.init_only) {
            if (!is_device_ptr(I.B)) { off_B[b] = ws; ws += round_up((size_t)(I.k * P.b_bytes), 256); }
            if (!is_device_ptr(I.C)) { off_C[b] = ws; ws += round_up((size_t)(I.k * P.c_bytes), 256); }
            if (!is_device_ptr(I.D)) { off_D[b] = ws; ws += round_up(sizeof(float) * (size_t)I.k, 256); }
            if (I.energy && !is_device_ptr(I.energy)) { off_E[b] = ws; ws += round_up(sizeof(double) * (size_t)I.k, 256); }
            if (I.d64 && !is_device_ptr(I.d64)) { off_d64[b] = ws; ws += round_up(sizeof(double) * (size_t)I.k, 256); }
        } else if (I.mode != MODE_FACTOR) {
            const int64_t lin = I.mode == MODE_HALF_V ? I.m : I.n;
            const int64_t lout = I.mode == MODE_HALF_V ? I.n : I.m;
            (void)lin;
            if (!is_device_ptr(I.pre_out)) { off_pre[b] = ws; ws += round_up(sizeof(double) * (size_t)lout, 256); }
            if (!is_device_ptr(I.thr_out)) { off_thr[b] = ws; ws += 256; }
            if (!is_device_ptr(I.trit_out)) { off_tro[b] = ws; ws += round_up(trit_bytes(lout), 256); }
        }
    }

    const bool async = opt.async_status != nullptr;
    if (fixed || async) {
        for (int b = 0; b < np; ++b)
            if (off_A[b] != SIZE_MAX || off_B[b] != SIZE_MAX || off_C[b] != SIZE_MAX || off_D[b] != SIZE_MAX ||
                off_E[b] != SIZE_MAX || off_d64[b] != SIZE_MAX || off_pre[b] != SIZE_MAX || off_thr[b] != SIZE_MAX ||
                off_tro[b] != SIZE_MAX || off_SE[b] != SIZE_MAX || off_h[b] != SIZE_MAX)
                return EXTERND_EINVAL;   // host buffers would need staging memory (and a synchronous copy)
        if (fixed && ws > fixed->cap) return EXTERND_ELIMIT;
        if (async && (fixed || opt.init_only || !is_device_ptr(opt.async_status))) return EXTERND_EINVAL;
        if (async)
            for (int b = 0; b < np; ++b)
                if (in[b].mode != MODE_FACTOR) return EXTERND_EINVAL;
    }
    unsigned char* dws = nullptr;
    cudaEvent_t ev[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
    std::vector<unsigned char> hctl(ctl, 0);
    std::vector<int> hstatus(np, ST_RUNNING);
    std::vector<DevStats> hstats(np);
    int launches = 0;
    float ms_setup = 0, ms_init = 0, ms_als = 0, ms_total = 0;

    if (fixed) {
        dws = fixed->base;
    } else {
        if (!async)
            for (int i = 0; i < 5; ++i) CK(cudaEventCreate(&ev[i]));
        CK(cudaMallocAsync((void**)&dws, ws, stream));
    }
    if (ev[0]) CK(cudaEventRecord(ev[0], stream));

    // ---- fill problem descriptors and the control region
    for (int b = 0; b < np; ++b) {
        const ProbIn& I = in[b];
        Prob& P = probs[b];
        P.A = off_A[b] == SIZE_MAX ? I.A : reinterpret_cast<const float*>(dws + off_A[b]);
        P.hw = off_hw[b] == SIZE_MAX ? nullptr : reinterpret_cast<const float*>(dws + off_hw[b]);
        P.Rv = reinterpret_cast<float*>(dws + off_rv[b]);
        P.Ru = reinterpret_cast<float*>(dws + off_ru[b]);
        P.Rv_lo = reinterpret_cast<float*>(dws + off_rvl[b]);
        P.Ru_lo = reinterpret_cast<float*>(dws + off_rul[b]);
        P.xbuf = reinterpret_cast<unsigned long long*>(dws + off_x[b]);
        P.ybuf = reinterpret_cast<unsigned long long*>(dws + off_y[b]);
        P.sums = reinterpret_cast<unsigned long long*>(dws + off_sums[b]);
        P.partV = P.sums + 2 * Gg;
        P.partU = P.sums + 3 * Gg;
        P.start = reinterpret_cast<uint32_t*>(dws + off_start[b]);
        P.norm_part = reinterpret_cast<double*>(dws + off_norm[b]);
        P.nonfinite = reinterpret_cast<unsigned*>(dws + off_nonfin) + 2 * b;
        P.status = reinterpret_cast<int*>(dws + off_status) + b;
        P.stats = reinterpret_cast<DevStats*>(dws + off_stats) + b;
        if (I.mode == MODE_FACTOR) {
            P.B = off_B[b] == SIZE_MAX ? I.B : dws + off_B[b];
            P.C = off_C[b] == SIZE_MAX ? I.C : dws + off_C[b];
            P.D = off_D[b] == SIZE_MAX ? I.D : reinterpret_cast<float*>(dws + off_D[b]);
            P.energy = off_E[b] == SIZE_MAX ? I.energy : reinterpret_cast<double*>(dws + off_E[b]);
            P.d64 = off_d64[b] == SIZE_MAX ? I.d64 : reinterpret_cast<double*>(dws + off_d64[b]);
            P.sweeps = off_dk[b] == SIZE_MAX ? 0 : I.sweeps;
            P.dk = off_dk[b] == SIZE_MAX ? nullptr : reinterpret_cast<double*>(dws + off_dk[b]);
            P.sweep_energy = off_SE[b] == SIZE_MAX ? (P.sweeps ? I.sweep_energy : nullptr)
                                                   : reinterpret_cast<double*>(dws + off_SE[b]);
        } else {
            P.pre_out = off_pre[b] == SIZE_MAX ? I.pre_out : reinterpret_cast<double*>(dws + off_pre[b]);
            P.thr_out = off_thr[b] == SIZE_MAX ? I.thr_out : reinterpret_cast<double*>(dws + off_thr[b]);
            P.trit_out = off_tro[b] == SIZE_MAX ? I.trit_out : dws + off_tro[b];
        }
        reinterpret_cast<int*>(hctl.data() + off_status)[b] = ST_RUNNING;
    }
    memcpy(hctl.data() + off_probs, probs.data(), sizeof(Prob) * np);
    if (fixed) {
        // control region: zeros, then the descriptors and statuses written by a kernel
        CK(cudaMemsetAsync(dws, 0, ctl, stream));
        for (int b = 0; b < np; ++b) {
            init_control_kernel<<<1, 32, 0, stream>>>(probs[b], reinterpret_cast<Prob*>(dws + off_probs) + b,
                                                      reinterpret_cast<int*>(dws + off_status) + b);
            CK(cudaGetLastError());
        }
    } else {
        CK(cudaMemcpyAsync(dws, hctl.data(), ctl, cudaMemcpyHostToDevice, stream));
    }
    if (zero_to > zero_from) CK(cudaMemsetAsync(dws + zero_from, 0, zero_to - zero_from, stream));
    for (int b = 0; b < np; ++b) {
        const ProbIn& I = in[b];
        if (off_A[b] != SIZE_MAX)
            CK(cudaMemcpyAsync(dws + off_A[b], I.A, sizeof(float) * (size_t)(I.m * I.n), cudaMemcpyHostToDevice, stream));
        if (off_h[b] != SIZE_MAX)
            CK(cudaMemcpyAsync(dws + off_h[b], I.h, sizeof(float) * (size_t)I.n, cudaMemcpyHostToDevice, stream));
        if (off_hw[b] != SIZE_MAX) {
            const float* hsrc = off_h[b] == SIZE_MAX ? I.h : reinterpret_cast<const float*>(dws + off_h[b]);
            weights_kernel<<<1, 1024, 0, stream>>>(hsrc, I.n, I.lambda, reinterpret_cast<float*>(dws + off_hw[b]),
                                                   reinterpret_cast<unsigned*>(dws + off_nonfin) + 2 * b + 1);
            CK(cudaGetLastError());
            ++launches;
        }
        if (I.start_in) {
            // caller-given start trits -> start row of component 0
            CK(cudaMemcpyAsync(dws + off_start[b], I.start_in, (size_t)probs[b].start_words * 4,
                               is_device_ptr(I.start_in) ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice, stream));
        }
        if (I.mode != MODE_FACTOR) {
            // debug input trits -> start row
            const bool dev_in = is_device_ptr(I.dbg_in);
            CK(cudaMemcpyAsync(dws + off_start[b], I.dbg_in, (size_t)probs[b].start_words * 4,
                               dev_in ? cudaMemcpyDeviceToDevice : cudaMemcpyHostToDevice, stream));
        }
    }

    {
        const Prob* dprobs = reinterpret_cast<const Prob*>(dws + off_probs);
        int64_t tx = 1, ty = 1, kmax = 1;
        for (int b = 0; b < np; ++b) {
            tx = (in[b].n + 31) / 32 > tx ? (in[b].n + 31) / 32 : tx;
            ty = (in[b].m + 31) / 32 > ty ? (in[b].m + 31) / 32 : ty;
            kmax = in[b].k > kmax ? in[b].k : kmax;
        }
        if (!opt.init_only) {
            if (clustered)
                setup2_kernel<<<dim3((unsigned)tx, (unsigned)ty, (unsigned)np), dim3(32, 8), 0, stream>>>(dprobs);
            else
                setup_kernel<<<dim3((unsigned)tx, (unsigned)ty, (unsigned)np), dim3(32, 8), 0, stream>>>(dprobs);
            CK(cudaGetLastError());
            ++launches;
        }
        if (ev[1]) CK(cudaEventRecord(ev[1], stream));
        bool any_factor = false;
        for (int b = 0; b < np; ++b) any_factor |= (in[b].mode == MODE_FACTOR);
        if (any_factor) {
            const unsigned gx = (unsigned)(kmax < 8192 ? kmax : 8192);
            init_kernel<<<dim3(gx, (unsigned)np), NTI, 0, stream>>>(dprobs);
            CK(cudaGetLastError());
            ++launches;
        }
        if (ev[2]) CK(cudaEventRecord(ev[2], stream));
        if (!opt.init_only) {
            KCfg cfg;
            cfg.probs = dprobs;
            cfg.nprob = np;
            cfg.Gg = Gg;
            cfg.NG = NG;
            cfg.gsync = reinterpret_cast<GroupSync*>(dws + off_gsync);
            cfg.Lcap = Lcap;
            cfg.m_max = (int)m_max;
            cfg.n_max = (int)n_max;
            cfg.pv_max = pv_max;
            cfg.pu_max = pu_max;
            const double lim = opt.wait_limit_s > 0 ? opt.wait_limit_s : 2.0;
            cfg.limit_ns = (uint64_t)(lim * 1e9);
            cfg.fault_skip = opt.fault_skip;
            cfg.weighted = weighted;
            if (clustered) {
                cfg.pv_max = pl.sv_max;
                cfg.pu_max = pl.su_max;
                cfg.qr_max = pl.qr_max;
                cfg.qc_max = pl.qc_max;
                cfg.wpm = pl.wpm;
                cudaLaunchConfig_t lc = {};
                lc.gridDim = dim3((unsigned)(NG * Gg));
                lc.blockDim = dim3(NT);
                lc.dynamicSmemBytes = smem;
                lc.stream = stream;
                cudaLaunchAttribute attr[2];
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.x = (unsigned)pl.c;
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                attr[1].id = cudaLaunchAttributeCooperative;   // all CTAs resident at once
                attr[1].val.cooperative = 1;
                lc.attrs = attr;
                lc.numAttrs = 2;
                void* args[] = {&cfg};
                CK(cudaLaunchKernelExC(&lc, als2_fn(weighted), args));
            } else {
                void* args[] = {&cfg};
                CK(cudaLaunchCooperativeKernel(als_fn(weighted, sweeping), dim3((unsigned)(NG * Gg)), dim3(NT), args, smem,
                                               stream));
            }
            ++launches;
        }
        if (ev[3]) CK(cudaEventRecord(ev[3], stream));
    }

    // ---- results back to host-side buffers
    for (int b = 0; b < np; ++b) {
        const ProbIn& I = in[b];
        const Prob& P = probs[b];
        if (opt.init_only) {
            if (is_device_ptr(I.B)) CK(cudaMemcpyAsync(I.B, P.start, (size_t)(P.start_words * 4 * I.k), cudaMemcpyDeviceToDevice, stream));
            else CK(cudaMemcpyAsync(I.B, P.start, (size_t)(P.start_words * 4 * I.k), cudaMemcpyDeviceToHost, stream));
            continue;
        }
        if (off_B[b] != SIZE_MAX) CK(cudaMemcpyAsync(I.B, P.B, (size_t)(I.k * P.b_bytes), cudaMemcpyDeviceToHost, stream));
        if (off_C[b] != SIZE_MAX) CK(cudaMemcpyAsync(I.C, P.C, (size_t)(I.k * P.c_bytes), cudaMemcpyDeviceToHost, stream));
        if (off_D[b] != SIZE_MAX) CK(cudaMemcpyAsync(I.D, P.D, sizeof(float) * (size_t)I.k, cudaMemcpyDeviceToHost, stream));
        if (off_E[b] != SIZE_MAX) CK(cudaMemcpyAsync(I.energy, P.energy, sizeof(double) * (size_t)I.k, cudaMemcpyDeviceToHost, stream));
        if (off_d64[b] != SIZE_MAX) CK(cudaMemcpyAsync(I.d64, P.d64, sizeof(double) * (size_t)I.k, cudaMemcpyDeviceToHost, stream));
        if (off_SE[b] != SIZE_MAX)
            CK(cudaMemcpyAsync(I.sweep_energy, P.sweep_energy, sizeof(double) * (size_t)I.sweeps, cudaMemcpyDeviceToHost, stream));
        if (I.mode != MODE_FACTOR) {
            const int64_t lout = I.mode == MODE_HALF_V ? I.n : I.m;
            if (off_pre[b] != SIZE_MAX) CK(cudaMemcpyAsync(I.pre_out, P.pre_out, sizeof(double) * (size_t)lout, cudaMemcpyDeviceToHost, stream));
            if (off_thr[b] != SIZE_MAX) CK(cudaMemcpyAsync(I.thr_out, P.thr_out, sizeof(double), cudaMemcpyDeviceToHost, stream));
            if (off_tro[b] != SIZE_MAX) CK(cudaMemcpyAsync(I.trit_out, P.trit_out, trit_bytes(lout), cudaMemcpyDeviceToHost, stream));
        }
    }
    if (async) {
        // the batch's status into the caller's int when the stream gets here; the workspace is
        // released in stream order below and the call returns without waiting
        async_status_kernel<<<1, 32, 0, stream>>>(reinterpret_cast<const int*>(dws + off_status), np, opt.async_status);
        CK(cudaGetLastError());
        ++launches;
        st.launches = launches;
        st.grid = NG * Gg;
        st.group = Gg;
        st.block = NT;
        st.vec_v = probs[0].pv.vec;
        st.vec_u = probs[0].pu.vec;
        st.pending = Lcap;
        st.cluster = clustered ? pl.c : 1;
        st.smem_bytes = smem;
        st.workspace_bytes = ws;
        for (int b = 0; b < np; ++b) statuses[b] = EXTERND_OK;
        rc = EXTERND_OK;
        goto done;
    }
    CK(cudaMemcpyAsync(hstatus.data(), dws + off_status, sizeof(int) * np, cudaMemcpyDeviceToHost, stream));
    CK(cudaMemcpyAsync(hstats.data(), dws + off_stats, sizeof(DevStats) * np, cudaMemcpyDeviceToHost, stream));
    if (ev[4]) CK(cudaEventRecord(ev[4], stream));
    CK(cudaStreamSynchronize(stream));

    if (ev[0]) {
        cudaEventElapsedTime(&ms_setup, ev[0], ev[1]);
        cudaEventElapsedTime(&ms_init, ev[1], ev[2]);
        cudaEventElapsedTime(&ms_als, ev[2], ev[3]);
        cudaEventElapsedTime(&ms_total, ev[0], ev[4]);
    }
    st.setup_ms = ms_setup;
    st.init_ms = ms_init;
    st.als_ms = ms_als;
    st.total_ms = ms_total;
    st.launches = launches;
    st.grid = NG * Gg;
    st.group = Gg;
    st.block = NT;
    st.vec_v = probs[0].pv.vec;
    st.vec_u = probs[0].pu.vec;
    st.pending = Lcap;
    st.cluster = clustered ? pl.c : 1;
    st.smem_bytes = smem;
    st.workspace_bytes = ws;
    for (int b = 0; b < np; ++b) {
        int s = hstatus[b];
        if (opt.init_only) s = ST_OK;
        if (s == ST_RUNNING) s = EXTERND_ETIMEOUT;   // group aborted before this matrix finished
        statuses[b] = s;
        if (s == ST_OK && in[b].mode == MODE_FACTOR && !opt.init_only) {
            const DevStats& d = hstats[b];
            st.alg_bytes += 4.0 * ((double)in[b].n * (double)d.sum_nu + (double)in[b].m * (double)d.sum_nv) +
                            8.0 * (double)d.sum_nunv;
            st.read_bytes += 4.0 * ((double)in[b].n * (double)d.sum_du + (double)in[b].m * (double)d.sum_dv) +
                             8.0 * (double)d.sum_nunv;
            st.components += in[b].k;
            st.half_steps += (int64_t)d.half_steps;
            st.fallbacks += (int64_t)d.fallbacks;
            if (b == 0) {
                st.residual_energy = d.norm_a2 > 0 ? 1.0 - d.residual2 / d.norm_a2 : 0.0;
                for (int k2 = 0; k2 < 11; ++k2) st.phase_cycles[k2] = (int64_t)d.phase[k2];
                st.sweep_kept = (int64_t)d.sweep_kept;
            }
            st.safeguard_hits += (int64_t)d.safeguard;
        }
    }
    rc = EXTERND_OK;
    for (int b = 0; b < np; ++b)
        if (statuses[b] != ST_OK) { rc = statuses[b]; break; }

done:
    // an asynchronous call that queued everything frees its workspace in stream order and returns;
    // every other exit waits for the work it queued
    if (dws && !fixed) {
        cudaFreeAsync(dws, stream);
        if (!(async && rc == EXTERND_OK)) cudaStreamSynchronize(stream);
    }
    // fixed scratch: work already queued on the shared array must end before the
    // call returns, also when a later queueing step failed
    if (fixed && rc != EXTERND_OK) cudaStreamSynchronize(stream);
    for (int i = 0; i < 5; ++i)
        if (ev[i]) cudaEventDestroy(ev[i]);
    cudaGetLastError();
    if (!fixed) g_last = st;   // the allocation-free call records no events and leaves the stats alone
    return rc;
}

// Trace buffers of the test hooks: all device memory, trit rows 16-byte aligned, the
// window inside [0, visits) (k extraction visits, then k per refinement sweep).
int check_trace(int64_t first, int64_t count, int64_t k, const double* pv, const double* tv, const uint8_t* rv,
                const double* pu, const double* tu, const uint8_t* ru) {
    if (first < 0 || count < 1 || first + count > k) return EXTERND_EINVAL;
    const void* ptrs[6] = {pv, tv, rv, pu, tu, ru};
    for (const void* q : ptrs)
        if (!q || !is_device_ptr(q)) return EXTERND_EINVAL;
    if ((reinterpret_cast<uintptr_t>(rv) & 15u) || (reinterpret_cast<uintptr_t>(ru) & 15u)) return EXTERND_EINVAL;
    return EXTERND_OK;
}

#ifdef EXTERND_SECONDARY
// Entry of a secondary build (another block size): the primary build validated the arguments and
// chose the block size; this build plans and runs the call, in the caller-fixed workspace if any.
int run_secondary(const void* in, int np, const void* opt, cudaStream_t stream, int* statuses, externd_stats* stats,
                  void* fixed_base, size_t fixed_cap) {
    FixedWs fw;
    fw.base = static_cast<unsigned char*>(fixed_base);
    fw.cap = fixed_cap;
    const int rc = run(static_cast<const ProbIn*>(in), np, *static_cast<const RunOpts*>(opt), stream, statuses,
                       fixed_base ? &fw : nullptr);
    *stats = g_last;
    return rc;
}
#endif

// Threads per CTA asked of the one-CTA-per-stripe kernel: 0 (automatic), 256, 512 or 1024; the
// clustered kernel (cluster > 1) runs at 512 only.
bool block_ok(int block, int cluster) {
    if (block != 0 && block != 256 && block != 512 && block != 1024) return false;
    return cluster <= 1 || block == 0 || block == 512;
}

int check_rows_aligned(const void* p) {
    return (reinterpret_cast<uintptr_t>(p) & 15u) == 0 ? EXTERND_OK : EXTERND_EINVAL;
}

int validate_factor(const float* A, int64_t m, int64_t n, double mu, double tau, int iters, const uint8_t* B,
                    const float* D, const uint8_t* C, int64_t* k_out) {
    if (!A || !B || !D || !C) return EXTERND_EINVAL;
    if (m < 1 || n < 1 || iters < 1) return EXTERND_EINVAL;
    if (!std::isfinite(mu) || !std::isfinite(tau) || tau < 0) return EXTERND_EINVAL;
    const int64_t k = rank_of(m, n, mu);
    if (k < 1) return EXTERND_EINVAL;
    if (m > INT_MAX / 2 || n > INT_MAX / 2 || k > INT_MAX) return EXTERND_ELIMIT;
    if (check_rows_aligned(B) || check_rows_aligned(C)) return EXTERND_EINVAL;
    *k_out = k;
    return EXTERND_OK;
}

}  // namespace

#ifndef EXTERND_SECONDARY
namespace {

// §2.4 batched block ALS on the device: blocks of b components, each a sequence of launches on
// `stream` (kernels in block_als.cuh; the plain GEMMs, Cholesky factorizations and solves in
// cuBLAS / cuSOLVER).  A and the outputs are device pointers.
// The vendor-library handles of one call: created on the current device at the start and
// destroyed at the end (a few milliseconds against a factorization of hundreds), so no handle
// outlives its context and concurrent calls share nothing.
struct Linalg {
    cublasHandle_t blas = nullptr;
    cusolverDnHandle_t sol = nullptr;
    bool open(cudaStream_t stream) {
        if (cublasCreate(&blas) != CUBLAS_STATUS_SUCCESS) { blas = nullptr; return false; }
        if (cusolverDnCreate(&sol) != CUSOLVER_STATUS_SUCCESS) { sol = nullptr; return false; }
        return cublasSetStream(blas, stream) == CUBLAS_STATUS_SUCCESS &&
               cusolverDnSetStream(sol, stream) == CUSOLVER_STATUS_SUCCESS;
    }
    ~Linalg() {
        if (sol) cusolverDnDestroy(sol);
        if (blas) cublasDestroy(blas);
    }
};

int run_block(const float* A, int64_t m, int64_t n, int64_t k, double tau, int iters, uint64_t seed, int b,
              uint8_t* B, float* D, uint8_t* C, double* E, double* d64, cudaStream_t stream, externd_stats& st) {
    int rc = EXTERND_OK;
    const int64_t bb = std::min<int64_t>(b, k);
    const int64_t nblocks = (k + bb - 1) / bb;
    const int ninfo = (int)(nblocks * (2 * (int64_t)iters + 1));   // one word per factorization
    const size_t f8 = sizeof(double);
    const int nparts = 296;
    Linalg lh;
    Linalg* la = &lh;
    if (!lh.open(stream)) { cudaGetLastError(); return EXTERND_ECUDA; }
    int lwork = 0;
    if (cusolverDnDpotrf_bufferSize(la->sol, CUBLAS_FILL_MODE_LOWER, (int)bb, nullptr, (int)bb, &lwork) !=
        CUSOLVER_STATUS_SUCCESS)
        return EXTERND_ECUDA;
    size_t off = 0;
    auto take = [&](size_t bytes) { const size_t at = off; off += round_up(bytes, 256); return at; };
    const size_t oR = take(f8 * (size_t)(m * n)), oU = take(f8 * (size_t)(m * bb)), oV = take(f8 * (size_t)(n * bb)),
                 oP = take(f8 * (size_t)(bb * n)), oQ = take(f8 * (size_t)(m * bb)), oS = take(f8 * (size_t)(m * bb)),
                 oGu = take(f8 * (size_t)(bb * bb)), oGv = take(f8 * (size_t)(bb * bb)), oL = take(f8 * (size_t)(bb * bb)),
                 oH = take(f8 * (size_t)(bb * bb)), orhs = take(f8 * (size_t)bb), opart = take(f8 * nparts),
                 oscal = take(f8 * 4), owork = take(f8 * (size_t)std::max(lwork, 1)),
                 oinfo = take(sizeof(int) * (size_t)(ninfo + 1)), oflag = take(sizeof(int) * 4);
    unsigned char* w = nullptr;
    cudaEvent_t e0 = nullptr, e1 = nullptr;
    int hflag[4] = {0, 0, 0, 0};
    double hn0 = 0.0;
    int launches = 0;
    float ms = 0.f;
    bool la_ok = true;
    CK(cudaEventCreate(&e0));
    CK(cudaEventCreate(&e1));
    CK(cudaMallocAsync((void**)&w, off, stream));
    CK(cudaEventRecord(e0, stream));
    {
        double *R = (double*)(w + oR), *U = (double*)(w + oU), *V = (double*)(w + oV), *PT = (double*)(w + oP),
               *Q = (double*)(w + oQ), *S = (double*)(w + oS), *Gu = (double*)(w + oGu), *Gv = (double*)(w + oGv),
               *Lm = (double*)(w + oL), *H = (double*)(w + oH), *rhs = (double*)(w + orhs), *part = (double*)(w + opart),
               *scal = (double*)(w + oscal), *work = (double*)(w + owork);
        int* info = (int*)(w + oinfo);
        int* flag = (int*)(w + oflag);
        CK(cudaMemsetAsync(flag, 0, sizeof(int) * 4, stream));
        CK(cudaMemsetAsync(info, 0, sizeof(int) * (size_t)(ninfo + 1), stream));
        block_setup_kernel<<<592, 256, 0, stream>>>(A, m * n, R, reinterpret_cast<unsigned*>(flag));
        sumsq_kernel<<<nparts, 1024, 0, stream>>>(R, m * n, part);
        sum_partials_kernel<<<1, 1024, 0, stream>>>(part, nparts, scal + 0);   // ||A||^2
        CK(cudaGetLastError());
        launches += 3;
        CK(cudaMemcpyAsync(hflag, flag, sizeof(int), cudaMemcpyDeviceToHost, stream));
        CK(cudaMemcpyAsync(&hn0, scal, sizeof(double), cudaMemcpyDeviceToHost, stream));
        CK(cudaStreamSynchronize(stream));
        if (hflag[0]) { rc = EXTERND_ENONFINITE; goto done; }
        if (!(hn0 > 0.0)) { rc = EXTERND_EZERO; goto done; }
        // row-major C (M x N) = alpha op(A) op(B) + beta C: the column-major product C^T = op(B)^T op(A)^T
        auto gemm = [&](int M, int N, int K, const double* Am, int lda, bool ta, const double* Bm, int ldb, bool tb,
                        double* Cm, int ldc, double alpha, double beta) {
            la_ok = la_ok && cublasDgemm(la->blas, tb ? CUBLAS_OP_T : CUBLAS_OP_N, ta ? CUBLAS_OP_T : CUBLAS_OP_N, N, M, K,
                                         &alpha, Bm, ldb, Am, lda, &beta, Cm, ldc) == CUBLAS_STATUS_SUCCESS;
        };
        // Cholesky of the b x b matrix in Lm, then solve (L L^T) X = Y for nrhs right-hand sides
        // stored as rows of a row-major nrhs x b matrix (= columns of a column-major b x nrhs one)
        auto factor = [&](int nb, double* Mat, int* inf) {
            la_ok = la_ok && cusolverDnDpotrf(la->sol, CUBLAS_FILL_MODE_LOWER, nb, Mat, nb, work, lwork, inf) ==
                                 CUSOLVER_STATUS_SUCCESS;
        };
        auto solve = [&](int nb, const double* Mat, double* Y, int nrhs, int* inf) {
            la_ok = la_ok && cusolverDnDpotrs(la->sol, CUBLAS_FILL_MODE_LOWER, nb, nrhs, Mat, nb, Y, nb, inf) ==
                                 CUSOLVER_STATUS_SUCCESS;
        };
        int slot = 0;
        for (int64_t s0 = 0; s0 < k; s0 += bb) {
            const int nb = (int)std::min<int64_t>(bb, k - s0);
            block_start_kernel<<<nb, 256, 0, stream>>>(seed, s0, m, tau, U, nb);
            ++launches;
            for (int it = 0; it < iters; ++it) {
                // V <- T_tau([(U^T U + eps I)^-1 U^T R]^T) = T_tau(R^T [U (U^T U + eps I)^-1]): the m rows
                // of U are solved (fewer right-hand sides than the n rows of R^T U), then one GEMM
                gemm(nb, nb, (int)m, U, nb, true, U, nb, false, Gu, nb, 1.0, 0.0);
                ridge_kernel<<<1, 1024, 0, stream>>>(Gu, nb, BLOCK_EPS_REL, Lm);
                factor(nb, Lm, info + slot++);
                CK(cudaMemcpyAsync(S, U, f8 * (size_t)(m * nb), cudaMemcpyDeviceToDevice, stream));
                solve(nb, Lm, S, (int)m, info + ninfo);
                gemm((int)n, nb, (int)m, R, (int)n, true, S, nb, false, PT, nb, 1.0, 0.0);
                ternarize_cols_kernel<<<nb, 256, 0, stream>>>(PT, n, nb, tau, V, nb);
                // U <- T_tau(R V (V^T V + eps I)^-1): the rows of Q = R V solved in place
                gemm(nb, nb, (int)n, V, nb, true, V, nb, false, Gv, nb, 1.0, 0.0);
                ridge_kernel<<<1, 1024, 0, stream>>>(Gv, nb, BLOCK_EPS_REL, Lm);
                factor(nb, Lm, info + slot++);
                gemm((int)m, nb, (int)n, R, (int)n, false, V, nb, false, Q, nb, 1.0, 0.0);
                if (it == iters - 1) CK(cudaMemcpyAsync(S, Q, f8 * (size_t)(m * nb), cudaMemcpyDeviceToDevice, stream));
                solve(nb, Lm, Q, (int)m, info + ninfo);
                ternarize_cols_kernel<<<nb, 256, 0, stream>>>(Q, m, nb, tau, U, nb);
                launches += 4;
                CK(cudaGetLastError());
            }
            // joint scales: [(U^T U) o (V^T V)] d = diag(U^T R V), with S = R V of the final V
            gemm(nb, nb, (int)m, U, nb, true, U, nb, false, Gu, nb, 1.0, 0.0);
            block_scale_system_kernel<<<std::max(1, std::min(nb, 148)), 256, 0, stream>>>(Gu, Gv, nb, U, S, m, H, rhs);
            factor(nb, H, info + slot++);
            solve(nb, H, rhs, 1, info + ninfo);
            // deflation R <- R - U diag(d) V^T, energy, outputs
            scale_cols_kernel<<<148, 256, 0, stream>>>(U, m, nb, rhs, S);
            gemm((int)m, (int)n, nb, S, nb, false, V, nb, true, R, (int)n, -1.0, 1.0);
            sumsq_kernel<<<nparts, 1024, 0, stream>>>(R, m * n, part);
            sum_partials_kernel<<<1, 1024, 0, stream>>>(part, nparts, scal + 1);
            block_pack_kernel<<<nb, 128, 0, stream>>>(U, m, nb, nb, s0, B, (int64_t)trit_bytes(m));
            block_pack_kernel<<<nb, 128, 0, stream>>>(V, n, nb, nb, s0, C, (int64_t)trit_bytes(n));
            block_out_kernel<<<1, 256, 0, stream>>>(rhs, nb, s0, scal + 1, scal + 0, D, d64, E);
            launches += 7;
            CK(cudaGetLastError());
            if (!la_ok) { rc = EXTERND_ECUDA; goto done; }
        }
        // a factorization that failed: a ridge system (cannot happen for eps > 0 and finite input)
        // or a scale system that is not positive definite (repeated components in a block)
        info_any_kernel<<<1, 256, 0, stream>>>(info, ninfo + 1, flag + 2);
        ++launches;
        CK(cudaEventRecord(e1, stream));
        CK(cudaMemcpyAsync(hflag, flag, sizeof(int) * 4, cudaMemcpyDeviceToHost, stream));
        CK(cudaStreamSynchronize(stream));
        cudaEventElapsedTime(&ms, e0, e1);
        if (hflag[2]) rc = EXTERND_ELIMIT;
    }
    st.total_ms = ms;
    st.als_ms = ms;
    st.launches = launches;
    st.components = k;
    st.group = (int)bb;   // block width
    st.workspace_bytes = off;
done:
    if (w) { cudaFreeAsync(w, stream); cudaStreamSynchronize(stream); }
    if (e0) cudaEventDestroy(e0);
    if (e1) cudaEventDestroy(e1);
    cudaGetLastError();
    return rc;
}

}  // namespace

// ---------------------------------------------------------------------------
// Scratch memory of externd_factor_noalloc: one file-scope device array,
// EXTERND_NOALLOC_SCRATCH_BYTES on every device that loads this library, kept
// until the process exits.  Host code may not use the array's name as a device
// address (it names a host-side shadow).  The address is looked up with
// cudaGetSymbolAddress on every call, with the caller's device current: a cached
// address could outlive its context (after cudaDeviceReset the module is loaded
// again and the array may sit elsewhere).
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[EXTERND_NOALLOC_SCRATCH_BYTES];

namespace {

// Device address of the scratch array in the current context.
int noalloc_scratch(unsigned char** out) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr) { cudaGetLastError(); return EXTERND_ECUDA; }
    *out = static_cast<unsigned char*>(ptr);
    return EXTERND_OK;
}

}  // namespace

extern "C" {

int64_t externd_rank(int64_t m, int64_t n, double mu) { return rank_of(m, n, mu); }

size_t externd_trit_bytes(int64_t len) { return trit_bytes(len); }

const char* externd_strerror(int status) {
    switch (status) {
        case EXTERND_OK: return "ok";
        case EXTERND_EINVAL: return "invalid argument";
        case EXTERND_EZERO: return "||A||_F = 0: energy undefined";
        case EXTERND_ENONFINITE: return "input holds NaN or Inf";
        case EXTERND_ENOMEM: return "device workspace allocation failed";
        case EXTERND_ECUDA: return "CUDA runtime error";
        case EXTERND_ELAUNCH: return "cooperative ALS grid cannot be co-resident on this device";
        case EXTERND_ETIMEOUT: return "a device-side wait exceeded its limit";
        case EXTERND_ELIMIT: return "shape beyond this build's limits";
        default: return "unknown status";
    }
}

int externd_factor_ex(const float* A, int64_t m, int64_t n, double mu, double tau, int iters, uint64_t seed,
                      uint8_t* B_out, float* D_out, uint8_t* C_out, double* energy_out, void* stream,
                      const externd_options* opt) {
    int64_t k = 0;
    int rc = validate_factor(A, m, n, mu, tau, iters, B_out, D_out, C_out, &k);
    if (rc != EXTERND_OK) return rc;
    ProbIn I = {};
    I.A = A; I.m = m; I.n = n; I.k = k; I.tau = tau; I.iters = iters; I.seed = seed;
    I.B = B_out; I.D = D_out; I.C = C_out; I.energy = energy_out; I.mode = MODE_FACTOR;
    RunOpts ro;
    if (opt) {
        ro.grid = opt->grid;
        ro.pending = opt->pending;
        if (opt->wait_limit_s > 0) ro.wait_limit_s = opt->wait_limit_s;
        ro.fault_skip = opt->fault_inject ? opt->fault_skip_cta : -1;
        if (opt->cluster < 0 || opt->cluster > 16 || (opt->cluster > 1 && (opt->cluster & (opt->cluster - 1))))
            return EXTERND_EINVAL;
        ro.cluster = opt->cluster;
        if (!block_ok(opt->block, opt->cluster)) return EXTERND_EINVAL;
        ro.block = opt->block;
        ro.async_status = opt->async_status;
        I.d64 = opt->d64_out;
        if (opt->sweeps < 0 || opt->sweeps > 1000) return EXTERND_EINVAL;
        I.sweeps = opt->sweeps;
        I.sweep_energy = opt->sweep_energy_out;
        if (opt->h) {
            if (!std::isfinite(opt->lambda) || opt->lambda < 0.0) return EXTERND_EINVAL;
            I.h = opt->h;
            I.lambda = opt->lambda;
        }
        if (opt->trace_pre_v) {
            if ((rc = check_trace(opt->trace_first, opt->trace_count, k * (1 + (int64_t)opt->sweeps), opt->trace_pre_v, opt->trace_thr_v,
                                  opt->trace_trit_v, opt->trace_pre_u, opt->trace_thr_u, opt->trace_trit_u)) != EXTERND_OK)
                return rc;
            I.tr_first = opt->trace_first;
            I.tr_count = opt->trace_count;
            I.tr_pre_v = opt->trace_pre_v; I.tr_thr_v = opt->trace_thr_v; I.tr_trit_v = opt->trace_trit_v;
            I.tr_pre_u = opt->trace_pre_u; I.tr_thr_u = opt->trace_thr_u; I.tr_trit_u = opt->trace_trit_u;
        }
    }
    int st = 0;
    return run(&I, 1, ro, reinterpret_cast<cudaStream_t>(stream), &st);
}

int externd_factor_weighted(const float* A, int64_t m, int64_t n, double mu, double tau, int iters, uint64_t seed,
                            const float* h, double lambda, uint8_t* B_out, float* D_out, uint8_t* C_out,
                            double* energy_out, void* stream) {
    int64_t k = 0;
    int rc = validate_factor(A, m, n, mu, tau, iters, B_out, D_out, C_out, &k);
    if (rc != EXTERND_OK) return rc;
    if (!h || !std::isfinite(lambda) || lambda < 0.0) return EXTERND_EINVAL;
    ProbIn I = {};
    I.A = A; I.m = m; I.n = n; I.k = k; I.tau = tau; I.iters = iters; I.seed = seed;
    I.h = h; I.lambda = lambda;
    I.B = B_out; I.D = D_out; I.C = C_out; I.energy = energy_out; I.mode = MODE_FACTOR;
    RunOpts ro;
    int st = 0;
    return run(&I, 1, ro, reinterpret_cast<cudaStream_t>(stream), &st);
}

int externd_factor(const float* A, int64_t m, int64_t n, double mu, double tau, int iters, uint64_t seed,
                   uint8_t* B_out, float* D_out, uint8_t* C_out, double* energy_out, void* stream) {
    return externd_factor_ex(A, m, n, mu, tau, iters, seed, B_out, D_out, C_out, energy_out, stream, nullptr);
}

int externd_factor_noalloc(const float* A, int64_t m, int64_t n, double mu, double tau, int iters, uint64_t seed,
                           uint8_t* B_out, float* D_out, uint8_t* C_out, double* energy_out, void* stream) {
    int64_t k = 0;
    int rc = validate_factor(A, m, n, mu, tau, iters, B_out, D_out, C_out, &k);
    if (rc != EXTERND_OK) return rc;
    unsigned char* base = nullptr;
    if ((rc = noalloc_scratch(&base)) != EXTERND_OK) return rc;
    ProbIn I = {};
    I.A = A; I.m = m; I.n = n; I.k = k; I.tau = tau; I.iters = iters; I.seed = seed;
    I.B = B_out; I.D = D_out; I.C = C_out; I.energy = energy_out; I.mode = MODE_FACTOR;
    RunOpts ro;
    FixedWs fw;
    fw.base = base;
    fw.cap = EXTERND_NOALLOC_SCRATCH_BYTES;
    int st = 0;
    return run(&I, 1, ro, reinterpret_cast<cudaStream_t>(stream), &st, &fw);
}

int externd_factor_block(const float* A, int64_t m, int64_t n, double mu, double tau, int iters, uint64_t seed, int b,
                         uint8_t* B_out, float* D_out, uint8_t* C_out, double* energy_out, double* d64_out,
                         void* stream) {
    int64_t k = 0;
    int rc = validate_factor(A, m, n, mu, tau, iters, B_out, D_out, C_out, &k);
    if (rc != EXTERND_OK) return rc;
    if (b < 0) return EXTERND_EINVAL;
    const void* ptrs[4] = {A, B_out, D_out, C_out};
    for (const void* q : ptrs)
        if (!is_device_ptr(q)) return EXTERND_EINVAL;
    if ((energy_out && !is_device_ptr(energy_out)) || (d64_out && !is_device_ptr(d64_out))) return EXTERND_EINVAL;
    // §2.4: b = 256 by default, capped at floor(min(m, n) / 8), at least 1
    const int64_t cap = std::max<int64_t>(1, std::min(m, n) / 8);
    const int bw = (int)std::min<int64_t>(b > 0 ? b : 256, b > 0 ? INT_MAX : cap);
    if (m * n > (int64_t)INT_MAX || (int64_t)bw * std::max(m, n) > (int64_t)INT_MAX) return EXTERND_ELIMIT;
    externd_stats st = {};
    rc = run_block(A, m, n, k, tau, iters, seed, bw, B_out, D_out, C_out, energy_out, d64_out,
                   reinterpret_cast<cudaStream_t>(stream), st);
    g_last = st;
    return rc;
}

int externd_factor_batched(int count, const float* const* A, const int64_t* m, const int64_t* n, const double* mu,
                           const double* tau, int iters, const uint64_t* seed, uint8_t* const* B_out,
                           float* const* D_out, uint8_t* const* C_out, double* const* energy_out, int* status_out,
                           void* stream) {
    return externd_factor_batched_ex(count, A, m, n, mu, tau, iters, seed, B_out, D_out, C_out, energy_out,
                                     status_out, stream, nullptr);
}

int externd_factor_batched_ex(int count, const float* const* A, const int64_t* m, const int64_t* n,
                              const double* mu, const double* tau, int iters, const uint64_t* seed,
                              uint8_t* const* B_out, float* const* D_out, uint8_t* const* C_out,
                              double* const* energy_out, int* status_out, void* stream,
                              const externd_batch_options* opt) {
    if (count < 1 || !A || !m || !n || !mu || !tau || !seed || !B_out || !D_out || !C_out || !status_out)
        return EXTERND_EINVAL;
    if (opt) {
        bool bad = opt->sweeps < 0 || opt->sweeps > 1000;
        if (opt->h) {
            for (int b = 0; b < count; ++b) {
                const double lam = opt->lambda ? opt->lambda[b] : 0.0;
                bad = bad || !opt->h[b] || !std::isfinite(lam) || lam < 0.0;
            }
        } else {
            bad = bad || opt->lambda != nullptr;
        }
        if (bad) {
            for (int c = 0; c < count; ++c) status_out[c] = EXTERND_EINVAL;
            return EXTERND_EINVAL;
        }
    }
    std::vector<ProbIn> ins(count);
    for (int b = 0; b < count; ++b) {
        int64_t k = 0;
        const int rc = validate_factor(A[b], m[b], n[b], mu[b], tau[b], iters, B_out[b], D_out[b], C_out[b], &k);
        if (rc != EXTERND_OK) {
            for (int c = 0; c < count; ++c) status_out[c] = (c == b) ? rc : EXTERND_EINVAL;
            return rc;
        }
        ProbIn& I = ins[b];
        memset(&I, 0, sizeof(I));
        I.A = A[b]; I.m = m[b]; I.n = n[b]; I.k = k; I.tau = tau[b]; I.iters = iters; I.seed = seed[b];
        I.B = B_out[b]; I.D = D_out[b]; I.C = C_out[b]; I.energy = energy_out ? energy_out[b] : nullptr;
        I.mode = MODE_FACTOR;
        if (opt) {
            if (opt->h) {
                I.h = opt->h[b];
                I.lambda = opt->lambda ? opt->lambda[b] : 0.0;
            }
            I.sweeps = opt->sweeps;
            I.sweep_energy = opt->sweep_energy_out ? opt->sweep_energy_out[b] : nullptr;
        }
    }
    RunOpts ro;
    if (opt) {
        if (opt->grid < 0 || opt->cluster < 0 || opt->cluster > 16 || (opt->cluster > 1 && (opt->cluster & (opt->cluster - 1))) ||
            !block_ok(opt->block, opt->cluster)) {
            for (int c = 0; c < count; ++c) status_out[c] = EXTERND_EINVAL;
            return EXTERND_EINVAL;
        }
        ro.grid = opt->grid;
        ro.cluster = opt->cluster;
        ro.block = opt->block;
        ro.plan_only = opt->plan_only != 0;
        ro.async_status = opt->async_status;
    }
    return run(ins.data(), count, ro, reinterpret_cast<cudaStream_t>(stream), status_out);
}

int externd_debug_halfstep(const float* R, int64_t m, int64_t n, int transpose, const uint8_t* in_trits, double tau,
                           double* pre_out, double* thresh_out, uint8_t* out_trits, void* stream) {
    if (!R || !in_trits || !pre_out || !thresh_out || !out_trits) return EXTERND_EINVAL;
    if (m < 1 || n < 1 || !std::isfinite(tau) || tau < 0) return EXTERND_EINVAL;
    if (check_rows_aligned(out_trits)) return EXTERND_EINVAL;
    ProbIn I = {};
    I.A = R; I.m = m; I.n = n; I.k = 1; I.tau = tau; I.iters = 1;
    I.mode = transpose ? MODE_HALF_V : MODE_HALF_U;
    I.dbg_in = in_trits;
    I.pre_out = pre_out; I.thr_out = thresh_out; I.trit_out = out_trits;
    RunOpts ro;
    int st = 0;
    return run(&I, 1, ro, reinterpret_cast<cudaStream_t>(stream), &st);
}

int externd_debug_start_trits(int64_t m, int64_t k, double tau, uint64_t seed, uint8_t* out, void* stream) {
    if (!out || m < 1 || k < 1 || !std::isfinite(tau) || tau < 0) return EXTERND_EINVAL;
    ProbIn I = {};
    I.m = m; I.n = 1; I.k = k; I.tau = tau; I.iters = 1; I.seed = seed; I.mode = MODE_FACTOR;
    I.B = out;
    RunOpts ro;
    ro.init_only = true;
    int st = 0;
    return run(&I, 1, ro, reinterpret_cast<cudaStream_t>(stream), &st);
}

int externd_debug_component(const float* R, int64_t m, int64_t n, double tau, int iters, const uint8_t* u0,
                            int n_pend, const double* pend_d, const uint8_t* pend_u, const uint8_t* pend_v,
                            double* pre_v, double* thr_v, uint8_t* trit_v, double* pre_u, double* thr_u,
                            uint8_t* trit_u, float* D_out, double* d64_out, uint8_t* u_out, uint8_t* v_out, int grid,
                            void* stream) {
    if (!R || !u0 || !D_out || !d64_out || !u_out || !v_out) return EXTERND_EINVAL;
    if (m < 1 || n < 1 || iters < 1 || !std::isfinite(tau) || tau < 0 || grid < 0) return EXTERND_EINVAL;
    if (m > INT_MAX / 2 || n > INT_MAX / 2) return EXTERND_ELIMIT;
    if (n_pend < 0 || n_pend >= MAX_PENDING) return n_pend < 0 ? EXTERND_EINVAL : EXTERND_ELIMIT;
    if (n_pend > 0) {
        if (!pend_d || !pend_u || !pend_v || !is_device_ptr(pend_d) || !is_device_ptr(pend_u) || !is_device_ptr(pend_v))
            return EXTERND_EINVAL;
        if (check_rows_aligned(pend_u) || check_rows_aligned(pend_v)) return EXTERND_EINVAL;
    }
    int rc = check_trace(0, 1, 1, pre_v, thr_v, trit_v, pre_u, thr_u, trit_u);
    if (rc != EXTERND_OK) return rc;
    if (check_rows_aligned(u_out) || check_rows_aligned(v_out)) return EXTERND_EINVAL;
    ProbIn I = {};
    I.A = R; I.m = m; I.n = n; I.k = 1; I.tau = tau; I.iters = iters; I.mode = MODE_FACTOR;
    I.B = u_out; I.C = v_out; I.D = D_out; I.d64 = d64_out;
    I.start_in = u0;
    I.n_pend = n_pend; I.pend_d = pend_d; I.pend_u = pend_u; I.pend_v = pend_v;
    I.tr_first = 0; I.tr_count = 1;
    I.tr_pre_v = pre_v; I.tr_thr_v = thr_v; I.tr_trit_v = trit_v;
    I.tr_pre_u = pre_u; I.tr_thr_u = thr_u; I.tr_trit_u = trit_u;
    RunOpts ro;
    ro.grid = grid;
    int st = 0;
    return run(&I, 1, ro, reinterpret_cast<cudaStream_t>(stream), &st);
}

int externd_reconstruct(const uint8_t* B, const float* D, const uint8_t* C, int64_t m, int64_t n, int64_t k,
                        float* A_hat_out, void* stream) {
    if (!B || !D || !C || !A_hat_out || m < 1 || n < 1 || k < 1) return EXTERND_EINVAL;
    if ((m + 31) / 32 > 65535) return EXTERND_ELIMIT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t bb = trit_bytes(m), cb = trit_bytes(n);
    const bool dB = is_device_ptr(B), dC = is_device_ptr(C), dD = is_device_ptr(D), dO = is_device_ptr(A_hat_out);
    size_t ws = 0, oB = 0, oC = 0, oD = 0, oO = 0;
    if (!dB) { oB = ws; ws += round_up(bb * (size_t)k, 256); }
    if (!dC) { oC = ws; ws += round_up(cb * (size_t)k, 256); }
    if (!dD) { oD = ws; ws += round_up(sizeof(float) * (size_t)k, 256); }
    if (!dO) { oO = ws; ws += round_up(sizeof(float) * (size_t)(m * n), 256); }
    int rc = EXTERND_OK;
    unsigned char* w = nullptr;
    cudaEvent_t e0 = nullptr, e1 = nullptr;
    const uint8_t* pB = B;
    const uint8_t* pC = C;
    const float* pD = D;
    float* pO = A_hat_out;
    float ms = 0;
    externd_stats st = {};
    CK(cudaEventCreate(&e0));
    CK(cudaEventCreate(&e1));
    CK(cudaEventRecord(e0, s));
    if (ws) CK(cudaMallocAsync((void**)&w, ws, s));
    if (!dB) { CK(cudaMemcpyAsync(w + oB, B, bb * (size_t)k, cudaMemcpyHostToDevice, s)); pB = w + oB; }
    if (!dC) { CK(cudaMemcpyAsync(w + oC, C, cb * (size_t)k, cudaMemcpyHostToDevice, s)); pC = w + oC; }
    if (!dD) { CK(cudaMemcpyAsync(w + oD, D, sizeof(float) * (size_t)k, cudaMemcpyHostToDevice, s)); pD = reinterpret_cast<float*>(w + oD); }
    if (!dO) pO = reinterpret_cast<float*>(w + oO);
    reconstruct_kernel<<<dim3((unsigned)((n + 31) / 32), (unsigned)((m + 31) / 32)), dim3(32, 8), 0, s>>>(
        pB, pD, pC, m, n, k, (int64_t)bb, (int64_t)cb, pO);
    CK(cudaGetLastError());
    if (!dO) CK(cudaMemcpyAsync(A_hat_out, pO, sizeof(float) * (size_t)(m * n), cudaMemcpyDeviceToHost, s));
    CK(cudaEventRecord(e1, s));
    CK(cudaStreamSynchronize(s));
    cudaEventElapsedTime(&ms, e0, e1);
    st.total_ms = ms;
    st.launches = 1;
done:
    if (w) { cudaFreeAsync(w, s); cudaStreamSynchronize(s); }
    if (e0) cudaEventDestroy(e0);
    if (e1) cudaEventDestroy(e1);
    cudaGetLastError();
    g_last = st;
    return rc;
}

int externd_last_stats(externd_stats* out) {
    if (!out) return EXTERND_EINVAL;
    *out = g_last;
    return EXTERND_OK;
}

}  // extern "C"

#endif  // EXTERND_SECONDARY
