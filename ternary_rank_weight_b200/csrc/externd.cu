// ExTernD greedy sequential ternary ALS for B200 (sm_100a): kernels + C ABI.
//
// Method: "ExTernD: Expanded-Rank Ternary Decomposition" (arXiv 2607.13511),
// §2.1 (factorization, energy), §2.2 (T_tau), §2.3 (greedy sequential ALS).
// The data layout and the synchronisation scheme are described at the top of
// externd_kernels.cuh.
#include <cuda_runtime.h>

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
            ss += (double)v * (double)v;
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
// Start trits u0_i = T_tau(z_i) for every component (reading of §2.3: the pages
// start from an unspecified u; here a seeded Gaussian vector).
// ---------------------------------------------------------------------------

constexpr int NTI = 256;

__global__ void __launch_bounds__(NTI) init_kernel(const Prob* __restrict__ probs) {
    const Prob& P = probs[blockIdx.y];
    if (P.mode != MODE_FACTOR) return;
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

// Shared-memory carve of the ALS kernel (host and device use the same layout).
struct SmemLayout {
    size_t red, pd, coef, scal, wS, wM, wp, gS, gM, wJ, gJ, wc, dotp, sflag, nzU, sgU, nzV, sgV, pnzU, psgU, pnzV,
        psgV, cnzV, csgV, cnzU, csgU, ulist, vlist, total;
    __host__ __device__ SmemLayout(int64_t m_max, int64_t n_max, int Lc, int pv_max, int pu_max) {
        const size_t Wm = (size_t)((m_max + 31) / 32), Wn = (size_t)((n_max + 31) / 32);
        size_t o = 0;
        red = o;  o += 8 * (size_t)NT * 4;
        pd = o;   o += 8 * (size_t)Lc;
        coef = o; o += 8 * (size_t)Lc;
        scal = o; o += 8 * 16;
        wS = o;   o += 8 * NWARP;
        wM = o;   o += 8 * NWARP;
        wp = o;   o += 8 * NWARP;
        gS = o;   o += 8 * NWARP;
        gM = o;   o += 8 * NWARP;
        wJ = o;   o += 8 * NWARP;
        gJ = o;   o += 8 * NWARP;
        wc = o;   o += 4 * NWARP;
        dotp = o; o += 4 * NWARP * MAX_PENDING;
        sflag = o; o += 16;
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
        total = (o + 15) & ~(size_t)15;
    }
};

struct Smem {
    double *red, *pd, *coef, *scal, *wS, *wM, *wp, *gS, *gM;
    long long *wJ, *gJ;
    int *wc, *dotp, *sflag;
    uint32_t *nzU, *sgU, *nzV, *sgV;         // current u, v
    uint32_t *pnzU, *psgU, *pnzV, *psgV;     // pending components (full length, stride W)
    uint32_t *cnzV, *csgV, *cnzU, *csgU;     // pending trits at this CTA's outputs, bit l = component l
    int *ulist, *vlist;                      // compacted supports (index | sign << 31)
};

__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
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

// Lazy-deflation correction at one of this CTA's outputs: sum_l coef_l t_l(c),
// t_l from the per-output pending bit masks, in increasing l.
struct HalfCorr {
    const double* coef;
    const uint32_t* cnz;
    const uint32_t* csg;
};

__device__ __forceinline__ double corr_local(int c, const HalfCorr& hc) {
    uint32_t bits = hc.cnz[c];
    const uint32_t sgn = hc.csg[c];
    double v = 0.0;
    while (bits) {
        const int l = __ffs(bits) - 1;
        bits &= bits - 1u;
        v += ((sgn >> l) & 1u) ? -hc.coef[l] : hc.coef[l];
    }
    return v;
}

__device__ __forceinline__ void emit_out(double v, int c, int64_t out0, double* gout, const HalfCorr& hc, double& S,
                                         double& M, long long& J) {
    v -= corr_local(c, hc);
    gout[out0 + c] = v;
    const double av = fabs(v);
    S += av;
    if (av > M) { M = av; J = out0 + c; }
}

// One half-step GEMV over this CTA's private block: out[c] = sum_{e in list} s_e blk[r_e][c]
// for the block's `valid` columns, minus the lazy-deflation correction, written to
// gout[out0 + c].  fp64 accumulation of exact fp32 terms, fixed summation order.
template <int VEC>
__device__ void gemv_emit(const float* __restrict__ blk, int pitch, int valid, int64_t out0,
                          const int* __restrict__ list, int nlist, double* red, double* gout, const HalfCorr& hc,
                          double& S, double& M, long long& J) {
    S = 0.0; M = -1.0; J = LLONG_MAX;
    const int nvec = pitch / VEC;
    if (nvec <= 0) return;
    constexpr int U = (VEC == 4) ? 16 : (VEC == 2 ? 24 : 32);
    if (nvec <= NT) {
        const int lanes = NT / nvec;
        const int j = threadIdx.x % nvec;
        const int g = threadIdx.x / nvec;
        if (g < lanes) {
            double acc[VEC];
            #pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = 0.0;
            const float* base = blk + j * VEC;
            // every batch issues all of its loads before using any (predicated tail)
            for (int idx = g; idx < nlist; idx += U * lanes) {
                int ent[U];
                float v[U][VEC];
                #pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int ii = idx + u * lanes;
                    ent[u] = ii < nlist ? list[ii] : 0;
                    if (ii < nlist) {
                        load_vec<VEC>(base + (int64_t)(ent[u] & 0x7fffffff) * pitch, v[u]);
                    } else {
                        #pragma unroll
                        for (int e = 0; e < VEC; ++e) v[u][e] = 0.f;
                    }
                }
                #pragma unroll
                for (int u = 0; u < U; ++u) {
                    const unsigned sm = (unsigned)ent[u] & 0x80000000u;
                    #pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[e] += (double)__uint_as_float(__float_as_uint(v[u][e]) ^ sm);
                }
            }
            #pragma unroll
            for (int e = 0; e < VEC; ++e) red[g * pitch + j * VEC + e] = acc[e];
        }
        __syncthreads();
        int tpc = 1;
        while (tpc < 32 && tpc * 2 * pitch <= NT) tpc *= 2;
        const int cpr = NT / tpc;
        for (int cb = 0; cb < pitch; cb += cpr) {
            const int c = cb + (int)threadIdx.x / tpc;
            const int s = (int)threadIdx.x % tpc;
            double v = 0.0;
            if (c < pitch)
                for (int gg = s; gg < lanes; gg += tpc) v += red[gg * pitch + c];
            for (int o = tpc >> 1; o; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
            if (s == 0 && c < valid) emit_out(v, c, out0, gout, hc, S, M, J);
        }
    } else {
        for (int j = threadIdx.x; j < nvec; j += NT) {
            double acc[VEC];
            #pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = 0.0;
            const float* base = blk + j * VEC;
            for (int idx = 0; idx < nlist; idx += U) {
                int ent[U];
                float v[U][VEC];
                #pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int ii = idx + u;
                    ent[u] = ii < nlist ? list[ii] : 0;
                    if (ii < nlist) {
                        load_vec<VEC>(base + (int64_t)(ent[u] & 0x7fffffff) * pitch, v[u]);
                    } else {
                        #pragma unroll
                        for (int e = 0; e < VEC; ++e) v[u][e] = 0.f;
                    }
                }
                #pragma unroll
                for (int u = 0; u < U; ++u) {
                    const unsigned sm = (unsigned)ent[u] & 0x80000000u;
                    #pragma unroll
                    for (int e = 0; e < VEC; ++e) acc[e] += (double)__uint_as_float(__float_as_uint(v[u][e]) ^ sm);
                }
            }
            #pragma unroll
            for (int e = 0; e < VEC; ++e) {
                const int c = j * VEC + e;
                if (c < valid) emit_out(acc[e], c, out0, gout, hc, S, M, J);
            }
        }
    }
}

__device__ __forceinline__ void gemv_dispatch(int vec, const float* blk, int pitch, int valid, int64_t out0,
                                              const int* list, int nlist, double* red, double* gout,
                                              const HalfCorr& hc, double& S, double& M, long long& J) {
    if (vec == 4) gemv_emit<4>(blk, pitch, valid, out0, list, nlist, red, gout, hc, S, M, J);
    else if (vec == 2) gemv_emit<2>(blk, pitch, valid, out0, list, nlist, red, gout, hc, S, M, J);
    else gemv_emit<1>(blk, pitch, valid, out0, list, nlist, red, gout, hc, S, M, J);
}

// Fold the L pending components into this CTA's block:
// blk[r][c] -= sum_l d_l * tR_l(r) * tC_l(col0 + c), fp64 sum in increasing l, one fp32 rounding.
template <int VEC>
__device__ void flush_block(float* blk, int pitch, int64_t rows, int valid, int L, const double* pd,
                            const uint32_t* pnzR, const uint32_t* psgR, int WR, const uint32_t* cnz,
                            const uint32_t* csg) {
    const int nvec = pitch / VEC;
    if (nvec <= 0 || L <= 0) return;
    const int64_t total = rows * nvec;
    for (int64_t t = threadIdx.x; t < total; t += NT) {
        const int64_t r = t / nvec;
        const int j = (int)(t - r * nvec);
        const int wr = (int)(r >> 5);
        const uint32_t br = 1u << (r & 31);
        uint32_t rnz = 0, rsg = 0;
        for (int l = 0; l < L; ++l) {
            rnz |= ((pnzR[l * WR + wr] & br) ? 1u : 0u) << l;
            rsg |= ((psgR[l * WR + wr] & br) ? 1u : 0u) << l;
        }
        if (!rnz) continue;
        float* p = blk + r * pitch + j * VEC;
        #pragma unroll
        for (int e = 0; e < VEC; ++e) {
            const int c = j * VEC + e;
            if (c >= valid) continue;
            uint32_t bits = rnz & cnz[c];
            if (!bits) continue;
            const uint32_t neg = rsg ^ csg[c];
            double corr = 0.0;
            while (bits) {
                const int l = __ffs(bits) - 1;
                bits &= bits - 1u;
                corr += ((neg >> l) & 1u) ? -pd[l] : pd[l];
            }
            p[e] = (float)((double)__ldcg(p + e) - corr);
        }
    }
}

__device__ __forceinline__ void flush_dispatch(int vec, float* blk, int pitch, int64_t rows, int valid, int L,
                                               const double* pd, const uint32_t* pnzR, const uint32_t* psgR, int WR,
                                               const uint32_t* cnz, const uint32_t* csg) {
    if (vec == 4) flush_block<4>(blk, pitch, rows, valid, L, pd, pnzR, psgR, WR, cnz, csg);
    else if (vec == 2) flush_block<2>(blk, pitch, rows, valid, L, pd, pnzR, psgR, WR, cnz, csg);
    else flush_block<1>(blk, pitch, rows, valid, L, pd, pnzR, psgR, WR, cnz, csg);
}

// Start trits (2-bit packed words) -> masks and list; returns nnz.
__device__ int build_from_trits(const uint32_t* words, int64_t nwords, int64_t len, uint32_t* nz, uint32_t* sg,
                                int* list, const Smem& s) {
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
                (int)(((unsigned)w << 5) + lane_id()) | (int)(((sg[w] >> lane_id()) & 1u) << 31);
        run += __popc(bz);
    }
    __syncthreads();
    return total;
}

// coef_l = d_l * (t_l . t) for every pending component (integer dot product of trit masks)
__device__ void pending_coef(int L, int W, const uint32_t* pnz, const uint32_t* psg, const uint32_t* nz,
                             const uint32_t* sg, const double* pd, double* coef) {
    for (int l = warp_id(); l < L; l += NWARP) {
        int acc = 0;
        for (int w = lane_id(); w < W; w += 32) {
            const uint32_t both = pnz[l * W + w] & nz[w];
            const uint32_t diff = psg[l * W + w] ^ sg[w];
            acc += __popc(both & ~diff) - __popc(both & diff);
        }
        #pragma unroll
        for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(FULL, acc, o);
        if (lane_id() == 0) coef[l] = pd[l] * (double)acc;
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

// Publish this CTA's (sum |out|, max |out|, argmax) and arrive at the group counter,
// then wait until every CTA of the group arrived.  Arrival is a release by one
// thread after a CTA barrier, the wait an acquire by the same thread followed by a
// CTA barrier, so the slice of the output vector each CTA stored before arriving
// is visible to all CTAs after the wait.  Bounded by limit_ns; on expiry the group
// abort flag and the status word are raised.
__device__ bool publish_and_wait(Slot* slot, double S, double M, long long J, const Smem& s, GroupSync* gs,
                                 unsigned& target, int Gg, uint64_t limit_ns, bool skip_arrive, int* status) {
    #pragma unroll
    for (int o = 16; o; o >>= 1) {
        S += __shfl_xor_sync(FULL, S, o);
        const double m2 = __shfl_xor_sync(FULL, M, o);
        const long long j2 = __shfl_xor_sync(FULL, J, o);
        maxloc_merge(M, J, m2, j2);
    }
    if (lane_id() == 0) { s.wS[warp_id()] = S; s.wM[warp_id()] = M; s.wJ[warp_id()] = J; }
    __syncthreads();
    if (threadIdx.x == 0) {
        double S2 = 0.0, M2 = -1.0;
        long long J2 = LLONG_MAX;
        for (int w = 0; w < NWARP; ++w) { S2 += s.wS[w]; maxloc_merge(M2, J2, s.wM[w], s.wJ[w]); }
        slot->S = S2;
        slot->M = M2;
        slot->J = J2;
        target += (unsigned)Gg;
        if (!skip_arrive) red_release_add(&gs->arrive, 1u);
        int ok = 1;
        const uint64_t t0 = gtimer();
        unsigned spins = 0;
        while ((int)(ld_acquire_u32(&gs->arrive) - target) < 0) {
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
        *s.sflag = ok;
    }
    __syncthreads();
    return *s.sflag != 0;
}

// After publish_and_wait: sum of the group's published S in a fixed order.
__device__ double gather_sum(const Slot* sl, int Gg, const Smem& s) {
    double S = ((int)threadIdx.x < Gg) ? __ldcg(&sl[threadIdx.x].S) : 0.0;
    #pragma unroll
    for (int o = 16; o; o >>= 1) S += __shfl_xor_sync(FULL, S, o);
    if (lane_id() == 0) s.gS[warp_id()] = S;
    __syncthreads();
    double t = 0.0;
    for (int w = 0; w < NWARP; ++w) t += s.gS[w];
    __syncthreads();
    return t;
}

// After publish_and_wait: read the group's slots and the whole published vector,
// threshold it (T_tau of §2.2 with the all-zero fallback), write its masks and
// compacted support list, the coefficients d_l (t_l . t) of the pending
// components for the next half-step, and p = sum over the support of |x| into
// s.scal[0].  Every CTA of the group derives identical results (same data, same
// order).  Returns nnz.
__device__ int gather_threshold(const Slot* sl, int Gg, const double* gvec, int64_t len, double tau, uint32_t* nz,
                                uint32_t* sg, int* list, const Smem& s, int L, const uint32_t* pnz,
                                const uint32_t* psg, double& thr_out) {
    const int lane = lane_id(), warp = warp_id();
    const int W = (int)((len + 31) >> 5);
    const int wpw = (W + NWARP - 1) / NWARP;
    const int w0 = min(W, warp * wpw), w1 = min(W, w0 + wpw);
    double S = 0.0, M = -1.0;
    long long J = LLONG_MAX;
    if ((int)threadIdx.x < Gg) {
        S = __ldcg(&sl[threadIdx.x].S);
        M = __ldcg(&sl[threadIdx.x].M);
        J = __ldcg(&sl[threadIdx.x].J);
    }
    constexpr int CH = 16;
    double xv[CH];
    #pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int w = w0 + i;
        const int64_t idx = ((int64_t)w << 5) + lane;
        xv[i] = (w < w1 && idx < len) ? __ldcg(gvec + idx) : 0.0;
    }
    #pragma unroll
    for (int o = 16; o; o >>= 1) {
        S += __shfl_xor_sync(FULL, S, o);
        const double m2 = __shfl_xor_sync(FULL, M, o);
        const long long j2 = __shfl_xor_sync(FULL, J, o);
        maxloc_merge(M, J, m2, j2);
    }
    if (lane == 0) { s.gS[warp] = S; s.gM[warp] = M; s.gJ[warp] = J; }
    __syncthreads();
    double St = 0.0, Mt = -1.0;
    long long Jt = LLONG_MAX;
    for (int w = 0; w < NWARP; ++w) { St += s.gS[w]; maxloc_merge(Mt, Jt, s.gM[w], s.gJ[w]); }
    const double thr = tau * St / (double)len;
    thr_out = thr;

    int cnt = 0, dot = 0;
    double ps = 0.0;
    for (int base = w0; base < w1; base += CH) {
        if (base != w0) {
            #pragma unroll
            for (int i = 0; i < CH; ++i) {
                const int w = base + i;
                const int64_t idx = ((int64_t)w << 5) + lane;
                xv[i] = (w < w1 && idx < len) ? __ldcg(gvec + idx) : 0.0;
            }
        }
        #pragma unroll
        for (int i = 0; i < CH; ++i) {
            const int w = base + i;
            if (w < w1) {
                const int64_t idx = ((int64_t)w << 5) + lane;
                const bool z = (idx < len) && (fabs(xv[i]) > thr);
                const bool ng = z && (xv[i] < 0.0);
                const unsigned bz = __ballot_sync(FULL, z);
                const unsigned bs = __ballot_sync(FULL, ng);
                if (lane == 0) { nz[w] = bz; sg[w] = bs; }
                cnt += __popc(bz);
                if (z) ps += fabs(xv[i]);
                if (lane < L) {
                    const uint32_t both = pnz[lane * W + w] & bz;
                    const uint32_t diff = psg[lane * W + w] ^ bs;
                    dot += __popc(both & ~diff) - __popc(both & diff);
                }
            }
        }
    }
    #pragma unroll
    for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(FULL, ps, o);
    if (lane == 0) { s.wc[warp] = cnt; s.wp[warp] = ps; }
    if (lane < L) s.dotp[warp * MAX_PENDING + lane] = dot;
    __syncthreads();
    int off = 0, total = 0;
    double p = 0.0;
    for (int w = 0; w < NWARP; ++w) {
        const int c = s.wc[w];
        off += (w < warp) ? c : 0;
        total += c;
        p += s.wp[w];
    }
    if (total > 0) {
        if ((int)threadIdx.x < L) {
            int d = 0;
            for (int w = 0; w < NWARP; ++w) d += s.dotp[w * MAX_PENDING + threadIdx.x];
            s.coef[threadIdx.x] = s.pd[threadIdx.x] * (double)d;
        }
        int run = off;
        for (int w = w0; w < w1; ++w) {
            const uint32_t bz = nz[w];
            if ((bz >> lane) & 1u)
                list[run + __popc(bz & ((1u << lane) - 1u))] =
                    (int)(((unsigned)w << 5) + lane) | (int)(((sg[w] >> lane) & 1u) << 31);
            run += __popc(bz);
        }
        if (threadIdx.x == 0) { s.scal[0] = p; s.scal[1] = 0.0; }
    } else {
        // all-zero fallback: keep the lowest index among the largest magnitudes
        const long long Jc = (Jt >= 0 && Jt < len) ? Jt : 0;   // out of range only with non-finite data
        const double x = __ldcg(gvec + Jc);
        const bool neg = x < 0.0;
        const int wj = (int)(Jc >> 5);
        const uint32_t bj = 1u << (Jc & 31);
        if ((int)threadIdx.x < L) {
            int t = (pnz[threadIdx.x * W + wj] & bj) ? 1 : 0;
            if (t && ((psg[threadIdx.x * W + wj] & bj) != 0u) != neg) t = -1;
            s.coef[threadIdx.x] = s.pd[threadIdx.x] * (double)t;
        }
        if (threadIdx.x == 0) {
            nz[wj] |= bj;
            if (neg) sg[wj] |= bj;
            list[0] = (int)Jc | (neg ? (int)0x80000000 : 0);
            s.scal[0] = fabs(x);
            s.scal[1] = 1.0;
        }
        total = 1;
    }
    __syncthreads();
    return total;
}

// Factor (or run one debug half-step of) one matrix with this CTA group.
// Returns false if the group aborted.
__device__ bool run_problem(const Prob& P, int q, const KCfg& cfg, const Smem& s, GroupSync* gs, Slot* slots,
                            unsigned& target, int& par) {
    const int64_t m = P.m, n = P.n;
    const int Wm = (int)((m + 31) >> 5), Wn = (int)((n + 31) >> 5);
    const int mode = P.mode;
    const int Gg = cfg.Gg;
    const int tid = threadIdx.x;
    const bool lead = (q == 0);
    const bool skip = (cfg.fault_skip == q);

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
    unsigned long long sum_nu = 0, sum_nv = 0, sum_nunv = 0, hs = 0, fb = 0;
    const int64_t kk = (mode == MODE_FACTOR) ? P.k : 1;
    int nU = 0, nV = 0;
    double p = 0.0, S, M, thr;
    long long J;
    const HalfCorr hcV{s.coef, s.cnzV, s.csgV};
    const HalfCorr hcU{s.coef, s.cnzU, s.csgU};
    // phase clock of thread 0 of CTA 0 (diagnostics; a few clock reads per half-step)
    const bool tim = lead && tid == 0;
    unsigned long long ph[4] = {0, 0, 0, 0};
    long long t_prev = clock64();
#define EXTERND_PHASE(k)                                   \
    if (tim) {                                             \
        const long long t_ = clock64();                    \
        ph[k] += (unsigned long long)(t_ - t_prev);        \
        t_prev = t_;                                       \
    }

    for (int64_t i = 0; i < kk; ++i) {
        if (mode != MODE_HALF_U) {
            nU = build_from_trits(P.start + i * P.start_words, P.start_words, m, s.nzU, s.sgU, s.ulist, s);
            if (L > 0) pending_coef(L, Wm, s.pnzU, s.psgU, s.nzU, s.sgU, s.pd, s.coef);
        } else {
            nV = build_from_trits(P.start, P.start_words, n, s.nzV, s.sgV, s.vlist, s);
        }
        for (int it = 0; it < P.iters; ++it) {
            if (mode != MODE_HALF_U) {
                // ---- V-step: x = R^T u on this CTA's columns (§2.3 step 1, first half)
                EXTERND_PHASE(3);
                gemv_dispatch(P.pv.vec, blkV, pitchV, validV, c0, s.ulist, nU, s.red, P.xbuf, hcV, S, M, J);
                EXTERND_PHASE(0);
                if (!publish_and_wait(slots + par * Gg + q, S, M, J, s, gs, target, Gg, cfg.limit_ns, skip, P.status))
                    return false;
                EXTERND_PHASE(1);
                const int nv2 = gather_threshold(slots + par * Gg, Gg, P.xbuf, n, P.tau, s.nzV, s.sgV, s.vlist, s, L,
                                                 s.pnzV, s.psgV, thr);
                EXTERND_PHASE(2);
                par ^= 1;
                fb += (s.scal[1] != 0.0) ? 1 : 0;
                nV = nv2;
                sum_nu += (unsigned long long)nU;
                ++hs;
                if (mode == MODE_HALF_V) {
                    if (lead) {
                        for (int64_t t = tid; t < n; t += NT) P.pre_out[t] = __ldcg(P.xbuf + t);
                        if (tid == 0) *P.thr_out = thr;
                        pack_row(s.nzV, s.sgV, Wn, reinterpret_cast<uint32_t*>(P.trit_out), P.c_bytes / 4);
                        __syncthreads();
                        if (tid == 0) { __threadfence(); atomicExch(P.status, ST_OK); }
                    }
                    return true;
                }
            }
            // ---- U-step: y = R v on this CTA's rows (§2.3 step 1, second half)
            EXTERND_PHASE(3);
            gemv_dispatch(P.pu.vec, blkU, pitchU, validU, r0, s.vlist, nV, s.red, P.ybuf, hcU, S, M, J);
            EXTERND_PHASE(0);
            if (!publish_and_wait(slots + par * Gg + q, S, M, J, s, gs, target, Gg, cfg.limit_ns, skip, P.status))
                return false;
            EXTERND_PHASE(1);
            nU = gather_threshold(slots + par * Gg, Gg, P.ybuf, m, P.tau, s.nzU, s.sgU, s.ulist, s, L, s.pnzU,
                                  s.psgU, thr);
            EXTERND_PHASE(2);
            par ^= 1;
            p = s.scal[0];
            fb += (s.scal[1] != 0.0) ? 1 : 0;
            sum_nv += (unsigned long long)nV;
            ++hs;
            if (mode == MODE_HALF_U) {
                if (lead) {
                    for (int64_t t = tid; t < m; t += NT) P.pre_out[t] = __ldcg(P.ybuf + t);
                    if (tid == 0) *P.thr_out = thr;
                    pack_row(s.nzU, s.sgU, Wm, reinterpret_cast<uint32_t*>(P.trit_out), P.b_bytes / 4);
                    __syncthreads();
                    if (tid == 0) { __threadfence(); atomicExch(P.status, ST_OK); }
                }
                return true;
            }
        }
        // ---- scale (§2.3 step 2): d = u^T R v / (nnz(u) nnz(v)), with u^T R v = u^T y = p
        const double d = (p == 0.0) ? 0.0 : p / ((double)nU * (double)nV);
        RN2 -= p * d;
        sum_nunv += (unsigned long long)nU * (unsigned long long)nV;
        if (lead) {
            pack_row(s.nzU, s.sgU, Wm, reinterpret_cast<uint32_t*>(P.B + i * P.b_bytes), P.b_bytes / 4);
            pack_row(s.nzV, s.sgV, Wn, reinterpret_cast<uint32_t*>(P.C + i * P.c_bytes), P.c_bytes / 4);
            if (tid == 0) {
                P.D[i] = (float)d;
                if (P.energy) P.energy[i] = 1.0 - RN2 / N0;
                if (P.d64) P.d64[i] = d;
            }
        }
        // ---- deflation (§2.3 step 3), held lazily as a pending rank-1 term
        if (tid == 0) s.pd[L] = d;
        for (int w = tid; w < Wm; w += NT) { s.pnzU[L * Wm + w] = s.nzU[w]; s.psgU[L * Wm + w] = s.sgU[w]; }
        for (int w = tid; w < Wn; w += NT) { s.pnzV[L * Wn + w] = s.nzV[w]; s.psgV[L * Wn + w] = s.sgV[w]; }
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
        ++L;
        __syncthreads();
        if (L == cfg.Lcap || i == kk - 1) {
            flush_dispatch(P.pv.vec, blkV, pitchV, m, validV, L, s.pd, s.pnzU, s.psgU, Wm, s.cnzV, s.csgV);
            flush_dispatch(P.pu.vec, blkU, pitchU, n, validU, L, s.pd, s.pnzV, s.psgV, Wn, s.cnzU, s.csgU);
            __syncthreads();
            for (int c = tid; c < pitchV; c += NT) { s.cnzV[c] = 0u; s.csgV[c] = 0u; }
            for (int c = tid; c < pitchU; c += NT) { s.cnzU[c] = 0u; s.csgU[c] = 0u; }
            L = 0;
            __syncthreads();
        }
    }

    // ---- explicit ||R_k||^2 from the folded fp32 residual (V-layout covers all of R)
    double rs = 0.0;
    if (validV > 0) {
        const int64_t tot = m * (int64_t)validV;
        for (int64_t t = tid; t < tot; t += NT) {
            const int64_t r = t / validV;
            const int c = (int)(t - r * validV);
            const double v = (double)__ldcg(blkV + r * pitchV + c);
            rs += v * v;
        }
    }
    if (!publish_and_wait(slots + par * Gg + q, rs, 0.0, 0, s, gs, target, Gg, cfg.limit_ns, skip, P.status))
        return false;
    const double R2 = gather_sum(slots + par * Gg, Gg, s);
    par ^= 1;
    if (lead && tid == 0) {
        P.stats->sum_nu = sum_nu;
        P.stats->sum_nv = sum_nv;
        P.stats->sum_nunv = sum_nunv;
        P.stats->half_steps = hs;
        P.stats->fallbacks = fb;
        P.stats->residual2 = R2;
        P.stats->norm_a2 = N0;
        EXTERND_PHASE(3);
        for (int k2 = 0; k2 < 4; ++k2) P.stats->phase[k2] = ph[k2];
        __threadfence();
        atomicExch(P.status, ST_OK);
    }
    __syncthreads();
    return true;
#undef EXTERND_PHASE
}

__global__ void __launch_bounds__(NT, 1) als_kernel(const KCfg cfg) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int grp = blockIdx.x / cfg.Gg;
    const int q = blockIdx.x - grp * cfg.Gg;
    const int Lc = cfg.Lcap > 0 ? cfg.Lcap : 1;
    const SmemLayout lay(cfg.m_max, cfg.n_max, Lc, cfg.pv_max, cfg.pu_max);
    Smem s;
    s.red = reinterpret_cast<double*>(smem_raw + lay.red);
    s.pd = reinterpret_cast<double*>(smem_raw + lay.pd);
    s.coef = reinterpret_cast<double*>(smem_raw + lay.coef);
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

    GroupSync* gs = cfg.gsync + grp;
    Slot* slots = cfg.slots + (size_t)grp * 2 * cfg.Gg;
    unsigned target = 0;
    int par = 0;
    for (int pi = grp; pi < cfg.nprob; pi += cfg.NG) {
        if (!run_problem(cfg.probs[pi], q, cfg, s, gs, slots, target, par)) return;
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
        if (cudaFuncSetAttribute(als_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)d.smem_optin) != cudaSuccess) {
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

// Largest vector width whose stripe imbalance stays within 6 %, else the least imbalanced.
int choose_vec(int64_t len, int G) {
    const double ideal = (double)len / G;
    int best = 1;
    double best_imb = 1e30;
    for (int vec : {4, 2, 1}) {
        const int64_t units = (len + vec - 1) / vec;
        const int64_t maxu = (units + G - 1) / G;
        const double imb = (double)(maxu * vec) / (ideal > 0 ? ideal : 1.0);
        if (imb <= 1.06) return vec;
        if (imb < best_imb - 1e-12) { best_imb = imb; best = vec; }
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

size_t als_smem_bytes(int64_t m_max, int64_t n_max, int L, int pv_max, int pu_max) {
    return SmemLayout(m_max, n_max, L > 0 ? L : 1, pv_max, pu_max).total;
}

struct ProbIn {
    const float* A;
    int64_t m, n, k;
    double tau;
    int iters;
    uint64_t seed;
    uint8_t* B;
    float* D;
    uint8_t* C;
    double* energy;
    double* d64;
    int mode;
    const uint8_t* dbg_in;
    double* pre_out;
    double* thr_out;
    uint8_t* trit_out;
};

struct RunOpts {
    int grid = 0;
    int pending = 0;
    double wait_limit_s = 2.0;
    int fault_skip = -1;
    bool init_only = false;
};

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
int run(const ProbIn* in, int np, const RunOpts& opt, cudaStream_t stream, int* statuses) {
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

    // ---- lazy deflation depth from the shared-memory budget
    if (Gg > NT) Gg = NT;   // one slot per thread when the group's slots are gathered
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
    int Lcap = MAX_PENDING;
    while (Lcap > 1 && als_smem_bytes(m_max, n_max, Lcap, pv_max, pu_max) > di.smem_optin) --Lcap;
    if (opt.pending > 0 && opt.pending < Lcap) Lcap = opt.pending;
    const size_t smem = als_smem_bytes(m_max, n_max, Lcap, pv_max, pu_max);
    if (smem > di.smem_optin) return EXTERND_ELIMIT;

    int nb = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, als_kernel, NT, smem) != cudaSuccess) {
        cudaGetLastError();
        return EXTERND_ECUDA;
    }
    if ((int64_t)nb * sms < (int64_t)NG * Gg) return EXTERND_ELAUNCH;

    // ---- plan the workspace
    std::vector<Prob> probs(np);
    std::vector<size_t> off_rv(np), off_ru(np), off_x(np), off_y(np), off_start(np), off_norm(np), off_A(np),
        off_B(np), off_C(np), off_D(np), off_E(np), off_d64(np), off_pre(np), off_thr(np), off_tro(np);
    size_t ctl = 0;
    const size_t off_gsync = ctl;
    ctl += round_up(sizeof(GroupSync) * NG, 256);
    const size_t off_slots = ctl;
    ctl += round_up(sizeof(Slot) * 2 * (size_t)Gg * NG, 256);
    const size_t off_status = ctl;
    ctl += round_up(sizeof(int) * np, 256);
    const size_t off_nonfin = ctl;
    ctl += round_up(sizeof(unsigned) * np, 256);
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
        P.n_norm_part = ((I.m + 31) / 32) * ((I.n + 31) / 32);
        off_rv[b] = ws; ws += round_up(sizeof(float) * (size_t)P.pv.total(I.m), 256);
        off_ru[b] = ws; ws += round_up(sizeof(float) * (size_t)P.pu.total(I.n), 256);
    }
    const size_t zero_to = ws;
    for (int b = 0; b < np; ++b) {
        const ProbIn& I = in[b];
        Prob& P = probs[b];
        off_x[b] = ws; ws += round_up(sizeof(double) * (size_t)I.n, 256);
        off_y[b] = ws; ws += round_up(sizeof(double) * (size_t)I.m, 256);
        const int64_t srows = (I.mode == MODE_FACTOR) ? I.k : 1;
        off_start[b] = ws; ws += round_up(sizeof(uint32_t) * (size_t)(P.start_words * srows), 256);
        off_norm[b] = ws; ws += round_up(sizeof(double) * (size_t)P.n_norm_part, 256);
        // staging for host pointers
        off_A[b] = SIZE_MAX;
        if (I.A && !is_device_ptr(I.A)) { off_A[b] = ws; ws += round_up(sizeof(float) * (size_t)(I.m * I.n), 256); }
        off_B[b] = off_C[b] = off_D[b] = off_E[b] = off_d64[b] = off_pre[b] = off_thr[b] = off_tro[b] = SIZE_MAX;
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

    unsigned char* dws = nullptr;
    cudaEvent_t ev[5] = {nullptr, nullptr, nullptr, nullptr, nullptr};
    std::vector<unsigned char> hctl(ctl, 0);
    std::vector<int> hstatus(np, ST_RUNNING);
    std::vector<DevStats> hstats(np);
    int launches = 0;
    float ms_setup = 0, ms_init = 0, ms_als = 0, ms_total = 0;

    for (int i = 0; i < 5; ++i) CK(cudaEventCreate(&ev[i]));
    CK(cudaMallocAsync((void**)&dws, ws, stream));
    CK(cudaEventRecord(ev[0], stream));

    // ---- fill problem descriptors and the control region
    for (int b = 0; b < np; ++b) {
        const ProbIn& I = in[b];
        Prob& P = probs[b];
        P.A = off_A[b] == SIZE_MAX ? I.A : reinterpret_cast<const float*>(dws + off_A[b]);
        P.Rv = reinterpret_cast<float*>(dws + off_rv[b]);
        P.Ru = reinterpret_cast<float*>(dws + off_ru[b]);
        P.xbuf = reinterpret_cast<double*>(dws + off_x[b]);
        P.ybuf = reinterpret_cast<double*>(dws + off_y[b]);
        P.start = reinterpret_cast<uint32_t*>(dws + off_start[b]);
        P.norm_part = reinterpret_cast<double*>(dws + off_norm[b]);
        P.nonfinite = reinterpret_cast<unsigned*>(dws + off_nonfin) + b;
        P.status = reinterpret_cast<int*>(dws + off_status) + b;
        P.stats = reinterpret_cast<DevStats*>(dws + off_stats) + b;
        if (I.mode == MODE_FACTOR) {
            P.B = off_B[b] == SIZE_MAX ? I.B : dws + off_B[b];
            P.C = off_C[b] == SIZE_MAX ? I.C : dws + off_C[b];
            P.D = off_D[b] == SIZE_MAX ? I.D : reinterpret_cast<float*>(dws + off_D[b]);
            P.energy = off_E[b] == SIZE_MAX ? I.energy : reinterpret_cast<double*>(dws + off_E[b]);
            P.d64 = off_d64[b] == SIZE_MAX ? I.d64 : reinterpret_cast<double*>(dws + off_d64[b]);
        } else {
            P.pre_out = off_pre[b] == SIZE_MAX ? I.pre_out : reinterpret_cast<double*>(dws + off_pre[b]);
            P.thr_out = off_thr[b] == SIZE_MAX ? I.thr_out : reinterpret_cast<double*>(dws + off_thr[b]);
            P.trit_out = off_tro[b] == SIZE_MAX ? I.trit_out : dws + off_tro[b];
        }
        reinterpret_cast<int*>(hctl.data() + off_status)[b] = ST_RUNNING;
    }
    memcpy(hctl.data() + off_probs, probs.data(), sizeof(Prob) * np);
    CK(cudaMemcpyAsync(dws, hctl.data(), ctl, cudaMemcpyHostToDevice, stream));
    if (zero_to > zero_from) CK(cudaMemsetAsync(dws + zero_from, 0, zero_to - zero_from, stream));
    for (int b = 0; b < np; ++b) {
        const ProbIn& I = in[b];
        if (off_A[b] != SIZE_MAX)
            CK(cudaMemcpyAsync(dws + off_A[b], I.A, sizeof(float) * (size_t)(I.m * I.n), cudaMemcpyHostToDevice, stream));
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
            setup_kernel<<<dim3((unsigned)tx, (unsigned)ty, (unsigned)np), dim3(32, 8), 0, stream>>>(dprobs);
            CK(cudaGetLastError());
            ++launches;
        }
        CK(cudaEventRecord(ev[1], stream));
        bool any_factor = false;
        for (int b = 0; b < np; ++b) any_factor |= (in[b].mode == MODE_FACTOR);
        if (any_factor) {
            const unsigned gx = (unsigned)(kmax < 8192 ? kmax : 8192);
            init_kernel<<<dim3(gx, (unsigned)np), NTI, 0, stream>>>(dprobs);
            CK(cudaGetLastError());
            ++launches;
        }
        CK(cudaEventRecord(ev[2], stream));
        if (!opt.init_only) {
            KCfg cfg;
            cfg.probs = dprobs;
            cfg.nprob = np;
            cfg.Gg = Gg;
            cfg.NG = NG;
            cfg.gsync = reinterpret_cast<GroupSync*>(dws + off_gsync);
            cfg.slots = reinterpret_cast<Slot*>(dws + off_slots);
            cfg.Lcap = Lcap;
            cfg.m_max = (int)m_max;
            cfg.n_max = (int)n_max;
            cfg.pv_max = pv_max;
            cfg.pu_max = pu_max;
            const double lim = opt.wait_limit_s > 0 ? opt.wait_limit_s : 2.0;
            cfg.limit_ns = (uint64_t)(lim * 1e9);
            cfg.fault_skip = opt.fault_skip;
            void* args[] = {&cfg};
            CK(cudaLaunchCooperativeKernel((void*)als_kernel, dim3((unsigned)(NG * Gg)), dim3(NT), args, smem, stream));
            ++launches;
        }
        CK(cudaEventRecord(ev[3], stream));
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
        if (I.mode != MODE_FACTOR) {
            const int64_t lout = I.mode == MODE_HALF_V ? I.n : I.m;
            if (off_pre[b] != SIZE_MAX) CK(cudaMemcpyAsync(I.pre_out, P.pre_out, sizeof(double) * (size_t)lout, cudaMemcpyDeviceToHost, stream));
            if (off_thr[b] != SIZE_MAX) CK(cudaMemcpyAsync(I.thr_out, P.thr_out, sizeof(double), cudaMemcpyDeviceToHost, stream));
            if (off_tro[b] != SIZE_MAX) CK(cudaMemcpyAsync(I.trit_out, P.trit_out, trit_bytes(lout), cudaMemcpyDeviceToHost, stream));
        }
    }
    CK(cudaMemcpyAsync(hstatus.data(), dws + off_status, sizeof(int) * np, cudaMemcpyDeviceToHost, stream));
    CK(cudaMemcpyAsync(hstats.data(), dws + off_stats, sizeof(DevStats) * np, cudaMemcpyDeviceToHost, stream));
    CK(cudaEventRecord(ev[4], stream));
    CK(cudaStreamSynchronize(stream));

    cudaEventElapsedTime(&ms_setup, ev[0], ev[1]);
    cudaEventElapsedTime(&ms_init, ev[1], ev[2]);
    cudaEventElapsedTime(&ms_als, ev[2], ev[3]);
    cudaEventElapsedTime(&ms_total, ev[0], ev[4]);
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
            st.components += in[b].k;
            st.half_steps += (int64_t)d.half_steps;
            st.fallbacks += (int64_t)d.fallbacks;
            if (b == 0) {
                st.residual_energy = d.norm_a2 > 0 ? 1.0 - d.residual2 / d.norm_a2 : 0.0;
                for (int k2 = 0; k2 < 4; ++k2) st.phase_cycles[k2] = (int64_t)d.phase[k2];
            }
        }
    }
    rc = EXTERND_OK;
    for (int b = 0; b < np; ++b)
        if (statuses[b] != ST_OK) { rc = statuses[b]; break; }

done:
    if (dws) { cudaFreeAsync(dws, stream); cudaStreamSynchronize(stream); }
    for (int i = 0; i < 5; ++i)
        if (ev[i]) cudaEventDestroy(ev[i]);
    cudaGetLastError();
    g_last = st;
    return rc;
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
        I.d64 = opt->d64_out;
    }
    int st = 0;
    return run(&I, 1, ro, reinterpret_cast<cudaStream_t>(stream), &st);
}

int externd_factor(const float* A, int64_t m, int64_t n, double mu, double tau, int iters, uint64_t seed,
                   uint8_t* B_out, float* D_out, uint8_t* C_out, double* energy_out, void* stream) {
    return externd_factor_ex(A, m, n, mu, tau, iters, seed, B_out, D_out, C_out, energy_out, stream, nullptr);
}

int externd_factor_batched(int count, const float* const* A, const int64_t* m, const int64_t* n, const double* mu,
                           const double* tau, int iters, const uint64_t* seed, uint8_t* const* B_out,
                           float* const* D_out, uint8_t* const* C_out, double* const* energy_out, int* status_out,
                           void* stream) {
    if (count < 1 || !A || !m || !n || !mu || !tau || !seed || !B_out || !D_out || !C_out || !status_out)
        return EXTERND_EINVAL;
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
    }
    RunOpts ro;
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
