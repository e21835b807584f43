// Clustered ALS kernel (sm_100a): the greedy sequential ALS of "ExTernD: Expanded-Rank
// Ternary Decomposition" §2.3 (with the §2.5 weights as an option) on a 2-D layout of the
// residual over thread-block clusters.
//
// A matrix is served by G = NC x c CTAs: NC clusters of c CTAs (c = 1, 2, 4, 8 or 16).
// Rows and columns are each cut into c word-aligned quarters (32-index units) Q_0..Q_{c-1};
// every quarter is cut further into NC pieces, piece (q, s) going to cluster q.
//
//   V-layout: CTA (q, r) holds the rows of row quarter r times the columns of cluster q's
//             pieces of every column quarter (its "stripe"), row-major.  The V-step
//             x = R^T u reads the rows of quarter r whose trit changed, sums them over
//             the stripe's columns, and the c CTAs of the cluster add their partial sums
//             in distributed shared memory: CTA (q, s) receives the sums for piece (q, s)
//             and publishes x there.
//   U-layout: CTA (q, r) holds the columns of column quarter r times the rows of cluster
//             q's row pieces (stored column by column); the U-step y = R v is the mirror.
//
// CTA (q, r) also thresholds the output vector over quarter r only (it gathers that
// quarter of the published words and the partial sums of |out| of all G CTAs): that gives
// exactly the changed input trits its next GEMV needs, so no CTA ever thresholds or
// compacts the whole vector.  Everything the cluster needs in full -- nonzero counts, the
// scale's u^T y, the changes of the pending-deflation dot products, the all-zero fallback
// -- is combined from per-quarter partials that ride along with the GEMV partial sums, in
// a fixed order (same bits in every cluster).  The lazy deflation, the tagged-word global
// exchange, the hi + lo residual and the bounded waits are those of the one-CTA-per-stripe
// kernel.
//
// Cluster barriers are collective, so no CTA leaves between two of them: a CTA whose global
// wait gave up carries the failure to the next cluster barrier in its message, and the
// whole cluster returns after it.

namespace externd {

namespace cg = cooperative_groups;

// Per-CTA message of one half-step: partials over the CTA's quarter of the vector it just
// thresholded, sent to every CTA of its cluster together with the GEMV partial sums.
struct Msg {
    int cnt;                    // nonzero trits in the quarter
    int nch;                    // trits that changed in the quarter
    int fail;                   // a wait of this CTA gave up
    int pad;
    double p;                   // sum of |out| over the new support (U-step outputs: u^T y)
    double hs;                  // weighted V-step outputs: sum of h~ over the new support
    double mx;                  // largest |out| in the quarter (fallback), lowest index first
    long long jx;               // its index (LLONG_MAX if the quarter is empty)
    double xj;                  // its signed value
    int ddot[MAX_PENDING];      // change of t_l . t over the quarter (plain objective)
    double ddotw[MAX_PENDING];  // change of sum h~ t_l t over the quarter (weighted U-side)
};

struct Smem2 {
    double* red;        // GEMV row-group partials (NT * 5)
    double* part;       // this CTA's partial sums over its stripe
    double* xin;        // [2][c + 1][wpm] incoming partial sums for the own output piece (slot c: the
                        // all-zero fallback's correction row)
    Msg* out;           // this CTA's message of the current half-step
    Msg* msg;           // [2][c] incoming messages
    double* pd;         // pending scales d_l
    double *coef, *coefV;          // d_l (t_l . u), d_l (t_l . v)
    int *dotU, *dotV;
    double* dotVw;      // weighted: sum h~ t_l v
    double* scal;       // scalars
    double *wS, *wP, *wH, *wM, *wX;    // per-warp partials
    long long* wJ;
    int *wc, *wd, *dotp;
    double* dotpw;
    unsigned long long* clk;
    uint32_t *nzU, *sgU, *onzU, *osgU;    // u over row quarter r (current, previous)
    uint32_t *nzV, *sgV, *onzV, *osgV;    // v over column quarter r
    uint32_t *pnzU, *psgU, *pnzV, *psgV;  // pending components, full length, word-major (stride Ls)
    uint32_t *cnzV, *csgV, *cnzU, *csgU;  // pending bits at the own output pieces
    uint32_t *bnz, *bsg;                  // pending bits along the stripe (fold)
    int *ulist, *vlist;
    float* vwl;         // weighted U-step list coefficients
    double *gV, *gU, *corr;
    long long* fbase;     // fold: first global index of each piece of the stripe
    int* fwidth;          // fold: width of each piece
    struct Ctx* x;        // this CTA's part of the current problem
    double* xq;           // this CTA's quarter of the output vector (staged)
    struct Tot* tot;      // totals of the cluster's messages
    int* stop;            // per-rank stop flags (c), then this CTA's own (index 16)
    double* sS;           // [2][16] single cluster: each rank's partial sum of |out|
};

struct SmemLayout2 {
    size_t red, part, xin, msg, out, pd, coef, coefV, dotU, dotV, dotVw, scal, wS, wP, wH, wM, wX, wJ, wc, wd, dotp, dotpw, clk,
        nzU, sgU, onzU, osgU, nzV, sgV, onzV, osgV, pnzU, psgU, pnzV, psgV, cnzV, csgV, cnzU, csgU, bnz, bsg, ulist, vlist,
        vwl, gV, gU, corr, fbase, fwidth, x, xq, tot, stop, sS, sm, total;
    // m_max, n_max: full lengths; qr_max, qc_max: quarter lengths; sv, su: stripe widths; wpv, wpu:
    // widest output pieces (pitches)
    __host__ __device__ SmemLayout2(int64_t m_max, int64_t n_max, int64_t qr_max, int64_t qc_max, int sv, int su,
                                    int wpv, int wpu, int c, int Lc, int weighted) {
        const size_t Wm = (size_t)((m_max + 31) / 32), Wn = (size_t)((n_max + 31) / 32);
        const size_t Wqr = (size_t)((qr_max + 31) / 32), Wqc = (size_t)((qc_max + 31) / 32);
        const size_t wpm = (size_t)(wpv > wpu ? wpv : wpu), smax = (size_t)(sv > su ? sv : su);
        size_t o = 0;
        auto take = [&](size_t bytes, size_t align) { o = (o + align - 1) / align * align; const size_t at = o; o += bytes; return at; };
        red = take(8 * (size_t)NT * 5, 16);
        part = take(8 * smax, 16);
        xin = take(8 * 2 * (size_t)(c + 1) * wpm, 16);
        msg = take(sizeof(Msg) * 2 * (size_t)c, 16);
        out = take(sizeof(Msg), 16);
        pd = take(8 * (size_t)Lc, 8);
        coef = take(8 * (size_t)Lc, 8);
        coefV = take(8 * (size_t)Lc, 8);
        dotU = take(4 * (size_t)Lc, 4);
        dotV = take(4 * (size_t)Lc, 4);
        dotVw = take(8 * (size_t)Lc, 8);
        scal = take(8 * 16, 8);
        wS = take(8 * NWARP, 8);
        wP = take(8 * NWARP, 8);
        wH = take(8 * NWARP, 8);
        wM = take(8 * NWARP, 8);
        wX = take(8 * NWARP, 8);
        wJ = take(8 * NWARP, 8);
        wc = take(4 * NWARP, 4);
        wd = take(4 * NWARP, 4);
        dotp = take(4 * (size_t)DSTR * MAX_PENDING, 4);
        dotpw = take(weighted ? 8 * (size_t)DSTR * MAX_PENDING : 0, 8);
        clk = take(8 * 12, 8);
        nzU = take(4 * Wqr, 4);
        sgU = take(4 * Wqr, 4);
        onzU = take(4 * Wqr, 4);
        osgU = take(4 * Wqr, 4);
        nzV = take(4 * Wqc, 4);
        sgV = take(4 * Wqc, 4);
        onzV = take(4 * Wqc, 4);
        osgV = take(4 * Wqc, 4);
        pnzU = take(4 * Wm * Lc, 4);
        psgU = take(4 * Wm * Lc, 4);
        pnzV = take(4 * Wn * Lc, 4);
        psgV = take(4 * Wn * Lc, 4);
        cnzV = take(4 * (size_t)wpv, 4);
        csgV = take(4 * (size_t)wpv, 4);
        cnzU = take(4 * (size_t)wpu, 4);
        csgU = take(4 * (size_t)wpu, 4);
        bnz = take(4 * smax, 4);
        bsg = take(4 * smax, 4);
        ulist = take(4 * (size_t)qr_max, 4);
        vlist = take(4 * (size_t)qc_max, 4);
        vwl = take(weighted ? 4 * (size_t)qc_max : 0, 4);
        gV = take(8 * (size_t)wpv, 8);
        gU = take(8 * (size_t)wpu, 8);
        corr = take(8 * wpm, 8);
        fbase = take(8 * 16, 8);
        fwidth = take(4 * 16, 4);
        x = take(512, 16);                                       // sizeof(Ctx) <= 512
        xq = take(8 * (size_t)(qr_max > qc_max ? qr_max : qc_max), 16);
        tot = take(64, 16);                                      // sizeof(Tot) <= 64
        stop = take(4 * 17, 4);
        sS = take(8 * 2 * 16, 8);                                // single cluster: partial sums of |out| per rank
        sm = take(sizeof(Smem2), 16);                            // the pointer table itself
        total = (o + 15) & ~(size_t)15;
    }
};

// ---------------------------------------------------------------------------
// Setup: A into the two 2-D layouts (the high halves; the low halves start at zero).
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(256) setup2_kernel(const Prob* __restrict__ probs) {
    const Prob& P = probs[blockIdx.z];
    const int64_t m = P.m, n = P.n;
    const int64_t tiles_x = (n + 31) >> 5, tiles_y = (m + 31) >> 5;
    if ((int64_t)blockIdx.x >= tiles_x || (int64_t)blockIdx.y >= tiles_y) return;
    __shared__ double red[9];
    const Grid2& g = P.g2;
    const Part QR = g.qr(), QC = g.qc();
    const int64_t rbase = (int64_t)blockIdx.y * 32, cbase = (int64_t)blockIdx.x * 32;
    double ss = 0.0;
    unsigned bad = 0;
    const int64_t c = cbase + threadIdx.x;
    int sc = 0, qv = 0, offv = 0;
    int64_t lc = 0;
    if (c < n) {
        sc = QC.owner(c);
        lc = c - QC.start(sc);
        const Part pc = g.pcol(sc);
        qv = pc.owner(lc);
        offv = g.soffV(qv, sc) + (int)(lc - pc.start(qv));
    }
    for (int rr = threadIdx.y; rr < 32; rr += 8) {
        const int64_t r = rbase + rr;
        if (r < m && c < n) {
            const float v = __ldcg(P.A + r * n + c);
            if (!isfinite(v)) ++bad;
            ss += (double)v * (double)v * (P.hw ? (double)__ldg(P.hw + c) : 1.0);
            const int sr = QR.owner(r);
            const int64_t lr = r - QR.start(sr);
            P.Rv[(int64_t)(qv * g.c + sr) * P.bsv + lr * g.pitchV(qv) + offv] = v;
            const Part pr = g.prow(sr);
            const int qu = pr.owner(lr);
            P.Ru[(int64_t)(qu * g.c + sc) * P.bsu + lc * g.pitchU(qu) + g.soffU(qu, sr) + (lr - pr.start(qu))] = v;
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
// GEMV partial sums: out[j] = sum over the list entries e of coef_e * blk[row_e][j] for
// the stripe columns j < pitch (fp64, fixed order: row groups, then the groups in order).
// ---------------------------------------------------------------------------

template <int VEC, bool WL>
__device__ void gemv_part(const float* __restrict__ blk, int pitch, const int* __restrict__ list,
                          const float* __restrict__ wl, int nlist, double* red, double* out) {
    const int nvec = pitch / VEC;
    if (nvec <= 0) return;
    if (nvec <= NT) {
        const int lanes = NT / nvec;
        const int act = min(lanes, nlist);
        const int j = threadIdx.x % nvec;
        const int g = threadIdx.x / nvec;
        const int rs = pitch | 1;
        if (g < act) {
            double acc[VEC];
            #pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = 0.0;
            const float* base = blk + j * VEC;
            const int per = (nlist + lanes - 1) / lanes;
            if (per <= 1) gemv_rows<VEC, 1, WL>(acc, base, list, wl, nlist, g, lanes);
            else if (per <= 2) gemv_rows<VEC, 2, WL>(acc, base, list, wl, nlist, g, lanes);
            else if (per <= 4) gemv_rows<VEC, 4, WL>(acc, base, list, wl, nlist, g, lanes);
            else gemv_rows<VEC, GEMV_U<VEC>(), WL>(acc, base, list, wl, nlist, g, lanes);
            #pragma unroll
            for (int e = 0; e < VEC; ++e) red[g * rs + j * VEC + e] = acc[e];
        }
        __syncthreads();
        int tpc = 1;
        while (tpc < 32 && tpc * 2 * pitch <= NT) tpc *= 2;
        const int cpr = NT / tpc;
        for (int cb = 0; cb < pitch; cb += cpr) {
            const int col = cb + (int)threadIdx.x / tpc;
            const int s = (int)threadIdx.x % tpc;
            double v = 0.0;
            if (col < pitch)
                for (int gg = s; gg < act; gg += tpc) v += red[gg * rs + col];
            for (int o = tpc >> 1; o; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
            if (s == 0 && col < pitch) out[col] = v;
        }
    } else {
        constexpr int U = GEMV_U<VEC>();
        for (int j = threadIdx.x; j < nvec; j += NT) {
            double acc[VEC];
            #pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = 0.0;
            const float* base = blk + j * VEC;
            gemv_rows<VEC, U, WL>(acc, base, list, wl, nlist, 0, 1);
            #pragma unroll
            for (int e = 0; e < VEC; ++e) out[j * VEC + e] = acc[e];
        }
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// This CTA's part of the current problem, kept in shared memory (so that the half-step
// code holds none of it in registers).
// ---------------------------------------------------------------------------

struct Ctx {
    int64_t m, n;
    int c, NC, q, r, qid, Gg, Ls, wpm;
    int64_t qr0, qr1;       // row quarter r (input of the V-step, output of the U-step)
    int64_t qc0, qc1;       // column quarter r
    int pitchV, pitchU;     // stripe widths of cluster q
    int64_t pv0, pu0;       // own output pieces: columns [pv0, pv0 + wpv), rows [pu0, pu0 + wpu)
    int wpv, wpu;
    int soffV[17], soffU[17];   // piece offsets in the two stripes
    float *blkV, *bloV, *blkU, *bloU;
    double tauV, tauU;      // tau / length
    int lead, skip;
    // running state of the launch and of the problem (kept here rather than in registers
    // across the out-of-line half-steps)
    unsigned arrivals;      // group exchanges this CTA took part in (counter targets)
    unsigned round;         // cluster message rounds (parity of the double-buffered slots)
    unsigned gen;           // half-steps of this problem (tags of the published words)
    int pad0;
    double N0, RN2;
    unsigned long long sum_nu, sum_nv, sum_du, sum_dv, sum_nunv, hs, fb, sgh;
};
static_assert(sizeof(Ctx) <= 512, "shared-memory slot of the context");

__device__ void ctx_init(const Prob& P, int q, int r, const KCfg& cfg, Ctx& x) {
    if (threadIdx.x == 0) {
        x.gen = 0;
        x.sum_nu = x.sum_nv = x.sum_du = x.sum_dv = x.sum_nunv = x.hs = x.fb = x.sgh = 0ull;
        const Grid2& g = P.g2;
        x.m = P.m;
        x.n = P.n;
        x.c = g.c;
        x.NC = g.NC;
        x.q = q;
        x.r = r;
        x.qid = q * g.c + r;
        x.Gg = cfg.Gg;
        x.Ls = cfg.Lcap > 0 ? cfg.Lcap : 1;
        x.wpm = cfg.wpm;
        const Part QR = g.qr(), QC = g.qc();
        x.qr0 = QR.start(r);
        x.qr1 = QR.end(r);
        x.qc0 = QC.start(r);
        x.qc1 = QC.end(r);
        int a = 0, b = 0;
        for (int s = 0; s < g.c; ++s) {
            x.soffV[s] = a;
            x.soffU[s] = b;
            a += g.pcol(s).pitch(q);
            b += g.prow(s).pitch(q);
        }
        x.soffV[g.c] = a;
        x.soffU[g.c] = b;
        x.pitchV = a;
        x.pitchU = b;
        const Part pc = g.pcol(r), pr = g.prow(r);
        x.pv0 = x.qc0 + pc.start(q);
        x.wpv = (int)(pc.end(q) - pc.start(q));
        x.pu0 = x.qr0 + pr.start(q);
        x.wpu = (int)(pr.end(q) - pr.start(q));
        const int64_t cta = (int64_t)x.qid;
        x.blkV = P.Rv + cta * P.bsv;
        x.bloV = P.Rv_lo + cta * P.bsv;
        x.blkU = P.Ru + cta * P.bsu;
        x.bloU = P.Ru_lo + cta * P.bsu;
        x.tauV = P.tau / (double)P.n;
        x.tauU = P.tau / (double)P.m;
        x.lead = (x.qid == 0);
        x.skip = (cfg.fault_skip == x.qid);
    }
    __syncthreads();
}

// ---------------------------------------------------------------------------
// Threshold of this CTA's quarter of the output vector (T_tau of §2.2 at the threshold of
// the whole vector): the quarter's values are staged in xq (shared memory).  Writes the new
// and previous masks, the list of changed trits for the next GEMV (element offsets in this
// CTA's block of the other layout, index order) and the quarter's partials in *mout.
// WD: the weighted objective's V-step outputs (the dots and the list coefficients carry h~,
// and the sum of h~ over the support is returned); want_p: U-step outputs (u^T y).
// ---------------------------------------------------------------------------

template <bool WD>
__device__ __noinline__ void threshold_quarter(const double* xq, int64_t q0, int64_t q1, double thr, bool want_p,
                                               uint32_t* nz, uint32_t* sg, uint32_t* onz, uint32_t* osg, int* list,
                                               int rowpitch, int L, int Ls, const uint32_t* pnz, const uint32_t* psg,
                                               const float* hw, float* wl, const Smem2& s, Msg* mout) {
    const int lane = lane_id(), warp = warp_id();
    const int64_t len = q1 - q0;
    const int W = (int)((len + 31) >> 5);
    const int per = (W + NWARP - 1) / NWARP;
    const int w0 = min(W, warp * per), w1 = min(W, w0 + per);
    const int64_t gw0 = q0 >> 5;   // quarters start on a word boundary
    int cnt = 0, dcnt = 0, dot = 0;
    double ps = 0.0, hsum = 0.0, dotw = 0.0, mx = -1.0, xj = 0.0;
    long long jx = LLONG_MAX;
    for (int w = w0; w < w1; ++w) {
        const int64_t li = ((int64_t)w << 5) + lane;
        double x = 0.0;
        if (li < len) {
            x = xq[li];
            const double a = fabs(x);
            if (a > mx) { mx = a; jx = q0 + li; xj = x; }
        }
        const bool z = fabs(x) > thr;
        const uint32_t bz = __ballot_sync(FULL, z);
        const uint32_t bs = __ballot_sync(FULL, z && (x < 0.0));
        if (want_p && z) ps += fabs(x);
        if constexpr (WD) if (z) hsum += (double)__ldg(hw + q0 + li);
        const uint32_t oz = nz[w], os = sg[w];
        uint32_t dn, dt;
        const uint32_t ch = delta_mask(oz, os, bz, bs, dn, dt);   // the same in every lane
        __syncwarp();
        if (lane == 0) {
            nz[w] = bz; sg[w] = bs; onz[w] = oz; osg[w] = os;
            cnt += __popc(bz);
            dcnt += __popc(ch);
        }
        if (ch && L > 0) {
            // change of t_l . t over this word (lane l = pending component l)
            if constexpr (WD) {
                const float hword = li < len ? __ldg(hw + q0 + li) : 0.f;
                const uint32_t pz = lane < L ? pnz[(gw0 + w) * Ls + lane] : 0u;
                const uint32_t pg = lane < L ? psg[(gw0 + w) * Ls + lane] : 0u;
                uint32_t mine = pz & ch;
                const int rounds = (int)__reduce_max_sync(FULL, (unsigned)__popc(mine));
                for (int t = 0; t < rounds; ++t) {
                    const int b = mine ? __ffs(mine) - 1 : 0;
                    const double hv = (double)__shfl_sync(FULL, hword, b);
                    if (mine) {
                        const double dv = (((dn >> b) & 1u) ? -1.0 : 1.0) * (((dt >> b) & 1u) ? 2.0 : 1.0);
                        dotw += ((pg >> b) & 1u) ? -hv * dv : hv * dv;
                        mine &= mine - 1u;
                    }
                }
            } else if (lane < L) {
                const uint32_t pz = pnz[(gw0 + w) * Ls + lane], pg = psg[(gw0 + w) * Ls + lane];
                const uint32_t zn = pz & bz & ch, zo = pz & oz & ch;
                const uint32_t sn = pg ^ bs, so = pg ^ os;
                dot += (__popc(zn & ~sn) - __popc(zn & sn)) - (__popc(zo & ~so) - __popc(zo & so));
            }
        }
    }
    #pragma unroll
    for (int o = 16; o; o >>= 1) {
        ps += __shfl_xor_sync(FULL, ps, o);
        hsum += __shfl_xor_sync(FULL, hsum, o);
        const double m2 = __shfl_xor_sync(FULL, mx, o);
        const long long j2 = __shfl_xor_sync(FULL, jx, o);
        const double x2 = __shfl_xor_sync(FULL, xj, o);
        if (m2 > mx || (m2 == mx && j2 < jx)) { mx = m2; jx = j2; xj = x2; }
    }
    if (lane == 0) {
        s.wc[warp] = cnt;
        s.wd[warp] = dcnt;
        s.wP[warp] = ps;
        s.wH[warp] = hsum;
        s.wM[warp] = mx;
        s.wJ[warp] = jx;
        s.wX[warp] = xj;
    }
    if (lane < L) {
        if constexpr (WD) s.dotpw[lane * DSTR + warp] = dotw;
        else s.dotp[lane * DSTR + warp] = dot;
    }
    __syncthreads();
    const int dw = lane < NWARP ? s.wd[lane] : 0;
    const int off = __reduce_add_sync(FULL, lane < warp ? dw : 0);
    if (warp == 0) {
        const int tot = __reduce_add_sync(FULL, lane < NWARP ? s.wc[lane] : 0);
        const int dtot = __reduce_add_sync(FULL, dw);
        double p2 = lane < NWARP ? s.wP[lane] : 0.0, h2 = lane < NWARP ? s.wH[lane] : 0.0;
        double m2 = lane < NWARP ? s.wM[lane] : -1.0, x2 = lane < NWARP ? s.wX[lane] : 0.0;
        long long j2 = lane < NWARP ? s.wJ[lane] : LLONG_MAX;
        #pragma unroll
        for (int o = 16; o; o >>= 1) {
            p2 += __shfl_xor_sync(FULL, p2, o);
            h2 += __shfl_xor_sync(FULL, h2, o);
            const double m3 = __shfl_xor_sync(FULL, m2, o);
            const long long j3 = __shfl_xor_sync(FULL, j2, o);
            const double x3 = __shfl_xor_sync(FULL, x2, o);
            if (m3 > m2 || (m3 == m2 && j3 < j2)) { m2 = m3; j2 = j3; x2 = x3; }
        }
        if (lane == 0) {
            mout->cnt = tot;
            mout->nch = dtot;
            mout->fail = 0;
            mout->p = p2;
            mout->hs = h2;
            mout->mx = m2;
            mout->jx = j2;
            mout->xj = x2;
        }
    }
    for (int l = warp; l < L; l += NWARP) {
        if constexpr (WD) {
            double d = lane < NWARP ? s.dotpw[l * DSTR + lane] : 0.0;
            #pragma unroll
            for (int o = 16; o; o >>= 1) d += __shfl_xor_sync(FULL, d, o);
            if (lane == 0) { mout->ddotw[l] = d; mout->ddot[l] = 0; }
        } else {
            const int d = __reduce_add_sync(FULL, lane < NWARP ? s.dotp[l * DSTR + lane] : 0);
            if (lane == 0) { mout->ddot[l] = d; mout->ddotw[l] = 0.0; }
        }
    }
    // the list, one word at a time across the lanes
    int run = off;
    for (int w = w0; w < w1; ++w) {
        uint32_t ng, tw;
        const uint32_t ch = delta_mask(onz[w], osg[w], nz[w], sg[w], ng, tw);
        if ((ch >> lane) & 1u) {
            const int at = run + __popc(ch & ((1u << lane) - 1u));
            const int e = delta_entry(((unsigned)w << 5) + lane, rowpitch, ng, tw, lane);
            list[at] = e;
            if constexpr (WD) wl[at] = entry_coef(e) * __ldg(hw + q0 + ((int64_t)w << 5) + lane);
        }
        run += __popc(ch);
    }
    __syncthreads();
}

// Start trits of a component over row quarter [q0, q1): masks, list (against u = 0) and
// the quarter's partials (count and t_l . u0 of the pending components).
__device__ __noinline__ void start_quarter(const uint32_t* words, int64_t q0, int64_t q1, uint32_t* nz, uint32_t* sg,
                                           uint32_t* onz, uint32_t* osg, int* list, int rowpitch, int L, int Ls,
                                           const uint32_t* pnz, const uint32_t* psg, const Smem2& s, Msg* mout) {
    const int lane = lane_id(), warp = warp_id();
    const int64_t len = q1 - q0;
    const int W = (int)((len + 31) >> 5);
    for (int w = threadIdx.x; w < W; w += NT) {
        const int64_t gw = (q0 >> 5) + w;   // 32 trits = two packed words
        const uint32_t lo = __ldcg(words + 2 * gw), hi = __ldcg(words + 2 * gw + 1);
        uint32_t z = compact_even(lo) | (compact_even(hi) << 16);
        const uint32_t sb = compact_even(lo >> 1) | (compact_even(hi >> 1) << 16);
        const int64_t rem = len - ((int64_t)w << 5);
        if (rem < 32) z &= (1u << rem) - 1u;
        nz[w] = z;
        sg[w] = sb & z;
        onz[w] = 0u;
        osg[w] = 0u;
    }
    __syncthreads();
    const int per = (W + NWARP - 1) / NWARP;
    const int w0 = min(W, warp * per), w1 = min(W, w0 + per);
    int cnt = 0, dot = 0;
    for (int w = w0; w < w1; ++w) {
        const uint32_t z = nz[w], g = sg[w];
        if (lane == 0) cnt += __popc(z);
        if (lane < L) {
            const uint32_t pz = pnz[((q0 >> 5) + w) * Ls + lane] & z, pg = psg[((q0 >> 5) + w) * Ls + lane] ^ g;
            dot += __popc(pz & ~pg) - __popc(pz & pg);
        }
    }
    if (lane == 0) s.wc[warp] = cnt;
    if (lane < L) s.dotp[lane * DSTR + warp] = dot;
    __syncthreads();
    const int dw = lane < NWARP ? s.wc[lane] : 0;
    const int off = __reduce_add_sync(FULL, lane < warp ? dw : 0);
    if (warp == 0) {
        const int tot = __reduce_add_sync(FULL, dw);
        if (lane == 0) {
            mout->cnt = tot;
            mout->nch = tot;
            mout->fail = 0;
            mout->p = 0.0;
            mout->hs = 0.0;
            mout->mx = 0.0;
            mout->jx = LLONG_MAX;
            mout->xj = 0.0;
        }
    }
    for (int l = warp; l < L; l += NWARP) {
        const int d = __reduce_add_sync(FULL, lane < NWARP ? s.dotp[l * DSTR + lane] : 0);
        if (lane == 0) { mout->ddot[l] = d; mout->ddotw[l] = 0.0; }
    }
    int run = off;
    for (int w = w0; w < w1; ++w) {
        const uint32_t z = nz[w];
        if ((z >> lane) & 1u)
            list[run + __popc(z & ((1u << lane) - 1u))] =
                (int)((((unsigned)w << 5) + lane) * (unsigned)rowpitch) | (int)(((sg[w] >> lane) & 1u) << 31);
        run += __popc(z);
    }
    __syncthreads();
}

// Totals of the c messages of parity hb, in rank order (warp 0; read by all after a barrier).
struct Tot {
    int cnt, nch, fail, pad;
    double p, hs, mx, xj;
    long long jx;
};
static_assert(sizeof(Tot) <= 64, "shared-memory slot of the totals");

// Lane s of warp 0 takes rank s's message; fixed butterflies combine them (the same order in
// every CTA of every cluster).
__device__ __forceinline__ void totals(const Msg* msg, int c, int hb, Tot* out) {
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int cnt = 0, nch = 0, fail = 0;
        double p = 0.0, hs = 0.0, mx = -1.0, xj = 0.0;
        long long jx = LLONG_MAX;
        if (lane < c) {
            const Msg& m = msg[hb * c + lane];
            cnt = m.cnt;
            nch = m.nch;
            fail = m.fail;
            p = m.p;
            hs = m.hs;
            if (m.jx != LLONG_MAX) { mx = m.mx; jx = m.jx; xj = m.xj; }
        }
        cnt = __reduce_add_sync(FULL, cnt);
        nch = __reduce_add_sync(FULL, nch);
        fail = __reduce_or_sync(FULL, fail);
        #pragma unroll
        for (int o = 16; o; o >>= 1) {
            p += __shfl_xor_sync(FULL, p, o);
            hs += __shfl_xor_sync(FULL, hs, o);
            const double m2 = __shfl_xor_sync(FULL, mx, o);
            const long long j2 = __shfl_xor_sync(FULL, jx, o);
            const double x2 = __shfl_xor_sync(FULL, xj, o);
            if (m2 > mx || (m2 == mx && j2 < jx)) { mx = m2; jx = j2; xj = x2; }
        }
        if (lane == 0) {
            Tot t{cnt, nch, fail, 0, p, hs, mx, xj, jx};
            *out = t;
        }
    }
}

// Words of a message that carry information: the header and the integer dots, plus the
// weighted dots in the weighted kernel.
__device__ __forceinline__ int msg_words(bool weighted) {
    return (int)((offsetof(Msg, ddotw) + (weighted ? sizeof(double) * MAX_PENDING : 0)) / 4);
}

// Trace of one half-step (test hook): this CTA's quarter of the vector, its trits, and
// (rank 0) the threshold.
__device__ __noinline__ void trace_quarter(const double* xq, int64_t q0, int64_t q1, double thr, const uint32_t* nz,
                                           const uint32_t* sg, double* pre, double* thr_out, uint8_t* trits,
                                           bool write_thr) {
    for (int64_t t = threadIdx.x; t < q1 - q0; t += NT) pre[q0 + t] = xq[t];
    if (write_thr && threadIdx.x == 0) *thr_out = thr;
    const int W = (int)((q1 - q0 + 31) >> 5);
    uint32_t* out = reinterpret_cast<uint32_t*>(trits);
    for (int w = threadIdx.x; w < W; w += NT) {
        const uint32_t z = nz[w], g = sg[w] & z;
        const int64_t pw = (q0 >> 4) + 2 * (int64_t)w;
        out[pw] = spread_even(z) | (spread_even(g) << 1);
        out[pw + 1] = spread_even(z >> 16) | (spread_even(g >> 16) << 1);
    }
}

// Bits of the pending components (bit l = component l) along a stripe made of pieces:
// stripe entry j of piece s is global index base(s) + (j - soff[s]).
__device__ void stripe_bits(const int* soff, int c, const long long* base, const int* width, const uint32_t* pnz,
                            const uint32_t* psg, int L, int Ls, int pitch, uint32_t* bnz, uint32_t* bsg) {
    for (int j = threadIdx.x; j < pitch; j += NT) {
        int sp = 0;
        while (sp + 1 < c && soff[sp + 1] <= j) ++sp;
        const int k = j - soff[sp];
        uint32_t z = 0u, g = 0u;
        if (k < width[sp]) {
            const int64_t gi = base[sp] + k;
            const uint32_t bit = 1u << (gi & 31);
            for (int l = 0; l < L; ++l) {
                if (pnz[(gi >> 5) * Ls + l] & bit) {
                    z |= 1u << l;
                    if (psg[(gi >> 5) * Ls + l] & bit) g |= 1u << l;
                }
            }
        }
        bnz[j] = z;
        bsg[j] = g;
    }
}

// Per-output pending bits of slot l at global positions [p0, p0 + w) from the full masks.
__device__ __forceinline__ void push_bits(const uint32_t* pnz, const uint32_t* psg, int l, int Ls, int64_t p0, int w,
                                          uint32_t* cnz, uint32_t* csg) {
    for (int j = threadIdx.x; j < w; j += NT) {
        const int64_t gi = p0 + j;
        const uint32_t bit = 1u << (gi & 31);
        if (pnz[(gi >> 5) * Ls + l] & bit) {
            cnz[j] |= 1u << l;
            if (psg[(gi >> 5) * Ls + l] & bit) csg[j] |= 1u << l;
        }
    }
}

// ---------------------------------------------------------------------------
// One half-step of the clustered kernel.  U = false: V-step x = R^T u (input u over the row
// quarter, output x over the column pieces); U = true: U-step y = R v.
//   1. GEMV over this CTA's block for its input quarter's changed trits;
//   2. partial sums to the CTAs owning the stripe's pieces and this CTA's message (the
//      partials of the input vector's last threshold) to all CTAs of the cluster; barrier;
//   3. totals; the all-zero fallback of the input vector; the pending dots;
//   4. own output piece: sum of the cluster's partials, running sums, corrections, publish;
//   5. group exchange: partial sums of |out| and this CTA's quarter of the output vector;
//   6. threshold of the quarter -> masks, next list, next message.
// Totals of the input vector go to s.scal[0..2] (count, changes, weighted support sum).
// Returns 1 if the cluster must stop (a CTA reported a failed wait), else 0; a failed wait
// of this CTA is reported in its next message.
// ---------------------------------------------------------------------------

template <bool WTD, bool U>
__device__ __noinline__ int half2(const Prob& P, Ctx& x, const KCfg& cfg, const Smem2& s, GroupSync* gs, int nlist,
                                  int L, int64_t trace_at) {
    cg::cluster_group cl = cg::this_cluster();
    const int c = x.c, Ls = x.Ls, wpm = x.wpm;
    const int tid = threadIdx.x;
    const unsigned gen = x.gen + 1, hb = x.round & 1u;
    const unsigned tag = gen_tag(gen);
    __syncthreads();   // every thread has read gen and round
    if (tid == 0) { x.gen = gen; x.round += 1u; x.arrivals += 1u; }
    // ---- 1. GEMV
    if (U) gemv_part<4, WTD>(x.blkU, x.pitchU, s.vlist, s.vwl, nlist, s.red, s.part);
    else gemv_part<4, false>(x.blkV, x.pitchV, s.ulist, nullptr, nlist, s.red, s.part);
    phase_mark(s.clk, 0);
    // ---- 2. partial sums and message to the cluster
    {
        const int pitch = U ? x.pitchU : x.pitchV;
        const int* soff = U ? x.soffU : x.soffV;
        for (int j = tid; j < pitch; j += NT) {
            int sp = 0;
            while (sp + 1 < c && soff[sp + 1] <= j) ++sp;
            cl.map_shared_rank(s.xin, sp)[((size_t)hb * (c + 1) + x.r) * wpm + (j - soff[sp])] = s.part[j];
        }
        const int words = msg_words(WTD);
        for (int t = tid; t < words * c; t += NT) {
            const int peer = t / words, k = t - peer * words;
            reinterpret_cast<uint32_t*>(cl.map_shared_rank(s.msg + hb * c + x.r, peer))[k] =
                reinterpret_cast<const uint32_t*>(s.out)[k];
        }
    }
    cl.sync();
    phase_mark(s.clk, 1);
    // ---- 3. totals, fallback, dots
    totals(s.msg, c, hb, s.tot);
    __syncthreads();
    if (s.tot->fail) return 1;
    const bool fbk = (s.tot->cnt == 0);
    int64_t fj = 0;
    int fsg = 0;
    if (fbk) {
        // no trit of the input vector survived T_tau: the lowest index among the largest
        // magnitudes keeps its sign (§2.2); the speculative change list left it at 0, so the
        // CTA of each cluster owning it sends that row times the trit in the extra slot
        fj = (s.tot->jx == LLONG_MAX) ? 0 : s.tot->jx;
        fsg = (s.tot->xj < 0.0) ? -1 : 1;
        const int64_t in0 = U ? x.qc0 : x.qr0, in1 = U ? x.qc1 : x.qr1;
        if (fj >= in0 && fj < in1) {
            const int64_t lj = fj - in0;
            uint32_t* nz = U ? s.nzV : s.nzU;
            uint32_t* sg = U ? s.sgV : s.sgU;
            if (tid == 0) {
                nz[lj >> 5] |= 1u << (lj & 31);
                if (fsg < 0) sg[lj >> 5] |= 1u << (lj & 31);
            }
            const double cf = (double)fsg * ((U && WTD) ? (double)__ldg(P.hw + fj) : 1.0);
            const int pitch = U ? x.pitchU : x.pitchV;
            const int* soff = U ? x.soffU : x.soffV;
            const float* row = (U ? x.blkU : x.blkV) + lj * pitch;
            for (int e = tid; e < pitch; e += NT) {
                int sp = 0;
                while (sp + 1 < c && soff[sp + 1] <= e) ++sp;
                cl.map_shared_rank(s.xin, sp)[((size_t)hb * (c + 1) + c) * wpm + (e - soff[sp])] = cf * (double)__ldcg(row + e);
            }
        }
        cl.sync();
    }
    for (int l = tid; l < L; l += NT) {
        const uint32_t bit = 1u << (fj & 31);
        if (!U) {
            int d = s.dotU[l];
            for (int rr = 0; rr < c; ++rr) d += s.msg[hb * c + rr].ddot[l];
            if (fbk && (s.pnzU[(fj >> 5) * Ls + l] & bit)) d += ((s.psgU[(fj >> 5) * Ls + l] & bit) ? -1 : 1) * fsg;
            s.dotU[l] = d;
            s.coef[l] = s.pd[l] * (double)d;
        } else if (WTD) {
            double d = s.dotVw[l];
            for (int rr = 0; rr < c; ++rr) d += s.msg[hb * c + rr].ddotw[l];
            if (fbk && (s.pnzV[(fj >> 5) * Ls + l] & bit))
                d += ((s.psgV[(fj >> 5) * Ls + l] & bit) ? -1.0 : 1.0) * (double)fsg * (double)__ldg(P.hw + fj);
            s.dotVw[l] = d;
            s.coefV[l] = s.pd[l] * d;
        } else {
            int d = s.dotV[l];
            for (int rr = 0; rr < c; ++rr) d += s.msg[hb * c + rr].ddot[l];
            if (fbk && (s.pnzV[(fj >> 5) * Ls + l] & bit)) d += ((s.psgV[(fj >> 5) * Ls + l] & bit) ? -1 : 1) * fsg;
            s.dotV[l] = d;
            s.coefV[l] = s.pd[l] * (double)d;
        }
    }
    if (tid == 0) {
        const int cnt = fbk ? 1 : s.tot->cnt;
        s.scal[0] = (double)cnt;
        if (U) s.scal[2] = WTD ? (fbk ? (double)__ldg(P.hw + fj) : s.tot->hs) : (double)cnt;
        (U ? x.sum_nv : x.sum_nu) += (unsigned long long)cnt;
        (U ? x.sum_dv : x.sum_du) += (unsigned long long)s.tot->nch;
        x.fb += fbk ? 1ull : 0ull;
        x.hs += 1ull;
    }
    __syncthreads();
    // ---- 4. own output piece
    const int w = U ? x.wpu : x.wpv;
    double* g = U ? s.gU : s.gV;
    {
        HalfCorr hc{U ? s.coefV : s.coef, U ? s.cnzU : s.cnzV, U ? s.csgU : s.csgV, s.corr, g, L};
        corrections(w, hc);
    }
    __syncthreads();
    double S = 0.0;
    // one cluster: its CTA r publishes exactly its quarter r, so the exchange stays on chip
    // (the fault-injection hook, a CTA that never signals a global arrival, keeps the global path)
    const bool single = (x.NC == 1) && cfg.fault_skip < 0;
    {
        unsigned long long* gout = U ? P.ybuf : P.xbuf;
        const int64_t out0 = U ? x.pu0 : x.pv0;
        for (int j = tid; j < w; j += NT) {
            double d = 0.0;
            for (int rr = 0; rr < c; ++rr) d += s.xin[((size_t)hb * (c + 1) + rr) * wpm + j];
            if (fbk) d += s.xin[((size_t)hb * (c + 1) + c) * wpm + j];
            const double gj = g[j] + d;
            g[j] = gj;
            const double v = L > 0 ? gj - s.corr[j] : gj;
            if (single) {
                // the value the threshold sees is the one the group exchange would carry: 44 bits
                const unsigned long long t = tag_value(v, tag) & ~0xFFull;
                const double vt = __longlong_as_double((long long)t);
                s.xq[j] = vt;
                S += fabs(vt);
            } else {
                emit_tagged(v, out0 + j, gout, tag, x.skip != 0, S);
            }
        }
        #pragma unroll
        for (int o = 16; o; o >>= 1) S += __shfl_xor_sync(FULL, S, o);
    }
    phase_mark(s.clk, 2);
    int ok = 1;
    const int lane = lane_id(), warp = warp_id();
    const int64_t q0 = U ? x.qr0 : x.qc0, q1 = U ? x.qr1 : x.qc1;
    double thr = 0.0;
    if (single) {
        // ---- 5'. the cluster is the group: partial sums of |out| in distributed shared memory
        if (lane == 0) s.wS[warp] = S;
        __syncthreads();
        if (warp == 0) {
            double S2 = lane < NWARP ? s.wS[lane] : 0.0;
            #pragma unroll
            for (int o = 16; o; o >>= 1) S2 += __shfl_xor_sync(FULL, S2, o);
            if (lane < c) cl.map_shared_rank(s.sS, lane)[hb * 16 + x.r] = S2;
        }
        cl.sync();
        double St = 0.0;
        for (int rr = 0; rr < c; ++rr) St += s.sS[hb * 16 + rr];
        thr = St * (U ? x.tauU : x.tauV);
        phase_mark(s.clk, 5);
    } else {
    // ---- 5. group exchange: publish the partial, arrive, wait; stage the quarter and the partials
    unsigned long long* partials = U ? P.partU : P.partV;
    if (lane == 0) s.wS[warp] = S;
    __syncthreads();
    if (warp == 0) {
        double S2 = lane < NWARP ? s.wS[lane] : 0.0;
        #pragma unroll
        for (int o = 16; o; o >>= 1) S2 += __shfl_xor_sync(FULL, S2, o);
        if (lane == 0 && !x.skip) {
            st_relaxed_u64(partials + x.qid, tag_value(S2, tag));
            red_relaxed_add(&gs->ctr[x.qid % NCTR][0], 1u);
        }
    }
    const int Gg = x.Gg;
    if (tid < NCTR && tid < Gg) {
        const unsigned want = x.arrivals * (unsigned)((Gg - tid + NCTR - 1) / NCTR);
        const unsigned* ctr = &gs->ctr[tid][0];
        if ((int)(ld_relaxed_u32(ctr) - want) < 0) {
            const uint64_t t0 = gtimer();
            unsigned spins = 0;
            while ((int)(ld_relaxed_u32(ctr) - want) < 0) {
                if ((++spins & 15u) == 0u) {
                    if (ld_relaxed_s32(&gs->abort)) { ok = 0; break; }
                    if (gtimer() - t0 > cfg.limit_ns) {
                        atomicExch(&gs->abort, 1);
                        atomicCAS(P.status, ST_RUNNING, ST_ETIMEOUT);
                        ok = 0;
                        break;
                    }
                }
            }
        }
    }
    ok = __syncthreads_and(ok);
    phase_mark(s.clk, 3);
    const unsigned long long* gvec = U ? P.ybuf : P.xbuf;
    if (ok) {
        // the quarter's words and the partials are loaded together (one round trip)
        for (int64_t t = tid; t < q1 - q0; t += NT) {
            unsigned long long b = ld_relaxed_u64(gvec + q0 + t);
            if ((unsigned)(b & 0xFFull) != tag) b = wait_tagged(gvec + q0 + t, tag, gs, cfg.limit_ns, P.status, ok);
            s.xq[t] = untag(b);
        }
        if (warp * 32 < Gg) {
            double Sq = 0.0;
            if (tid < Gg) Sq = untag(wait_tagged(partials + tid, tag, gs, cfg.limit_ns, P.status, ok));
            #pragma unroll
            for (int o = 16; o; o >>= 1) Sq += __shfl_xor_sync(FULL, Sq, o);
            if (lane == 0) s.wS[warp] = Sq;
        }
        ok = __syncthreads_and(ok);
        double St = 0.0;
        for (int w2 = 0; w2 < Gg; w2 += 32) St += s.wS[w2 >> 5];
        thr = St * (U ? x.tauU : x.tauV);
    }
    phase_mark(s.clk, 5);
    }
    if (!ok) {
        // report it at the next cluster barrier
        if (tid == 0) { s.out->fail = 1; s.out->cnt = 1; s.out->nch = 0; }
        __syncthreads();
        return 0;
    }
    // ---- 6. threshold of the quarter (§2.2), next list and message
    if (U) {
        threshold_quarter<false>(s.xq, q0, q1, thr, true, s.nzU, s.sgU, s.onzU, s.osgU, s.ulist, x.pitchV, L, Ls, s.pnzU,
                                 s.psgU, nullptr, nullptr, s, s.out);
        if (trace_at >= 0)
            trace_quarter(s.xq, q0, q1, thr, s.nzU, s.sgU, P.tr_pre_u + trace_at * P.m, P.tr_thr_u + trace_at,
                          P.tr_trit_u + trace_at * P.b_bytes, x.r == 0);
    } else {
        threshold_quarter<WTD>(s.xq, q0, q1, thr, false, s.nzV, s.sgV, s.onzV, s.osgV, s.vlist, x.pitchU, L, Ls,
                               s.pnzV, s.psgV, P.hw, s.vwl, s, s.out);
        if (trace_at >= 0)
            trace_quarter(s.xq, q0, q1, thr, s.nzV, s.sgV, P.tr_pre_v + trace_at * P.n, P.tr_thr_v + trace_at,
                          P.tr_trit_v + trace_at * P.c_bytes, x.r == 0);
    }
    __syncthreads();
    phase_mark(s.clk, 4);
    return 0;
}

// End of a component: the final quarters of u and v go to every CTA's pending slot L, with
// this CTA's message (u's count, u^T y, fallback).  Returns 1 if the cluster must stop;
// else the totals are in *s.tot (u's count is corrected for a fallback, whose trit is set
// in the slot).
__device__ __noinline__ int end_round(Ctx& x, const Smem2& s, int L) {
    cg::cluster_group cl = cg::this_cluster();
    const int c = x.c, Ls = x.Ls, tid = threadIdx.x;
    const unsigned hb = x.round & 1u;
    __syncthreads();
    if (tid == 0) x.round += 1u;
    const int Wqr = (int)((x.qr1 - x.qr0 + 31) >> 5), Wqc = (int)((x.qc1 - x.qc0 + 31) >> 5);
    const int64_t wr0 = x.qr0 >> 5, wc0 = x.qc0 >> 5;
    for (int t = tid; t < c * (Wqr + Wqc); t += NT) {
        const int peer = t / (Wqr + Wqc);
        const int k = t - peer * (Wqr + Wqc);
        if (k < Wqr) {
            cl.map_shared_rank(s.pnzU, peer)[(wr0 + k) * Ls + L] = s.nzU[k];
            cl.map_shared_rank(s.psgU, peer)[(wr0 + k) * Ls + L] = s.sgU[k];
        } else {
            const int kv = k - Wqr;
            cl.map_shared_rank(s.pnzV, peer)[(wc0 + kv) * Ls + L] = s.nzV[kv];
            cl.map_shared_rank(s.psgV, peer)[(wc0 + kv) * Ls + L] = s.sgV[kv];
        }
    }
    const int words = (int)(offsetof(Msg, ddot) / 4);   // the header (count, u^T y, fallback)
    for (int t = tid; t < words * c; t += NT) {
        const int peer = t / words, k = t - peer * words;
        reinterpret_cast<uint32_t*>(cl.map_shared_rank(s.msg + hb * c + x.r, peer))[k] =
            reinterpret_cast<const uint32_t*>(s.out)[k];
    }
    cl.sync();
    totals(s.msg, c, hb, s.tot);
    __syncthreads();
    if (s.tot->fail) return 1;
    if (s.tot->cnt == 0) {   // u fell back to one trit
        const int64_t fj = (s.tot->jx == LLONG_MAX) ? 0 : s.tot->jx;
        if (tid == 0) {
            s.pnzU[(fj >> 5) * Ls + L] |= 1u << (fj & 31);
            if (s.tot->xj < 0.0) s.psgU[(fj >> 5) * Ls + L] |= 1u << (fj & 31);
            s.tot->cnt = 1;
            s.tot->p = fabs(s.tot->xj);
            s.tot->pad = 1;   // marks the fallback
        }
    }
    __syncthreads();
    return 0;
}

// Fold the L pending terms into both blocks (hi + lo), then clear the per-output bits.
__device__ __noinline__ void fold2(const Prob& P, const Ctx& x, const Smem2& s, int L) {
    const int tid = threadIdx.x, c = x.c, Ls = x.Ls;
    const Grid2& g2 = P.g2;
    if (tid < c) {
        const Part pc = g2.pcol(tid);
        s.fbase[tid] = g2.qc().start(tid) + pc.start(x.q);
        s.fwidth[tid] = (int)(pc.end(x.q) - pc.start(x.q));
    }
    __syncthreads();
    stripe_bits(x.soffV, c, s.fbase, s.fwidth, s.pnzV, s.psgV, L, Ls, x.pitchV, s.bnz, s.bsg);
    __syncthreads();
    flush_dispatch(4, x.blkV, x.bloV, x.pitchV, x.qr1 - x.qr0, x.pitchV, L, Ls, s.pd, s.pnzU + (x.qr0 >> 5) * Ls,
                   s.psgU + (x.qr0 >> 5) * Ls, s.bnz, s.bsg, reinterpret_cast<uint32_t*>(s.red));
    __syncthreads();
    if (tid < c) {
        const Part pr = g2.prow(tid);
        s.fbase[tid] = g2.qr().start(tid) + pr.start(x.q);
        s.fwidth[tid] = (int)(pr.end(x.q) - pr.start(x.q));
    }
    __syncthreads();
    stripe_bits(x.soffU, c, s.fbase, s.fwidth, s.pnzU, s.psgU, L, Ls, x.pitchU, s.bnz, s.bsg);
    __syncthreads();
    flush_dispatch(4, x.blkU, x.bloU, x.pitchU, x.qc1 - x.qc0, x.pitchU, L, Ls, s.pd, s.pnzV + (x.qc0 >> 5) * Ls,
                   s.psgV + (x.qc0 >> 5) * Ls, s.bnz, s.bsg, reinterpret_cast<uint32_t*>(s.red));
    __syncthreads();
    for (int j = tid; j < x.wpv; j += NT) { s.cnzV[j] = 0u; s.csgV[j] = 0u; }
    for (int j = tid; j < x.wpu; j += NT) { s.cnzU[j] = 0u; s.csgU[j] = 0u; }
    __syncthreads();
}

// Factor one matrix with this cluster group.  Returns false if the group stopped.
template <bool WTD>
__device__ bool run_problem2(const Prob& P, int q, int r, const KCfg& cfg, const Smem2& s, GroupSync* gs) {
    const int tid = threadIdx.x;
    ctx_init(P, q, r, cfg, *s.x);
    Ctx& x = *s.x;
    const int Ls = x.Ls;
    const int64_t m = P.m, n = P.n;
    const int Wm = (int)((m + 31) >> 5), Wn = (int)((n + 31) >> 5);

    // every CTA reads the same flags, so the whole group takes the same early exit
    if (__ldcg(P.nonfinite) != 0u) {
        if (x.lead && tid == 0) atomicExch(P.status, ST_ENONFINITE);
        return true;
    }
    if (__ldcg(P.nonfinite + 1) != 0u) {
        if (x.lead && tid == 0) atomicExch(P.status, ST_EINVAL);
        return true;
    }
    {
        double ps = 0.0;
        for (int64_t t = tid; t < P.n_norm_part; t += NT) ps += __ldcg(P.norm_part + t);
        const double N0 = block_sum(ps, s.red);
        if (!(N0 > 0.0)) {
            if (x.lead && tid == 0) atomicExch(P.status, ST_EZERO);
            return true;
        }
        if (tid == 0) { x.N0 = N0; x.RN2 = N0; }
    }
    for (int j = tid; j < x.wpv; j += NT) { s.cnzV[j] = 0u; s.csgV[j] = 0u; }
    for (int j = tid; j < x.wpu; j += NT) { s.cnzU[j] = 0u; s.csgU[j] = 0u; }
    __syncthreads();
    int L = 0;
    // test hook: rank-1 terms supplied by the caller, held pending
    for (int j = 0; j < P.n_pend; ++j) {
        const uint32_t* ur = P.pend_u + j * (P.b_bytes / 4);
        const uint32_t* vr = P.pend_v + j * (P.c_bytes / 4);
        for (int w = tid; w < Wm + Wn; w += NT) {
            const bool isu = w < Wm;
            const int ww = isu ? w : w - Wm;
            const uint32_t* row = isu ? ur : vr;
            const uint32_t lo = __ldcg(row + 2 * ww), hi = __ldcg(row + 2 * ww + 1);
            const uint32_t z = compact_even(lo) | (compact_even(hi) << 16);
            const uint32_t sb = compact_even(lo >> 1) | (compact_even(hi >> 1) << 16);
            const int64_t rem = (isu ? m : n) - ((int64_t)ww << 5);
            const uint32_t msk = rem < 32 ? (1u << rem) - 1u : FULL;
            (isu ? s.pnzU : s.pnzV)[ww * Ls + L] = z & msk;
            (isu ? s.psgU : s.psgV)[ww * Ls + L] = sb & z & msk;
        }
        if (tid == 0) s.pd[L] = P.pend_d[j];
        __syncthreads();
        push_bits(s.pnzV, s.psgV, L, Ls, x.pv0, x.wpv, s.cnzV, s.csgV);
        push_bits(s.pnzU, s.psgU, L, Ls, x.pu0, x.wpu, s.cnzU, s.csgU);
        __syncthreads();
        ++L;
    }

    const int64_t kk = P.k;
    if (blockIdx.x == 0 && tid == 0) {
        for (int k2 = 0; k2 < 11; ++k2) s.clk[k2] = 0ull;
        s.clk[11] = (unsigned long long)clock64();
    }
    for (int64_t i = 0; i < kk; ++i) {
        const bool trv = P.tr_pre_v != nullptr && x.q == 0 && i >= P.tr_first && i - P.tr_first < P.tr_count;
        for (int j = tid; j < x.wpv; j += NT) s.gV[j] = 0.0;
        for (int j = tid; j < x.wpu; j += NT) s.gU[j] = 0.0;
        for (int l = tid; l < L; l += NT) { s.dotU[l] = 0; s.dotV[l] = 0; s.dotVw[l] = 0.0; }
        {
            const int Wqc = (int)((x.qc1 - x.qc0 + 31) >> 5);
            for (int w = tid; w < Wqc; w += NT) { s.nzV[w] = 0u; s.sgV[w] = 0u; }
        }
        start_quarter(P.start + (P.start_given ? 0 : i) * P.start_words, x.qr0, x.qr1, s.nzU, s.sgU, s.onzU, s.osgU,
                      s.ulist, x.pitchV, L, Ls, s.pnzU, s.psgU, s, s.out);
        phase_mark(s.clk, 7);
        for (int it = 0; it < P.iters; ++it) {
            const int64_t at = trv ? (i - P.tr_first) * P.iters + it : -1;
            if (half2<WTD, false>(P, x, cfg, s, gs, s.out->nch, L, at)) return false;
            if (half2<WTD, true>(P, x, cfg, s, gs, s.out->nch, L, at)) return false;
        }
        // s.scal[0] / [2]: nnz(v) and the weighted support sum of the last U-step's input
        const double nV = s.scal[0], hsv = s.scal[2];
        if (end_round(x, s, L)) return false;
        if (tid == 0) {
            const int nU = s.tot->cnt;
            const double p = s.tot->p;
            // ---- scale (§2.3 step 2), energy, safeguard (§7)
            const double d = (p == 0.0) ? 0.0 : p / ((double)nU * (WTD ? hsv : nV));
            x.sgh += (p * d < x.RN2 / ((double)m * (double)n)) ? 1ull : 0ull;
            x.RN2 -= p * d;
            x.sum_nunv += (unsigned long long)nU * (unsigned long long)nV;
            x.fb += (unsigned long long)s.tot->pad;
            s.pd[L] = d;
            if (x.lead) {
                P.D[i] = (float)d;
                if (P.energy) P.energy[i] = 1.0 - x.RN2 / x.N0;
                if (P.d64) P.d64[i] = d;
            }
        }
        // outputs: each CTA of cluster 0 packs its quarters of row i of B and C
        if (x.q == 0) {
            uint32_t* Bw = reinterpret_cast<uint32_t*>(P.B + i * P.b_bytes);
            uint32_t* Cw = reinterpret_cast<uint32_t*>(P.C + i * P.c_bytes);
            const int64_t bw0 = x.qr0 >> 4, bw1 = (x.r == x.c - 1) ? P.b_bytes / 4 : (x.qr1 >> 4);
            const int64_t cw0 = x.qc0 >> 4, cw1 = (x.r == x.c - 1) ? P.c_bytes / 4 : (x.qc1 >> 4);
            for (int64_t t = tid; t < (bw1 - bw0) + (cw1 - cw0); t += NT) {
                const bool isb = t < bw1 - bw0;
                const int64_t w = isb ? bw0 + t : cw0 + (t - (bw1 - bw0));
                const int64_t mw = w >> 1;
                uint32_t z = 0u, sg = 0u;
                if (mw < (isb ? Wm : Wn)) {
                    z = (isb ? s.pnzU : s.pnzV)[mw * Ls + L];
                    sg = (isb ? s.psgU : s.psgV)[mw * Ls + L];
                    if (w & 1) { z >>= 16; sg >>= 16; }
                }
                (isb ? Bw : Cw)[w] = spread_even(z) | (spread_even(sg & z) << 1);
            }
        }
        // ---- deflation (§2.3 step 3), held as pending term L
        push_bits(s.pnzV, s.psgV, L, Ls, x.pv0, x.wpv, s.cnzV, s.csgV);
        push_bits(s.pnzU, s.psgU, L, Ls, x.pu0, x.wpu, s.cnzU, s.csgU);
        __syncthreads();
        ++L;
        phase_mark(s.clk, 8);
        if (L + 1 > cfg.Lcap || i == kk - 1) {
            fold2(P, x, s, L);
            L = 0;
        }
        phase_mark(s.clk, 9);
    }

    // ---- explicit ||R_k||^2 from the folded residual hi + lo (the V-blocks cover R once)
    double rs = 0.0;
    {
        const Grid2& g2 = P.g2;
        const Part QC = g2.qc();
        const int64_t rows = x.qr1 - x.qr0;
        for (int sp = 0; sp < x.c; ++sp) {
            const Part pc = g2.pcol(sp);
            const int wdt = (int)(pc.end(x.q) - pc.start(x.q));
            const int64_t cb = QC.start(sp) + pc.start(x.q);
            const int64_t tot = rows * wdt;
            for (int64_t t = tid; t < tot; t += NT) {
                const int64_t rr = t / wdt;
                const int cc = (int)(t - rr * wdt);
                const int64_t e = rr * x.pitchV + x.soffV[sp] + cc;
                const double v = (double)__ldcg(x.blkV + e) + (double)__ldcg(x.bloV + e);
                rs += v * v * (WTD ? (double)__ldg(P.hw + cb + cc) : 1.0);
            }
        }
    }
    double R2 = 0.0;
    if (!exchange_sum(P.sums, x.qid, x.Gg, rs, s.red, gs, cfg.limit_ns, P.status, x.skip != 0, 1u, R2)) return false;
    if (x.lead && tid == 0) {
        P.stats->sum_nu = x.sum_nu;
        P.stats->sum_nv = x.sum_nv;
        P.stats->sum_du = x.sum_du;
        P.stats->sum_dv = x.sum_dv;
        P.stats->sum_nunv = x.sum_nunv;
        P.stats->half_steps = x.hs;
        P.stats->fallbacks = x.fb;
        P.stats->residual2 = R2;
        P.stats->norm_a2 = x.N0;
        P.stats->sweep_kept = 0ull;
        P.stats->safeguard = x.sgh;
        phase_mark(s.clk, 7);
        for (int k2 = 0; k2 < 11; ++k2) P.stats->phase[k2] = s.clk[k2];
        __threadfence();
        atomicExch(P.status, ST_OK);
    }
    __syncthreads();
    return true;
}

template <bool WTD>
__global__ void __launch_bounds__(NT, 1) als2_kernel(const __grid_constant__ KCfg cfg) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    cg::cluster_group cl = cg::this_cluster();
    const int c = (int)cl.num_blocks();
    const int grp = blockIdx.x / cfg.Gg;
    const int qid = blockIdx.x - grp * cfg.Gg;
    const int q = qid / c, r = qid - (qid / c) * c;   // (the cluster rank equals blockIdx.x % c)
    const int Lc = cfg.Lcap > 0 ? cfg.Lcap : 1;
    const SmemLayout2 lay(cfg.m_max, cfg.n_max, cfg.qr_max, cfg.qc_max, cfg.pv_max, cfg.pu_max, cfg.wpm, cfg.wpm, c, Lc,
                          cfg.weighted);
    // the pointer table lives in shared memory too (functions take it by reference)
    Smem2& s = *reinterpret_cast<Smem2*>(smem_raw + lay.sm);
    if (threadIdx.x == 0) {
#define EXTERND_SMEM2(f, T) s.f = reinterpret_cast<T*>(smem_raw + lay.f)
        EXTERND_SMEM2(red, double); EXTERND_SMEM2(part, double); EXTERND_SMEM2(xin, double); EXTERND_SMEM2(msg, Msg);
        EXTERND_SMEM2(out, Msg); EXTERND_SMEM2(pd, double); EXTERND_SMEM2(coef, double); EXTERND_SMEM2(coefV, double);
        EXTERND_SMEM2(dotU, int); EXTERND_SMEM2(dotV, int); EXTERND_SMEM2(dotVw, double); EXTERND_SMEM2(scal, double);
        EXTERND_SMEM2(wS, double); EXTERND_SMEM2(wP, double); EXTERND_SMEM2(wH, double); EXTERND_SMEM2(wM, double);
        EXTERND_SMEM2(wX, double); EXTERND_SMEM2(wJ, long long); EXTERND_SMEM2(wc, int); EXTERND_SMEM2(wd, int);
        EXTERND_SMEM2(dotp, int); EXTERND_SMEM2(dotpw, double); EXTERND_SMEM2(clk, unsigned long long);
        EXTERND_SMEM2(nzU, uint32_t); EXTERND_SMEM2(sgU, uint32_t); EXTERND_SMEM2(onzU, uint32_t); EXTERND_SMEM2(osgU, uint32_t);
        EXTERND_SMEM2(nzV, uint32_t); EXTERND_SMEM2(sgV, uint32_t); EXTERND_SMEM2(onzV, uint32_t); EXTERND_SMEM2(osgV, uint32_t);
        EXTERND_SMEM2(pnzU, uint32_t); EXTERND_SMEM2(psgU, uint32_t); EXTERND_SMEM2(pnzV, uint32_t); EXTERND_SMEM2(psgV, uint32_t);
        EXTERND_SMEM2(cnzV, uint32_t); EXTERND_SMEM2(csgV, uint32_t); EXTERND_SMEM2(cnzU, uint32_t); EXTERND_SMEM2(csgU, uint32_t);
        EXTERND_SMEM2(bnz, uint32_t); EXTERND_SMEM2(bsg, uint32_t); EXTERND_SMEM2(ulist, int); EXTERND_SMEM2(vlist, int);
        EXTERND_SMEM2(vwl, float); EXTERND_SMEM2(gV, double); EXTERND_SMEM2(gU, double); EXTERND_SMEM2(corr, double);
        EXTERND_SMEM2(fbase, long long); EXTERND_SMEM2(fwidth, int); EXTERND_SMEM2(x, Ctx); EXTERND_SMEM2(xq, double);
        EXTERND_SMEM2(tot, Tot); EXTERND_SMEM2(stop, int); EXTERND_SMEM2(sS, double);
#undef EXTERND_SMEM2
    }
    __syncthreads();

    GroupSync* gs = cfg.gsync + grp;
    if (threadIdx.x == 0) { s.x->arrivals = 0u; s.x->round = 0u; }
    __syncthreads();
    for (int pi = grp; pi < cfg.nprob; pi += cfg.NG) {
        const bool ok = run_problem2<WTD>(cfg.probs[pi], q, r, cfg, s, gs);
        // the cluster agrees before the next problem: a CTA whose last wait gave up (or a group
        // that aborted) stops all of them at the same barrier; the abort word is read once
        if (threadIdx.x == 0) s.stop[16] = (!ok || ld_relaxed_s32(&gs->abort)) ? 1 : 0;
        __syncthreads();
        if (threadIdx.x < (unsigned)c) cl.map_shared_rank(s.stop, threadIdx.x)[r] = s.stop[16];
        cl.sync();
        int any = 0;
        for (int k = 0; k < c; ++k) any |= s.stop[k];
        cl.sync();   // the flags are rewritten only after everyone read them
        if (any) break;
    }
    // no CTA leaves while a peer may still write into its shared memory
    cl.sync();
}

}  // namespace externd
