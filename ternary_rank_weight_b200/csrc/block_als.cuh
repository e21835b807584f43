// Batched block ALS with decorrelated targets ("ExTernD: Expanded-Rank Ternary
// Decomposition", §2.4 "Batched block ALS"): components are extracted b at a time,
//   V <- T_tau([(U^T U + eps I)^-1 U^T R]^T),   U <- T_tau(R V (V^T V + eps I)^-1)   (column-wise),
// `iters` times from the start vectors of the block's components, then the scales solve
// [(U^T U) o (V^T V)] d = diag(U^T R V) jointly and R <- R - U diag(d) V^T.  Deflation across
// blocks is sequential.  Reading of the unspecified ridge: eps = 1e-6 x the mean diagonal of
// the Gram matrix it regularizes.
//
// B200 design: the block method is dense linear algebra on the fp64 residual (m x n, kept
// in fp64 so that its deflation by whole blocks does not round).  Each block is a short
// sequence of launches on one stream: the plain fp64 GEMMs (U^T U, R^T U, V^T V, R V and the
// deflation) and the Cholesky factorizations and solves of the b x b systems go to the
// vendor libraries (cuBLAS DGEMM, cuSOLVER POTRF/POTRS); the method's own steps run in the
// kernels below: start trits, the ridge, the column-wise T_tau, the joint scale system, the
// energy, and the packing of the trits.  U and V are held as fp64 +-1/0 matrices.

namespace externd {

constexpr double BLOCK_EPS_REL = 1e-6;   // the ridge: eps = this x the Gram matrix's mean diagonal
__global__ void block_setup_kernel(const float* __restrict__ A, int64_t total, double* __restrict__ R,
                                   unsigned* nonfinite) {
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
        const float v = A[t];
        if (!isfinite(v)) atomicAdd(nonfinite, 1u);
        R[t] = (double)v;
    }
}

// Partial sums of R^2, one per CTA (fixed order; sum_partials_kernel adds them in order).
__global__ void __launch_bounds__(1024) sumsq_kernel(const double* __restrict__ R, int64_t total, double* partial) {
    __shared__ double sh[33];
    double s = 0.0;
    for (int64_t t = (int64_t)blockIdx.x * 1024 + threadIdx.x; t < total; t += (int64_t)gridDim.x * 1024) s += R[t] * R[t];
    #pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
    if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
        double w = sh[threadIdx.x];
        #pragma unroll
        for (int o = 16; o; o >>= 1) w += __shfl_xor_sync(FULL, w, o);
        if (threadIdx.x == 0) partial[blockIdx.x] = w;
    }
}

__global__ void __launch_bounds__(1024) sum_partials_kernel(const double* partial, int np, double* out) {
    __shared__ double sh[33];
    double s = 0.0;
    for (int t = threadIdx.x; t < np; t += 1024) s += partial[t];
    #pragma unroll
    for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
    if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
        double w = sh[threadIdx.x];
        #pragma unroll
        for (int o = 16; o; o >>= 1) w += __shfl_xor_sync(FULL, w, o);
        if (threadIdx.x == 0) *out = w;
    }
}

// T_tau of one column of a matrix (CTA j: column j of an len x ld row-major matrix X), written
// as +-1 / 0 into column j of O (len x ldo, fp64).  §2.2 with the all-zero fallback (lowest
// index among the largest magnitudes).
__global__ void __launch_bounds__(256) ternarize_cols_kernel(const double* __restrict__ X, int64_t len, int ld,
                                                            double tau, double* __restrict__ O, int ldo) {
    __shared__ double shs[9], shm[9];
    __shared__ long long shj[9];
    const int j = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    double s = 0.0, mx = -1.0;
    long long jx = LLONG_MAX;
    for (int64_t i = threadIdx.x; i < len; i += 256) {
        const double v = X[i * ld + j];
        const double a = fabs(v);
        s += a;
        if (a > mx) { mx = a; jx = i; }
    }
    #pragma unroll
    for (int o = 16; o; o >>= 1) {
        s += __shfl_xor_sync(FULL, s, o);
        const double m2 = __shfl_xor_sync(FULL, mx, o);
        const long long j2 = __shfl_xor_sync(FULL, jx, o);
        maxloc_merge(mx, jx, m2, j2);
    }
    if (lane == 0) { shs[warp] = s; shm[warp] = mx; shj[warp] = jx; }
    __syncthreads();
    if (threadIdx.x == 0) {
        double S = 0.0, M = -1.0;
        long long J = LLONG_MAX;
        for (int w = 0; w < 8; ++w) { S += shs[w]; maxloc_merge(M, J, shm[w], shj[w]); }
        shs[8] = S;
        shj[8] = J;
    }
    __syncthreads();
    const double thr = tau * shs[8] / (double)len;
    int any = 0;
    for (int64_t i = threadIdx.x; i < len; i += 256) {
        const double v = X[i * ld + j];
        const double t = fabs(v) > thr ? (v < 0.0 ? -1.0 : 1.0) : 0.0;
        any |= (t != 0.0);
        O[i * ldo + j] = t;
    }
    any = __syncthreads_or(any);
    if (!any && threadIdx.x == 0) {
        const long long J = (shj[8] >= 0 && shj[8] < len) ? shj[8] : 0;
        const double v = X[J * ld + j];
        O[J * ldo + j] = v < 0.0 ? -1.0 : 1.0;
    }
}

// Lm = G + eps I, eps = eps_rel x mean diagonal of G (b x b, one CTA).
__global__ void __launch_bounds__(1024) ridge_kernel(const double* __restrict__ G, int b, double eps_rel,
                                                     double* __restrict__ Lm) {
    __shared__ double part[32];
    double tr = 0.0;
    for (int i = threadIdx.x; i < b; i += blockDim.x) tr += G[(int64_t)i * b + i];
    #pragma unroll
    for (int o = 16; o; o >>= 1) tr += __shfl_xor_sync(FULL, tr, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = tr;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += part[w];   // fixed order
        part[0] = eps_rel * t / (double)b;
    }
    __syncthreads();
    const double eps = part[0];
    for (int64_t t = threadIdx.x; t < (int64_t)b * b; t += blockDim.x)
        Lm[t] = G[t] + ((t / b == t % b) ? eps : 0.0);
}

// Any nonzero status among n (the factorization info words) -> *flag = 1.
__global__ void info_any_kernel(const int* __restrict__ info, int n, int* flag) {
    int bad = 0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) bad |= (info[i] != 0);
    if (__syncthreads_or(bad) && threadIdx.x == 0) *flag = 1;
}

// Start vectors of components s0 .. s0 + nb - 1 as fp64 columns of U (m x ldu): T_tau of the
// Philox normals (the sequential method's start vectors).
__global__ void __launch_bounds__(256) block_start_kernel(uint64_t seed, int64_t s0, int64_t m, double tau, double* U,
                                                         int ldu) {
    __shared__ double shs[9], shm[9];
    __shared__ long long shj[9];
    const int j = blockIdx.x;
    const uint32_t comp = (uint32_t)(s0 + j);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    double s = 0.0, mx = -1.0;
    long long jx = LLONG_MAX;
    for (int64_t r = threadIdx.x; r < m; r += 256) {
        const double a = fabs(start_normal(seed, comp, (uint32_t)r));
        s += a;
        if (a > mx) { mx = a; jx = r; }
    }
    #pragma unroll
    for (int o = 16; o; o >>= 1) {
        s += __shfl_xor_sync(FULL, s, o);
        const double m2 = __shfl_xor_sync(FULL, mx, o);
        const long long j2 = __shfl_xor_sync(FULL, jx, o);
        maxloc_merge(mx, jx, m2, j2);
    }
    if (lane == 0) { shs[warp] = s; shm[warp] = mx; shj[warp] = jx; }
    __syncthreads();
    if (threadIdx.x == 0) {
        double S = 0.0, M = -1.0;
        long long J = LLONG_MAX;
        for (int w = 0; w < 8; ++w) { S += shs[w]; maxloc_merge(M, J, shm[w], shj[w]); }
        shs[8] = S;
        shj[8] = J;
    }
    __syncthreads();
    const double thr = tau * shs[8] / (double)m;
    int any = 0;
    for (int64_t r = threadIdx.x; r < m; r += 256) {
        const double z = start_normal(seed, comp, (uint32_t)r);
        const double t = fabs(z) > thr ? (z < 0.0 ? -1.0 : 1.0) : 0.0;
        any |= (t != 0.0);
        U[r * ldu + j] = t;
    }
    any = __syncthreads_or(any);
    if (!any && threadIdx.x == 0) {
        const long long J = shj[8];
        U[J * ldu + j] = start_normal(seed, comp, (uint32_t)J) < 0.0 ? -1.0 : 1.0;
    }
}

// H = (Gu o Gv) and rhs_j = sum_r U_rj Q_rj (U^T R V's diagonal, Q = R V); b x b, fp64.
__global__ void block_scale_system_kernel(const double* Gu, const double* Gv, int b, const double* U, const double* Q,
                                          int64_t m, double* H, double* rhs) {
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < b * b; t += gridDim.x * blockDim.x) H[t] = Gu[t] * Gv[t];
    for (int j = blockIdx.x; j < b; j += gridDim.x) {
        __shared__ double sh[33];
        double s = 0.0;
        for (int64_t r = threadIdx.x; r < m; r += blockDim.x) s += U[r * b + j] * Q[r * b + j];
        #pragma unroll
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(FULL, s, o);
        if ((threadIdx.x & 31) == 0) sh[threadIdx.x >> 5] = s;
        __syncthreads();
        if (threadIdx.x == 0) {
            double w = 0.0;
            for (int k = 0; k < (int)(blockDim.x >> 5); ++k) w += sh[k];
            rhs[j] = w;
        }
        __syncthreads();
    }
}

// W = U diag(d) (m x b), to deflate with one GEMM: R <- R - W V^T.
__global__ void scale_cols_kernel(const double* U, int64_t m, int b, const double* d, double* W) {
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < m * b; t += (int64_t)gridDim.x * blockDim.x)
        W[t] = U[t] * d[t % b];
}

// Pack the block's columns into trit rows (row s0 + j of the output = column j of X, len x b),
// scales into D, energy into E.
__global__ void block_pack_kernel(const double* X, int64_t len, int b, int nb, int64_t s0, uint8_t* out, int64_t row_bytes) {
    const int j = blockIdx.x;
    if (j >= nb) return;
    uint32_t* row = reinterpret_cast<uint32_t*>(out + (s0 + j) * row_bytes);
    for (int64_t w = threadIdx.x; w < row_bytes / 4; w += blockDim.x) {
        uint32_t word = 0;
        for (int e = 0; e < 16; ++e) {
            const int64_t i = w * 16 + e;
            if (i < len) {
                const double v = X[i * b + j];
                if (v != 0.0) word |= (v < 0.0 ? 3u : 1u) << (2 * e);
            }
        }
        row[w] = word;
    }
}

__global__ void block_out_kernel(const double* d, int nb, int64_t s0, const double* r2, const double* n0, float* D,
                                 double* d64, double* E) {
    for (int j = threadIdx.x; j < nb; j += blockDim.x) {
        D[s0 + j] = (float)d[j];
        if (d64) d64[s0 + j] = d[j];
        if (E) E[s0 + j] = 1.0 - *r2 / *n0;
    }
}

}  // namespace externd
