// Inference with ExTernD factors and their mask+sign storage (sm_100a).
//
// "ExTernD: Expanded-Rank Ternary Decomposition" (arXiv 2607.13511), §2.6 Cost
// model: inference computes y = B (diag(D) (C x)) with k (m + n) ternary
// add/subtracts and k multiplies; mask+sign packing stores one zero/nonzero bit
// per element and one sign bit per nonzero, Eq. (1).
//
// Layout for inference: C is used as the factorization returns it (row i =
// row i of C, 2-bit trits); B is transposed once (externd_transpose_trits) so
// that output r's trits B[r, 0..k) are contiguous.  Both products are then row
// dots of 2-bit trit rows with a dense fp32 vector:
//     z_i = D_i * sum_j C[i, j] x_j        (k rows of n trits)
//     y_r = sum_i B[r, i] z_i              (m rows of k trits)
// One warp per row; each lane takes 16-byte chunks of the row (64 trits),
// turns each 32-bit word into nonzero/negative masks and adds the selected
// entries of the vector (which stays in L1: a few tens of KB).
#include <cuda_runtime.h>

#include <cstdint>
#include <vector>

#include "externd.h"

namespace externd_infer {

constexpr unsigned FULL = 0xffffffffu;
constexpr int MAXB = 8;          // vectors per call handled in registers
constexpr int RD_THREADS = 256;  // row-dot block: 8 warps

__device__ __forceinline__ uint32_t even_bits(uint32_t x) {   // bits 0,2,...,30 -> 0..15
    x &= 0x55555555u;
    x = (x | (x >> 1)) & 0x33333333u;
    x = (x | (x >> 2)) & 0x0F0F0F0Fu;
    x = (x | (x >> 4)) & 0x00FF00FFu;
    x = (x | (x >> 8)) & 0x0000FFFFu;
    return x;
}

size_t trit_bytes(int64_t len) { return len < 1 ? 0 : (size_t)(((len + 3) / 4 + 15) / 16 * 16); }

// out[b * rows + r] = scale_r * sum_j T[r, j] V[b * len + j]   (scale_r = 1 without scale)
template <int NB>
__global__ void __launch_bounds__(RD_THREADS) rowdot_kernel(const uint8_t* __restrict__ T, int64_t rows, int64_t len,
                                                          int64_t tb, const float* __restrict__ V, int64_t vstride,
                                                          const float* __restrict__ scale, float* __restrict__ out,
                                                          int64_t ostride) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (RD_THREADS / 32);
    const int64_t nchunk = tb / 16;
    for (int64_t r = (int64_t)blockIdx.x * (RD_THREADS / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
        const uint4* row = reinterpret_cast<const uint4*>(T + r * tb);
        float acc[NB];
        #pragma unroll
        for (int b = 0; b < NB; ++b) acc[b] = 0.f;
        for (int64_t c = lane; c < nchunk; c += 32) {
            const uint4 q = __ldg(row + c);
            const uint32_t w4[4] = {q.x, q.y, q.z, q.w};
            #pragma unroll
            for (int h = 0; h < 4; ++h) {
                // positions j0 .. j0+15; padding trits beyond len are zero codes
                const int64_t j0 = c * 64 + 16 * h;
                uint32_t nz = even_bits(w4[h]);
                const uint32_t ng = even_bits(w4[h] >> 1);
                while (nz) {
                    const int t = __ffs(nz) - 1;
                    nz &= nz - 1u;
                    const bool neg = (ng >> t) & 1u;
                    #pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        const float v = __ldg(V + b * vstride + j0 + t);
                        acc[b] += neg ? -v : v;
                    }
                }
            }
        }
        #pragma unroll
        for (int b = 0; b < NB; ++b) {
            float a = acc[b];
            #pragma unroll
            for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(FULL, a, o);
            acc[b] = a;
        }
        if (lane == 0) {
            const float sc = scale ? __ldg(scale + r) : 1.f;
            #pragma unroll
            for (int b = 0; b < NB; ++b) out[b * ostride + r] = sc * acc[b];
        }
    }
}

// Tt[j, r] = T[r, j]: rows x len 2-bit trits -> len x rows.  A block transposes a
// 64 (rows) x 64 (trits) tile through shared memory.
__global__ void __launch_bounds__(256) transpose_trits_kernel(const uint8_t* __restrict__ T, int64_t rows, int64_t len,
                                                              int64_t tb, uint8_t* __restrict__ Tt, int64_t ttb) {
    __shared__ uint8_t tile[64][65];
    const int64_t r0 = (int64_t)blockIdx.y * 64, j0 = (int64_t)blockIdx.x * 64;
    for (int e = threadIdx.x; e < 64 * 16; e += 256) {      // 64 rows x 16 bytes (64 trits)
        const int rr = e >> 4, bb = e & 15;
        const int64_t r = r0 + rr;
        const uint8_t byte = (r < rows && j0 / 4 + bb < tb) ? T[r * tb + j0 / 4 + bb] : 0;
        #pragma unroll
        for (int t = 0; t < 4; ++t) tile[rr][bb * 4 + t] = (byte >> (2 * t)) & 3;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < 64 * 16; e += 256) {      // 64 trit-columns x 16 bytes of rows
        const int jj = e >> 4, bb = e & 15;
        const int64_t j = j0 + jj;
        if (j >= len || r0 / 4 + bb >= ttb) continue;
        uint8_t byte = 0;
        #pragma unroll
        for (int t = 0; t < 4; ++t) byte |= (uint8_t)(tile[bb * 4 + t][jj] << (2 * t));
        Tt[j * ttb + r0 / 4 + bb] = byte;
    }
}

// nonzero count of each row
__global__ void __launch_bounds__(256) row_nnz_kernel(const uint8_t* __restrict__ T, int64_t rows, int64_t tb,
                                                      int64_t* __restrict__ nnz) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * 8;
    for (int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); r < rows; r += warps) {
        const uint32_t* row = reinterpret_cast<const uint32_t*>(T + r * tb);
        long long c = 0;
        for (int64_t w = lane; w < tb / 4; w += 32) c += __popc(even_bits(__ldg(row + w)));
        #pragma unroll
        for (int o = 16; o; o >>= 1) c += __shfl_xor_sync(FULL, c, o);
        if (lane == 0) nnz[r] = c;
    }
}

// exclusive prefix sum of n int64 values by one block (n up to a few million)
__global__ void __launch_bounds__(1024) exclusive_scan_kernel(const int64_t* __restrict__ in, int64_t n,
                                                              int64_t* __restrict__ out) {
    __shared__ long long part[1024];
    const int64_t per = (n + 1023) / 1024;
    const int64_t b = threadIdx.x * per, e = b + per < n ? b + per : n;
    long long s = 0;
    for (int64_t i = b; i < e; ++i) s += in[i];
    part[threadIdx.x] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        long long run = 0;
        for (int t = 0; t < 1024; ++t) { const long long v = part[t]; part[t] = run; run += v; }
        out[n] = run;
    }
    __syncthreads();
    long long run = part[threadIdx.x];
    for (int64_t i = b; i < e; ++i) { out[i] = run; run += in[i]; }
}

// mask bytes of each row, and its sign bits appended to one bit stream at off[r]
__global__ void __launch_bounds__(256) mask_sign_kernel(const uint8_t* __restrict__ T, int64_t rows, int64_t len,
                                                        int64_t tb, const int64_t* __restrict__ off,
                                                        uint8_t* __restrict__ mask, int64_t mb,
                                                        uint32_t* __restrict__ signs) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * 8;
    const int64_t groups = (len + 31) / 32;                 // 32 trits = 8 bytes of T
    for (int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); r < rows; r += warps) {
        const uint8_t* row = T + r * tb;
        int64_t base = off[r];
        for (int64_t g0 = 0; g0 < groups; g0 += 32) {
            const int64_t g = g0 + lane;
            uint32_t nz = 0u, ng = 0u;
            if (g < groups) {
                const uint32_t lo = *reinterpret_cast<const uint32_t*>(row + 8 * g);
                const uint32_t hi = (8 * g + 4 < tb) ? *reinterpret_cast<const uint32_t*>(row + 8 * g + 4) : 0u;
                nz = even_bits(lo) | (even_bits(hi) << 16);
                ng = (even_bits(lo >> 1) | (even_bits(hi >> 1) << 16)) & nz;
                for (int t = 0; t < 4; ++t) {
                    const int64_t byte = 4 * g + t;
                    if (byte < mb) mask[r * mb + byte] = (uint8_t)(nz >> (8 * t));
                }
            }
            // signs of the nonzeros of this group, in order
            uint32_t packed = 0u;
            int cnt = 0;
            for (uint32_t m = nz; m; m &= m - 1u) {
                const int t = __ffs(m) - 1;
                packed |= ((ng >> t) & 1u) << cnt;
                ++cnt;
            }
            int incl = cnt;
            #pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(FULL, incl, o);
                if (lane >= o) incl += v;
            }
            if (packed) {
                const int64_t bit = base + incl - cnt;
                const int64_t w = bit >> 5;
                const int sh = (int)(bit & 31);
                atomicOr(signs + w, packed << sh);
                if (sh && cnt > 32 - sh) atomicOr(signs + w + 1, packed >> (32 - sh));
            }
            base += __shfl_sync(FULL, incl, 31);
        }
    }
}

bool is_device(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) { cudaGetLastError(); return false; }
    return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

int sms() {
    int dev = 0, v = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    cudaGetLastError();
    return v;
}

template <int NB>
void launch_rowdot(const uint8_t* T, int64_t rows, int64_t len, int64_t tb, const float* V, int64_t vstride,
                   const float* scale, float* out, int64_t ostride, cudaStream_t s) {
    const int64_t want = (rows + 7) / 8;
    const int64_t cap = (int64_t)sms() * 8;
    const unsigned grid = (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
    rowdot_kernel<NB><<<grid, RD_THREADS, 0, s>>>(T, rows, len, tb, V, vstride, scale, out, ostride);
}

void rowdot(int nb, const uint8_t* T, int64_t rows, int64_t len, int64_t tb, const float* V, int64_t vstride,
            const float* scale, float* out, int64_t ostride, cudaStream_t s) {
    switch (nb) {
        case 1: launch_rowdot<1>(T, rows, len, tb, V, vstride, scale, out, ostride, s); break;
        case 2: launch_rowdot<2>(T, rows, len, tb, V, vstride, scale, out, ostride, s); break;
        case 3: launch_rowdot<3>(T, rows, len, tb, V, vstride, scale, out, ostride, s); break;
        case 4: launch_rowdot<4>(T, rows, len, tb, V, vstride, scale, out, ostride, s); break;
        default: launch_rowdot<MAXB>(T, rows, len, tb, V, vstride, scale, out, ostride, s); break;
    }
}

}  // namespace externd_infer

using namespace externd_infer;

extern "C" {

int externd_transpose_trits(const uint8_t* T, int64_t rows, int64_t len, uint8_t* Tt_out, void* stream) {
    if (!T || !Tt_out || rows < 1 || len < 1) return EXTERND_EINVAL;
    if (!is_device(T) || !is_device(Tt_out)) return EXTERND_EINVAL;
    if ((len + 63) / 64 > 0x7fffffff || (rows + 63) / 64 > 65535) return EXTERND_ELIMIT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t tb = (int64_t)trit_bytes(len), ttb = (int64_t)trit_bytes(rows);
    if (cudaMemsetAsync(Tt_out, 0, (size_t)(len * ttb), s) != cudaSuccess) { cudaGetLastError(); return EXTERND_ECUDA; }
    transpose_trits_kernel<<<dim3((unsigned)((len + 63) / 64), (unsigned)((rows + 63) / 64)), 256, 0, s>>>(T, rows, len, tb,
                                                                                                         Tt_out, ttb);
    if (cudaGetLastError() != cudaSuccess) return EXTERND_ECUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) { cudaGetLastError(); return EXTERND_ECUDA; }
    return EXTERND_OK;
}

int externd_matvec(const uint8_t* Bt, const float* D, const uint8_t* C, int64_t m, int64_t n, int64_t k,
                   const float* X, int64_t batch, float* Y, float* z_work, void* stream) {
    if (!Bt || !D || !C || !X || !Y || !z_work || m < 1 || n < 1 || k < 1 || batch < 1) return EXTERND_EINVAL;
    if (!is_device(Bt) || !is_device(D) || !is_device(C) || !is_device(X) || !is_device(Y) || !is_device(z_work))
        return EXTERND_EINVAL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t cb = (int64_t)trit_bytes(n), bb = (int64_t)trit_bytes(k);
    for (int64_t b0 = 0; b0 < batch; b0 += MAXB) {
        const int nb = (int)(batch - b0 < MAXB ? batch - b0 : MAXB);
        // z = diag(D) (C x): k rows of n trits
        rowdot(nb, C, k, n, cb, X + b0 * n, n, D, z_work, k, s);
        // y = B z: m rows of k trits (B transposed)
        rowdot(nb, Bt, m, k, bb, z_work, k, nullptr, Y + b0 * m, m, s);
    }
    if (cudaGetLastError() != cudaSuccess) return EXTERND_ECUDA;
    return EXTERND_OK;
}

int externd_pack_mask_sign(const uint8_t* T, int64_t rows, int64_t len, uint8_t* mask_out, uint32_t* sign_out,
                           int64_t sign_words, int64_t* sign_offsets_out, void* stream) {
    if (!T || !mask_out || !sign_out || !sign_offsets_out || rows < 1 || len < 1 || sign_words < 1)
        return EXTERND_EINVAL;
    if (!is_device(T) || !is_device(mask_out) || !is_device(sign_out) || !is_device(sign_offsets_out))
        return EXTERND_EINVAL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t tb = (int64_t)trit_bytes(len), mb = (len + 7) / 8;
    int64_t* nnz = nullptr;
    int rc = EXTERND_OK;
    int64_t total = 0;
    const unsigned grid = (unsigned)((rows + 7) / 8 < (int64_t)sms() * 8 ? (rows + 7) / 8 : (int64_t)sms() * 8);
    if (cudaMallocAsync((void**)&nnz, sizeof(int64_t) * (size_t)rows, s) != cudaSuccess) { cudaGetLastError(); return EXTERND_ENOMEM; }
    row_nnz_kernel<<<grid, 256, 0, s>>>(T, rows, tb, nnz);
    exclusive_scan_kernel<<<1, 1024, 0, s>>>(nnz, rows, sign_offsets_out);
    if (cudaGetLastError() != cudaSuccess) { rc = EXTERND_ECUDA; goto done; }
    if (cudaMemcpyAsync(&total, sign_offsets_out + rows, sizeof(int64_t), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess) { cudaGetLastError(); rc = EXTERND_ECUDA; goto done; }
    if ((total + 31) / 32 > sign_words) { rc = EXTERND_ELIMIT; goto done; }
    if (cudaMemsetAsync(sign_out, 0, sizeof(uint32_t) * (size_t)sign_words, s) != cudaSuccess) { cudaGetLastError(); rc = EXTERND_ECUDA; goto done; }
    mask_sign_kernel<<<grid, 256, 0, s>>>(T, rows, len, tb, sign_offsets_out, mask_out, mb, sign_out);
    if (cudaGetLastError() != cudaSuccess) { rc = EXTERND_ECUDA; goto done; }
    if (cudaStreamSynchronize(s) != cudaSuccess) { cudaGetLastError(); rc = EXTERND_ECUDA; goto done; }
done:
    cudaFreeAsync(nnz, s);
    cudaStreamSynchronize(s);
    cudaGetLastError();
    return rc;
}

}  // extern "C"
