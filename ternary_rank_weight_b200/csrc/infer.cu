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
// One warp per row.  When the vectors fit in shared memory (NB * len * 4 bytes
// up to ~200 KB) they are staged there and every trit is one fused multiply-add
// with its code read as a signed 2-bit integer (rowdot_smem_kernel); otherwise each lane walks
// the nonzero trits of its 16-byte chunks and reads the vector through L1
// (rowdot_kernel).
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

// Shared-memory variant: the NB vectors (NB * len fp32) are staged in shared
// memory.  Each nibble of a trit row (two trits) indexes a 16-entry table of
// coefficient pairs in {-1, 0, 1} (a 2-bit code read as a signed 2-bit integer is
// the trit); the table is exactly 128 bytes, so lanes that read the same entry
// share one access and different entries sit in different banks.  Each trit is
// then one fused multiply-add per vector, with no divergence.  A warp
// takes R rows at once: lane l reads the 32-bit words l, l + 32, ... of each (16
// trits per word, up to G words per row issued before any is used), and every
// vector value it loads from shared memory serves the R rows.  The staged vector
// is swizzled: the four 16-byte groups of word w are rotated by (w / 2) % 4, so
// the eight lanes of a quarter-warp (eight consecutive words) read distinct banks.
constexpr int RS_THREADS = 128;   // shared-memory row-dot block: 4 warps; several blocks per SM

__device__ __forceinline__ int64_t swz(int64_t j) {    // position of vector entry j in shared memory
    const int64_t w = j >> 4;
    const int h = (int)((j >> 2) & 3);
    return 16 * w + 4 * ((h + (int)(w >> 1)) & 3) + (j & 3);
}

template <int NB, int R>
__global__ void __launch_bounds__(RS_THREADS) rowdot_smem_kernel(const uint8_t* __restrict__ T, int64_t rows,
                                                               int64_t len, int64_t tb, const float* __restrict__ V,
                                                               int64_t vstride, const float* __restrict__ scale,
                                                               float* __restrict__ out, int64_t ostride) {
    extern __shared__ __align__(128) float smem_rd[];
    float2* lut2 = reinterpret_cast<float2*>(smem_rd);     // 16 entries, 128 bytes: a nibble -> 2 trits
    float* sv = smem_rd + 32;                               // NB x lenp, lenp = 16 * words, swizzled
    const int64_t words = tb / 4;
    const int64_t lenp = words * 16;
    if (threadIdx.x < 16) {
        const int v = threadIdx.x;
        lut2[v] = make_float2((float)((v << 30) >> 30), (float)(((v >> 2) << 30) >> 30));
    }
    const bool vec4 = ((len & 3) == 0) && ((vstride & 3) == 0) && ((reinterpret_cast<uintptr_t>(V) & 15) == 0);
    for (int b = 0; b < NB; ++b) {
        if (vec4) {   // 16-byte groups copied asynchronously (all in flight at once); the swizzle moves whole groups
            const float4* V4 = reinterpret_cast<const float4*>(V + b * vstride);
            for (int64_t g = threadIdx.x; g < lenp / 4; g += RS_THREADS) {
                float* dst = sv + b * lenp + swz(4 * g);
                if (4 * g < len) {
                    const unsigned saddr = (unsigned)__cvta_generic_to_shared(dst);
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(V4 + g) : "memory");
                } else {
                    *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        } else {
            for (int64_t j = threadIdx.x; j < lenp; j += RS_THREADS)
                sv[b * lenp + swz(j)] = j < len ? __ldg(V + b * vstride + j) : 0.f;
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t groups = (rows + R - 1) / R;
    const int64_t warps = (int64_t)gridDim.x * (RS_THREADS / 32);
    constexpr int G = (R >= 4) ? 4 : 8;                     // words per row and lane issued together
    for (int64_t grp = (int64_t)blockIdx.x * (RS_THREADS / 32) + (threadIdx.x >> 5); grp < groups; grp += warps) {
        const int64_t r0 = grp * R;
        float acc[R][NB];
        #pragma unroll
        for (int rr = 0; rr < R; ++rr)
            #pragma unroll
            for (int b = 0; b < NB; ++b) acc[rr][b] = 0.f;
        for (int64_t w0 = 0; w0 < words; w0 += 32 * G) {
            uint32_t q[R][G];
            #pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                const uint32_t* row = reinterpret_cast<const uint32_t*>(T + (r0 + rr) * tb);
                #pragma unroll
                for (int g = 0; g < G; ++g) {
                    const int64_t w = w0 + lane + 32 * g;
                    q[rr][g] = (r0 + rr < rows && w < words) ? __ldg(row + w) : 0u;
                }
            }
            #pragma unroll
            for (int g = 0; g < G; ++g) {
                const int64_t w = w0 + lane + 32 * g;
                if (w >= words) break;
                const int rot = (int)(w >> 1);
                #pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int64_t at = 16 * w + 4 * ((h + rot) & 3);
                    float x[NB][4];
                    #pragma unroll
                    for (int b = 0; b < NB; ++b) {
                        const float4 t4 = *reinterpret_cast<const float4*>(sv + b * lenp + at);
                        x[b][0] = t4.x; x[b][1] = t4.y; x[b][2] = t4.z; x[b][3] = t4.w;
                    }
                    #pragma unroll
                    for (int rr = 0; rr < R; ++rr) {
                        const uint32_t byte = (q[rr][g] >> (8 * h)) & 0xFFu;   // trits 4h .. 4h+3
                        const float2 c01 = lut2[byte & 15u];
                        const float2 c23 = lut2[byte >> 4];
                        #pragma unroll
                        for (int b = 0; b < NB; ++b) {
                            acc[rr][b] = fmaf(c01.x, x[b][0], acc[rr][b]);
                            acc[rr][b] = fmaf(c01.y, x[b][1], acc[rr][b]);
                            acc[rr][b] = fmaf(c23.x, x[b][2], acc[rr][b]);
                            acc[rr][b] = fmaf(c23.y, x[b][3], acc[rr][b]);
                        }
                    }
                }
            }
        }
        #pragma unroll
        for (int rr = 0; rr < R; ++rr)
            #pragma unroll
            for (int b = 0; b < NB; ++b) {
                float a = acc[rr][b];
                #pragma unroll
                for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(FULL, a, o);
                acc[rr][b] = a;
            }
        if (lane == 0) {
            #pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                if (r0 + rr >= rows) break;
                const float sc = scale ? __ldg(scale + r0 + rr) : 1.f;
                #pragma unroll
                for (int b = 0; b < NB; ++b) out[b * ostride + r0 + rr] = sc * acc[rr][b];
            }
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

constexpr size_t SMEM_CAP = 200 * 1024;   // shared memory for the staged vectors + table

size_t rowdot_smem_bytes(int nb, int64_t tb) { return (32 + (size_t)nb * (size_t)(tb / 4) * 16) * sizeof(float); }

template <int NB, int R>
bool launch_rowdot_smem(const uint8_t* T, int64_t rows, int64_t len, int64_t tb, const float* V, int64_t vstride,
                        const float* scale, float* out, int64_t ostride, cudaStream_t s) {
    const size_t smem = rowdot_smem_bytes(NB, tb);
    if (smem > SMEM_CAP) return false;
    static bool attr = false;   // per process; the attribute applies to every device
    if (!attr) {
        cudaFuncSetAttribute(rowdot_smem_kernel<NB, R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_CAP);
        attr = true;
    }
    const int64_t want = ((rows + R - 1) / R + RS_THREADS / 32 - 1) / (RS_THREADS / 32);
    const int64_t cap = 16 * (int64_t)sms();
    const unsigned grid = (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
    rowdot_smem_kernel<NB, R><<<grid, RS_THREADS, smem, s>>>(T, rows, len, tb, V, vstride, scale, out, ostride);
    return true;
}

template <int NB>
void launch_rowdot(const uint8_t* T, int64_t rows, int64_t len, int64_t tb, const float* V, int64_t vstride,
                   const float* scale, float* out, int64_t ostride, cudaStream_t s) {
    // rows per warp: share each staged vector load among R rows, but keep >= 16
    // warps per SM busy (R = 1 for short matrices)
    const int64_t nsm = sms();
    bool done;
    if (NB == 1 && rows >= 4 * 24 * nsm) done = launch_rowdot_smem<NB, NB == 1 ? 4 : 1>(T, rows, len, tb, V, vstride, scale, out, ostride, s);
    else if (NB <= 2 && rows >= 2 * 16 * nsm) done = launch_rowdot_smem<NB, NB <= 2 ? 2 : 1>(T, rows, len, tb, V, vstride, scale, out, ostride, s);
    else done = launch_rowdot_smem<NB, 1>(T, rows, len, tb, V, vstride, scale, out, ostride, s);
    if (done) return;
    const int64_t want = (rows + 7) / 8;
    const int64_t cap = nsm * 8;
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
    // vectors per pass: the most that still fit shared memory for both products
    int per = MAXB;
    while (per > 1 && (rowdot_smem_bytes(per, cb) > SMEM_CAP || rowdot_smem_bytes(per, bb) > SMEM_CAP)) per /= 2;
    for (int64_t b0 = 0; b0 < batch; b0 += per) {
        const int nb = (int)(batch - b0 < per ? batch - b0 : per);
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
