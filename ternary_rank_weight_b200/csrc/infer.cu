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
// When the vectors fit in shared memory (NB * len * 4 bytes up to 200 KB) they are
// staged there once per CTA and every trit is decoded exactly in registers and applied
// with f32x2 arithmetic (tdot_kernel); otherwise one warp per row walks the nonzero
// trits of its 16-byte chunks and reads the vector through L1 (rowdot_kernel).
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
                // positions j0 .. j0+15; padding trits past len are skipped
                const int64_t j0 = c * 64 + 16 * h;
                uint32_t nz = even_bits(w4[h]);
                const uint32_t ng = even_bits(w4[h] >> 1);
                while (nz) {
                    const int t = __ffs(nz) - 1;
                    nz &= nz - 1u;
                    if (j0 + t >= len) break;                 // padding trits past len are not read
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

// Shared-memory variant with exact in-register trit decoding (sm_100a f32x2 arithmetic).
//
// A trit's 2-bit code q (bit 0: nonzero, bit 1: negative) is the trit read as a signed
// 2-bit integer, t = q0 - 2 q1.  With its high bit flipped it becomes the field
// v = t + 2 in {1, 2, 3}.  Placed at bit 2p (p <= 10) of the mantissa of 2.0 by one
// three-input logic operation, it gives F = 2 + v 2^(2p-22) exactly, and
// F - (2 + 2^(2p-21)) = t 2^(2p-22) is exact as well (both operands lie in [2, 4)).
// The staged vector entry is pre-scaled by 2^(22-2p), so the product of the two is
// exactly t x, and each row dot is a plain fp32 sum of exact terms in a fixed order.
// Trits 0..10 of a 32-bit word sit at p = 0..10 of the word itself, trits 11..15 at
// p = 0..4 of the word shifted right by 22.  Pairs of trits go through one f32x2
// subtraction and one f32x2 fused multiply-add per vector: with the logic operations,
// about two instructions per trit and row, and no table lookups.
//
// Layout: a warp takes R rows at once; lane l reads 32-bit words l, l + 32, ... of each row
// (G words per lane issued ahead of their use: the next chunk's words are loaded while the
// current chunk is decoded), and each float4 of the staged vector serves the R rows.  The staged
// vector keeps the 16 entries of word w at floats 20 w .. 20 w + 15 (4 floats of padding per
// word), so the eight lanes of a quarter-warp, reading eight consecutive words, hit distinct banks
// and each quad's offset within its word is a constant.  The grid is at most one CTA per SM; each
// CTA stages the vectors once and its warps take row groups interleaved across CTAs.  Vectors
// whose largest magnitude reaches 2^104 are staged with an extra power-of-two scale (undone on
// the outputs), so the pre-scaling cannot overflow.
//
// The second product of a matvec (y = B z) is launched as a programmatic dependent of
// the first: its CTAs may start while the first kernel runs, prefetch their trit rows into
// L2, and wait (griddepcontrol.wait) before they read z.
constexpr int TD_MAX_WARPS = 16;

constexpr int SW = 20;   // floats per staged word of 16 entries (4 of padding: conflict-free float4 reads)

__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float2 upk2(uint64_t v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ uint64_t sub_x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma_x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// position p of trit j (0..15) of a word, and the word it is read from
template <int J> struct TritPos { static constexpr int P = J <= 10 ? J : J - 11; static constexpr bool HI = J > 10; };

// The words a trit is read from carry the exponent bits of 2.0 already (wa = flipped word | 2.0,
// wb = flipped word >> 22 | 2.0), so F = 2 + (t + 2) 2^(2p-22) is one AND with the field mask plus bit 30.
// the subtrahend 2 + 2 * 2^(2p-22) of each trit pair, as the packed pairs the loop uses
// (pairs (0,1) (2,3) (4,5) (6,7) (8,9) (10,11) (12,13) (14,15) of a word)
__host__ __device__ constexpr uint32_t trit_bias_bits(int j) {
    return 0x40000000u | (2u << (2 * (j <= 10 ? j : j - 11)));
}
__constant__ uint64_t c_trit_bias[8] = {
    (uint64_t)trit_bias_bits(0) | ((uint64_t)trit_bias_bits(1) << 32),
    (uint64_t)trit_bias_bits(2) | ((uint64_t)trit_bias_bits(3) << 32),
    (uint64_t)trit_bias_bits(4) | ((uint64_t)trit_bias_bits(5) << 32),
    (uint64_t)trit_bias_bits(6) | ((uint64_t)trit_bias_bits(7) << 32),
    (uint64_t)trit_bias_bits(8) | ((uint64_t)trit_bias_bits(9) << 32),
    (uint64_t)trit_bias_bits(10) | ((uint64_t)trit_bias_bits(11) << 32),
    (uint64_t)trit_bias_bits(12) | ((uint64_t)trit_bias_bits(13) << 32),
    (uint64_t)trit_bias_bits(14) | ((uint64_t)trit_bias_bits(15) << 32)};
// coefficient pair of trits J, J+1 (exact t 2^(2p-22) each); kb = c_trit_bias[J / 2].  The pair is
// masked out of a 64-bit source that holds the words of both trits (wa:wa, wa:wb or wb:wb), so the two
// halves land in the register pair the f32x2 subtraction reads.
__host__ __device__ constexpr uint32_t trit_mask(int j) {
    return (3u << (2 * (j <= 10 ? j : j - 11))) | 0x40000000u;
}
template <int J>
__device__ __forceinline__ uint64_t trit_pair(uint64_t waa, uint64_t wab, uint64_t wbb, uint64_t kb) {
    constexpr uint64_t M = (uint64_t)trit_mask(J) | ((uint64_t)trit_mask(J + 1) << 32);
    const uint64_t src = (J + 1 <= 10) ? waa : (J >= 11 ? wbb : wab);
    return sub_x2(src & M, kb);
}

__host__ __device__ __forceinline__ float pow2f(int e) {       // 2^e for -126 <= e <= 127
    union { uint32_t u; float f; } c;
    c.u = (uint32_t)(127 + e) << 23;
    return c.f;
}

template <int NB, int R>
__global__ void __launch_bounds__(32 * TD_MAX_WARPS) tdot_kernel(const uint8_t* __restrict__ T, int64_t rows,
                                                                  int64_t len, int64_t tb, const float* __restrict__ V,
                                                                  int64_t vstride, const float* __restrict__ scale,
                                                                  float* __restrict__ out, int64_t ostride,
                                                                  int dependent) {
    extern __shared__ __align__(16) float sv[];   // NB x spitch, pre-scaled, word w at SW * w
    __shared__ uint32_t vmax[NB];
    const int lane = threadIdx.x & 31;
    const int nw = blockDim.x >> 5;
    const int64_t words = tb / 4;
    const int64_t lenp = words * 16;
    const int64_t spitch = words * SW;
    const int64_t groups = (rows + R - 1) / R;
    const int64_t g0 = (int64_t)(threadIdx.x >> 5) * gridDim.x + blockIdx.x;
    const int64_t gstride = (int64_t)nw * gridDim.x;
    // the first chunk of this warp's first row group is loaded before anything else, so that its
    // memory latency overlaps the staging (and, in a dependent launch, the producer's tail: the
    // trits are not written by the producer)
    constexpr int G = R >= 4 ? 4 : 8;                          // words per row and lane in flight
    auto load_chunk = [&](uint32_t (&dst)[G][R], int64_t grp, int64_t w0) {
        #pragma unroll
        for (int g = 0; g < G; ++g) {
            const int64_t w = w0 + lane + 32 * g;
            #pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                const int64_t r = grp * R + rr;
                dst[g][rr] = (r < rows && w < words) ? __ldg(reinterpret_cast<const uint32_t*>(T + r * tb) + w) : 0u;
            }
        }
    };
    uint32_t q[G][R], qn[G][R];
    if (g0 < groups) load_chunk(q, g0, 0);
    if (dependent) {
        // this warp's trit rows into L2 while the producer of V runs, then wait for it
        for (int64_t g = g0; g < groups; g += gstride) {
            const int64_t r = g * R + lane;
            if (lane < R && r < rows)
                asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(T + r * tb), "r"((uint32_t)tb) : "memory");
        }
        asm volatile("griddepcontrol.wait;" ::: "memory");
    } else {
        asm volatile("griddepcontrol.launch_dependents;");
    }
    if (threadIdx.x < NB) vmax[threadIdx.x] = 0u;
    // stage the raw vectors: 16-byte asynchronous copies, all in flight at once, or plain loads
    // when V is not 16-byte aligned.  Group g (entries 4 g .. 4 g + 3) goes to word g / 4, quad g % 4.
    const bool vec4 = ((len & 3) == 0) && ((vstride & 3) == 0) && ((reinterpret_cast<uintptr_t>(V) & 15) == 0);
    const int64_t ngroups = lenp / 4;
    auto slot = [&](int64_t g) { return SW * (g >> 2) + 4 * (g & 3); };
    for (int b = 0; b < NB; ++b) {
        if (vec4) {
            const float4* V4 = reinterpret_cast<const float4*>(V + b * vstride);
            for (int64_t g = threadIdx.x; g < ngroups; g += blockDim.x) {
                float* dst = sv + b * spitch + slot(g);
                if (4 * g < len) {
                    const unsigned saddr = (unsigned)__cvta_generic_to_shared(dst);
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(saddr), "l"(V4 + g) : "memory");
                } else {
                    *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        } else {
            for (int64_t g0s = threadIdx.x; g0s < ngroups; g0s += 2 * (int64_t)blockDim.x) {
                float v[2][4];
                #pragma unroll
                for (int u = 0; u < 2; ++u)
                    #pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int64_t j = 4 * (g0s + u * (int64_t)blockDim.x) + e;
                        v[u][e] = j < len ? __ldg(V + b * vstride + j) : 0.f;
                    }
                #pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int64_t g = g0s + u * (int64_t)blockDim.x;
                    if (g < ngroups)
                        *reinterpret_cast<float4*>(sv + b * spitch + slot(g)) = make_float4(v[u][0], v[u][1], v[u][2], v[u][3]);
                }
            }
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    // largest magnitude of each vector (from shared memory), then the pre-scaling in place
    for (int b = 0; b < NB; ++b) {
        uint32_t mx = 0u;
        for (int64_t g = threadIdx.x; g < ngroups; g += blockDim.x) {
            const float4 t = *reinterpret_cast<const float4*>(sv + b * spitch + slot(g));
            mx = max(mx, max(max(__float_as_uint(t.x) & 0x7fffffffu, __float_as_uint(t.y) & 0x7fffffffu),
                             max(__float_as_uint(t.z) & 0x7fffffffu, __float_as_uint(t.w) & 0x7fffffffu)));
        }
        #pragma unroll
        for (int o = 16; o; o >>= 1) mx = max(mx, __shfl_xor_sync(FULL, mx, o));
        if (lane == 0) atomicMax(&vmax[b], mx);
    }
    __syncthreads();
    int shift[NB];
    #pragma unroll
    for (int b = 0; b < NB; ++b) {
        const int e = (int)(vmax[b] >> 23) - 127;               // inf / NaN: 128, left unscaled
        shift[b] = (e >= 104 && e < 128) ? e - 103 : 0;
    }
    for (int b = 0; b < NB; ++b) {
        for (int64_t g = threadIdx.x; g < ngroups; g += blockDim.x) {
            float4* p4 = reinterpret_cast<float4*>(sv + b * spitch + slot(g));
            float4 t = *p4;
            float* tv = &t.x;
            #pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int q = 4 * (int)(g & 3) + u;               // trit position within the word
                const int p = q <= 10 ? q : q - 11;
                tv[u] *= pow2f(22 - 2 * p - shift[b]);
            }
            *p4 = t;
        }
    }
    __syncthreads();
    uint64_t kb[8];                                            // loop-invariant subtrahends, in registers
    #pragma unroll
    for (int i = 0; i < 8; ++i) kb[i] = c_trit_bias[i];
    for (int64_t grp = g0; grp < groups; grp += gstride) {
        const int64_t r0 = grp * R;
        uint64_t acc[R][NB], acc2[R][NB];   // for one or two vectors, two sums per row and vector: shorter chains
        #pragma unroll
        for (int rr = 0; rr < R; ++rr)
            #pragma unroll
            for (int b = 0; b < NB; ++b) acc[rr][b] = acc2[rr][b] = 0ull;
        // software pipeline: the words of the next chunk are loaded before the current chunk is used
        if (grp != g0) load_chunk(q, grp, 0);
        for (int64_t w0 = 0; w0 < words; w0 += 32 * G) {
            load_chunk(qn, grp, w0 + 32 * G);
            #pragma unroll
            for (int g = 0; g < G; ++g) {
                const int64_t w = w0 + lane + 32 * g;
                if (w >= words) break;
                const float* svw = sv + SW * w;
                uint64_t waa[R], wab[R], wbb[R];
                #pragma unroll
                for (int rr = 0; rr < R; ++rr) {
                    const uint32_t fl = q[g][rr] ^ 0xAAAAAAAAu;   // field v = t + 2 of every trit
                    const uint32_t wa = fl | 0x40000000u;
                    const uint32_t wb = (fl >> 22) | 0x40000000u;
                    waa[rr] = ((uint64_t)wa << 32) | wa;
                    wab[rr] = ((uint64_t)wb << 32) | wa;
                    wbb[rr] = ((uint64_t)wb << 32) | wb;
                }
#define EXTERND_TDOT_QUAD(H, J0)                                                                                   \
                {                                                                                                   \
                    float4 x4[NB];                                                                                  \
                    _Pragma("unroll") for (int b = 0; b < NB; ++b)                                                 \
                        x4[b] = *reinterpret_cast<const float4*>(svw + b * spitch + 4 * H);                         \
                    _Pragma("unroll") for (int rr = 0; rr < R; ++rr) {                                             \
                        const uint64_t c01 = trit_pair<J0>(waa[rr], wab[rr], wbb[rr], kb[J0 / 2]);                  \
                        const uint64_t c23 = trit_pair<J0 + 2>(waa[rr], wab[rr], wbb[rr], kb[J0 / 2 + 1]);          \
                        _Pragma("unroll") for (int b = 0; b < NB; ++b) {                                           \
                            acc[rr][b] = fma_x2(c01, pk2(x4[b].x, x4[b].y), acc[rr][b]);                            \
                            if constexpr (NB <= 2) acc2[rr][b] = fma_x2(c23, pk2(x4[b].z, x4[b].w), acc2[rr][b]);   \
                            else acc[rr][b] = fma_x2(c23, pk2(x4[b].z, x4[b].w), acc[rr][b]);                       \
                        }                                                                                           \
                    }                                                                                               \
                }
                EXTERND_TDOT_QUAD(0, 0)
                EXTERND_TDOT_QUAD(1, 4)
                EXTERND_TDOT_QUAD(2, 8)
                EXTERND_TDOT_QUAD(3, 12)
#undef EXTERND_TDOT_QUAD
            }
            #pragma unroll
            for (int g = 0; g < G; ++g)
                #pragma unroll
                for (int rr = 0; rr < R; ++rr) q[g][rr] = qn[g][rr];
        }
        float res[R][NB];
        #pragma unroll
        for (int rr = 0; rr < R; ++rr)
            #pragma unroll
            for (int b = 0; b < NB; ++b) {
                const float2 v2 = upk2(acc[rr][b]), w2 = upk2(acc2[rr][b]);
                float a = (v2.x + v2.y) + (w2.x + w2.y);
                #pragma unroll
                for (int o = 16; o; o >>= 1) a += __shfl_xor_sync(FULL, a, o);
                res[rr][b] = a;
            }
        if (lane == 0) {
            #pragma unroll
            for (int rr = 0; rr < R; ++rr) {
                if (r0 + rr >= rows) break;
                const float sc = scale ? __ldg(scale + r0 + rr) : 1.f;
                #pragma unroll
                for (int b = 0; b < NB; ++b) out[b * ostride + r0 + rr] = sc * (res[rr][b] * pow2f(shift[b]));
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

constexpr size_t SMEM_CAP = 200 * 1024;   // shared memory for the staged vectors

size_t tdot_smem_bytes(int nb, int64_t tb) { return (size_t)nb * (size_t)(tb / 4) * SW * sizeof(float); }

template <int NB, int R>
cudaError_t launch_tdot(const uint8_t* T, int64_t rows, int64_t len, int64_t tb, const float* V, int64_t vstride,
                        const float* scale, float* out, int64_t ostride, bool dependent, cudaStream_t s) {
    const size_t smem = tdot_smem_bytes(NB, tb);
    static bool attr[64] = {};   // set once per device of the process
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return cudaGetLastError();
    if (dev < 0 || dev >= 64 || !attr[dev]) {
        const cudaError_t e = cudaFuncSetAttribute(tdot_kernel<NB, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (int)SMEM_CAP);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr[dev] = true;
    }
    const int64_t nsm = sms();
    const int64_t groups = (rows + R - 1) / R;
    int64_t warps = (groups + nsm - 1) / nsm;
    warps = warps < 1 ? 1 : (warps > TD_MAX_WARPS ? TD_MAX_WARPS : warps);
    int64_t grid = (groups + warps - 1) / warps;
    grid = grid < nsm ? grid : nsm;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)(32 * warps));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = dependent ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, tdot_kernel<NB, R>, T, rows, len, tb, V, vstride, scale, out, ostride,
                              dependent ? 1 : 0);
}

template <int NB>
cudaError_t launch_rowdot(const uint8_t* T, int64_t rows, int64_t len, int64_t tb, const float* V, int64_t vstride,
                          const float* scale, float* out, int64_t ostride, bool dependent, cudaStream_t s) {
    if (tdot_smem_bytes(NB, tb) <= SMEM_CAP) {
        // rows per warp: four when that still leaves >= 8 warps per SM, else two, so each staged float4
        // serves several rows (one row per warp makes the staged-vector reads the limit for batches)
        const int64_t nsm = sms();
        if constexpr (NB == 1) {
            if (rows >= 4 * 8 * nsm) return launch_tdot<NB, 4>(T, rows, len, tb, V, vstride, scale, out, ostride, dependent, s);
            return launch_tdot<NB, 2>(T, rows, len, tb, V, vstride, scale, out, ostride, dependent, s);
        } else if constexpr (NB == 2) {
            return launch_tdot<NB, 2>(T, rows, len, tb, V, vstride, scale, out, ostride, dependent, s);
        } else {
            return launch_tdot<NB, 2>(T, rows, len, tb, V, vstride, scale, out, ostride, dependent, s);
        }
    }
    const int64_t want = (rows + 7) / 8;
    const int64_t cap = (int64_t)sms() * 8;
    const unsigned grid = (unsigned)(want < cap ? (want > 0 ? want : 1) : cap);
    rowdot_kernel<NB><<<grid, RD_THREADS, 0, s>>>(T, rows, len, tb, V, vstride, scale, out, ostride);
    return cudaGetLastError();
}

cudaError_t rowdot(int nb, const uint8_t* T, int64_t rows, int64_t len, int64_t tb, const float* V, int64_t vstride,
                   const float* scale, float* out, int64_t ostride, bool dependent, cudaStream_t s) {
    switch (nb) {   // one instantiation per vector count: a kernel touches exactly nb vectors
        case 1: return launch_rowdot<1>(T, rows, len, tb, V, vstride, scale, out, ostride, dependent, s);
        case 2: return launch_rowdot<2>(T, rows, len, tb, V, vstride, scale, out, ostride, dependent, s);
        case 3: return launch_rowdot<3>(T, rows, len, tb, V, vstride, scale, out, ostride, dependent, s);
        case 4: return launch_rowdot<4>(T, rows, len, tb, V, vstride, scale, out, ostride, dependent, s);
        case 5: return launch_rowdot<5>(T, rows, len, tb, V, vstride, scale, out, ostride, dependent, s);
        case 6: return launch_rowdot<6>(T, rows, len, tb, V, vstride, scale, out, ostride, dependent, s);
        case 7: return launch_rowdot<7>(T, rows, len, tb, V, vstride, scale, out, ostride, dependent, s);
        case 8: return launch_rowdot<8>(T, rows, len, tb, V, vstride, scale, out, ostride, dependent, s);
        default: return cudaErrorInvalidValue;
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
    if ((reinterpret_cast<uintptr_t>(Bt) & 15) || (reinterpret_cast<uintptr_t>(C) & 15)) return EXTERND_EINVAL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t cb = (int64_t)trit_bytes(n), bb = (int64_t)trit_bytes(k);
    // vectors per pass: the most that still fit shared memory for both products
    int per = MAXB;
    while (per > 1 && (tdot_smem_bytes(per, cb) > SMEM_CAP || tdot_smem_bytes(per, bb) > SMEM_CAP)) --per;
    for (int64_t b0 = 0; b0 < batch; b0 += per) {
        const int nb = (int)(batch - b0 < per ? batch - b0 : per);
        // z = diag(D) (C x): k rows of n trits
        if (rowdot(nb, C, k, n, cb, X + b0 * n, n, D, z_work, k, false, s) != cudaSuccess) { cudaGetLastError(); return EXTERND_ECUDA; }
        // y = B z: m rows of k trits (B transposed), a programmatic dependent of the first product
        if (rowdot(nb, Bt, m, k, bb, z_work, k, nullptr, Y + b0 * m, m, true, s) != cudaSuccess) { cudaGetLastError(); return EXTERND_ECUDA; }
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
