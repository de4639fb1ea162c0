// Device helpers shared by the libtq kernels.
#pragma once

#include <algorithm>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace tq {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

// Load E consecutive elements of a fp32 or bf16 row starting at element `off`.
template <int E>
__device__ __forceinline__ void load_elems(const void* base, int dtype, int64_t off, float (&v)[E]) {
    if (dtype == TQ_F32) {
        const float* p = reinterpret_cast<const float*>(base) + off;
        if constexpr (E % 4 == 0) {
#pragma unroll
            for (int i = 0; i < E; i += 4) {
                float4 f = __ldg(reinterpret_cast<const float4*>(p + i));
                v[i] = f.x; v[i + 1] = f.y; v[i + 2] = f.z; v[i + 3] = f.w;
            }
        } else if constexpr (E == 2) {
            float2 f = __ldg(reinterpret_cast<const float2*>(p));
            v[0] = f.x; v[1] = f.y;
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i) v[i] = __ldg(p + i);
        }
    } else {
        const uint16_t* p = reinterpret_cast<const uint16_t*>(base) + off;
        if constexpr (E % 8 == 0) {
#pragma unroll
            for (int i = 0; i < E; i += 8) {
                uint4 w = __ldg(reinterpret_cast<const uint4*>(p + i));
                uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    v[i + 2 * k] = bf16_bits_to_float(a[k] & 0xffffu);
                    v[i + 2 * k + 1] = bf16_bits_to_float(a[k] >> 16);
                }
            }
        } else if constexpr (E == 4) {
            uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
            v[0] = bf16_bits_to_float(w.x & 0xffffu); v[1] = bf16_bits_to_float(w.x >> 16);
            v[2] = bf16_bits_to_float(w.y & 0xffffu); v[3] = bf16_bits_to_float(w.y >> 16);
        } else if constexpr (E == 2) {
            uint32_t w = __ldg(reinterpret_cast<const unsigned int*>(p));
            v[0] = bf16_bits_to_float(w & 0xffffu); v[1] = bf16_bits_to_float(w >> 16);
        } else {
#pragma unroll
            for (int i = 0; i < E; ++i) v[i] = bf16_bits_to_float(__ldg(p + i));
        }
    }
}

// One element of a matrix stored fp32 or bf16.
__device__ __forceinline__ float mat_elem(const void* m, int dtype, int64_t i) {
    return dtype == TQ_F32 ? __ldg(reinterpret_cast<const float*>(m) + i)
                           : bf16_bits_to_float(__ldg(reinterpret_cast<const uint16_t*>(m) + i));
}

// acc[e] += sum_k MT[k][base + e] * v[k] for e < E, with MT a row-major d x d matrix
// (fp32 or bf16) and v in shared memory: y = M v for the E outputs base..base+E-1.
template <int E>
__device__ __forceinline__ void matvec_cols(const void* MT, int dtype, int d, int base,
                                            const float* __restrict__ v, float (&acc)[E]) {
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    if (dtype == TQ_F32) {
        const float* m = reinterpret_cast<const float*>(MT) + base;
#pragma unroll 4
        for (int k = 0; k < d; ++k) {
            const float vk = v[k];
            float row[E];
            load_elems<E>(m, TQ_F32, (int64_t)k * d, row);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = fmaf(row[e], vk, acc[e]);
        }
    } else {
        const uint16_t* m = reinterpret_cast<const uint16_t*>(MT) + base;
#pragma unroll 4
        for (int k = 0; k < d; ++k) {
            const float vk = v[k];
            float row[E];
            load_elems<E>(m, TQ_BF16, (int64_t)k * d, row);
#pragma unroll
            for (int e = 0; e < E; ++e) acc[e] = fmaf(row[e], vk, acc[e]);
        }
    }
}

__device__ __forceinline__ bool rht_neg(const DevState& st, int j) { return (st.signs[j >> 5] >> (j & 31)) & 1u; }

// Cell index of y: #{k : t_k <= y} over the L-1 boundaries (upper cell on a tie).
__device__ __forceinline__ int quantize_coord(const DevState& st, const float* __restrict__ tsh, float y) {
    if (st.L <= 16) {
        int c = 0;
        for (int k = 0; k < st.L - 1; ++k) c += (y >= st.t[k]) ? 1 : 0;
        return c;
    }
    int lo = 0, hi = st.L - 1;   // answer in [0, L-1]
    while (lo < hi) {
        int mid = (lo + hi) >> 1;   // is t[mid] <= y ?
        if (tsh[mid] <= y) lo = mid + 1; else hi = mid;
    }
    return lo;
}

// Extract code j (b bits, LSB-first stream) from a packed row of 32-bit words.
__device__ __forceinline__ uint32_t extract_code(const uint32_t* __restrict__ row, int nwords, int j, int b) {
    const int bit = j * b;
    const int w = bit >> 5;
    const int sh = bit & 31;
    uint64_t win = __ldg(row + w);
    if (w + 1 < nwords) win |= (uint64_t)__ldg(row + w + 1) << 32;
    return (uint32_t)(win >> sh) & ((1u << b) - 1u);
}


// Table lookups over the 8 nibbles of a packed word: acc[qi].x + acc[qi].y grows by
// sum_m T_m[e_m], e_m the m-th nibble of w and T_m the 16-entry float table at t0 + 16 m
// (query qi's tables STRIDE floats further on). Two masks put the nibbles, times 4, into
// bytes; a lookup is then one byte permute and one shared-memory load, and the two values of
// each permute go into .x and .y with one f32x2 add (two independent chains per query).
template <int QT, int STRIDE>
__device__ __forceinline__ void add_nibbles(uint32_t w, const float* t0, float2 (&acc)[QT]) {
    const uint32_t lo4 = (w << 2) & 0x3C3C3C3Cu;   // nibbles 0, 2, 4, 6
    const uint32_t hi4 = (w >> 2) & 0x3C3C3C3Cu;   // nibbles 1, 3, 5, 7
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const uint32_t o0 = __byte_perm(lo4, 0u, 0x4440u | m);
        const uint32_t o1 = __byte_perm(hi4, 0u, 0x4440u | m);
#pragma unroll
        for (int qi = 0; qi < QT; ++qi) {
            const char* t = reinterpret_cast<const char*>(t0 + qi * STRIDE + 2 * m * 16);
            const float2 v = make_float2(*reinterpret_cast<const float*>(t + o0),
                                         *reinterpret_cast<const float*>(t + 64 + o1));
            acc[qi] = __fadd2_rn(acc[qi], v);
        }
    }
}

// In-place Hadamard transform of order d = 12 m (m a power of two) on buf[0..d), viewed as
// 12 rows of m: Sylvester's transform along each row, then Paley's H_12 (rows of st.h12,
// bit c of row a <=> H_12[a][c] = -1) across the rows; `transpose` applies H_12^T instead
// (Sylvester's factor is symmetric), which inverts the transform up to 1/d. Threads
// tid = 0..nt-1 of a group share buf; `sync` orders their shared-memory accesses.
template <typename Sync>
__device__ __forceinline__ void kron_hadamard(float* buf, int d, const uint32_t* __restrict__ h12, bool transpose,
                                              int tid, int nt, Sync sync) {
    const int m = d / 12;
    for (int h = 1; h < m; h <<= 1) {
        for (int p = tid; p < d / 2; p += nt) {
            const int row = p / (m >> 1), pr = p - row * (m >> 1);
            const int j = row * m + (pr / h) * 2 * h + (pr % h);
            const float a = buf[j], b = buf[j + h];
            buf[j] = a + b;
            buf[j + h] = a - b;
        }
        sync();
    }
    for (int col = tid; col < m; col += nt) {
        float t[12];
#pragma unroll
        for (int c = 0; c < 12; ++c) t[c] = buf[c * m + col];
#pragma unroll
        for (int a = 0; a < 12; ++a) {
            float acc = 0.f;
#pragma unroll
            for (int c = 0; c < 12; ++c) {
                const bool neg = transpose ? ((h12[c] >> a) & 1u) : ((h12[a] >> c) & 1u);
                acc += neg ? -t[c] : t[c];
            }
            buf[a * m + col] = acc;
        }
    }
    sync();
}

}  // namespace tq
