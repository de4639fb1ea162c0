// Encoder for d = 128 with a dense rotation (Haar-random Pi stored fp32 or bf16), fp32 or bf16
// input, TurboQuant_mse or TurboQuant_prod with 0- to 4-bit MSE codes (0: prod at b = 1, where
// the residual is the whole rotated vector).
//
// TurboQuant review (Jump2Paper): Theorem 1 (store ||x||, rotate by Pi, give every coordinate
// of the rotated unit vector its Lloyd-Max cell), Definition 1 + Theorem 2 (QJL signs of S r on
// the residual, ||r|| kept). The rotation y = Pi x and the projection S r are fp32 products over
// 128 coordinates, so this kernel treats them as two small GEMMs on the CUDA cores:
//   a persistent block of 256 threads stages Pi^T (and S^T) once, as fp32, in shared memory and
//   then walks tiles of 128 vectors. A tile's input is staged transposed (coordinate-major), so
//   that for each k the 128 vectors' values are contiguous; thread t owns the 8 x 8 outputs of
//   8 vectors (4 (t % 16) .. +3 and 64 + 4 (t % 16) .. +3) and coordinates 8 (t / 16) .. +7,
//   reads 8 + 8 operands per k
//   (four 16-byte shared loads) and does 64 FMAs. Y = X Pi^T in registers is divided by ||x||,
//   quantized against the boundaries (branch-free binary search), the residual r = y - c[idx]
//   replaces the input tile, and Z = R S^T gives the signs. Codes and signs are packed per
//   thread (its 8 coordinates are 8 b contiguous bits of the vector's row), staged as the tile's
//   rows and written out with 16-byte stores.
// Decisions are made on fp32 values as the other kernels make them (y_j against the fp32
// boundaries, (S r)_j >= 0); zero vectors follow the same rule (codes of 0, all signs +1).
#include <cuda_bf16.h>

#include "common.cuh"

namespace tq {

namespace {

constexpr int kD = 128;
constexpr int kT = 128;        // vectors per tile
constexpr int kThreads = 256;
constexpr int kLd = kT + 4;    // row stride (floats) of the transposed tiles

struct DenseSmem {
    float piT[kD * kD];        // Pi^T[k][j] = Pi[j][k]
    float sT[kD * kD];         // S^T (prod)
    float xt[kD * kLd];        // x tile transposed: xt[k][v]; then the residual r[k][v]
    float nrm[kT];             // ||x|| of the tile's vectors
    float rr[16][kT];          // partial ||r||^2: [coordinate group][vector]
    uint8_t rows[kT * 64];     // the tile's packed code rows (16 b bytes each)
    uint8_t zrows[kT * 16];    // the tile's packed sign rows
    float c[16];
    float t[16];
};

// y (fp32) -> its cell #{k : t_k <= y} for L = 2^B levels, by binary search on the sorted
// boundaries t[0..L-2] (upper cell on a tie).
template <int B>
__device__ __forceinline__ int cell(const float* t, float y) {
    static_assert(B >= 1, "a cell search needs at least two levels");
    int idx = 0;
#pragma unroll
    for (int step = 1 << (B - 1); step >= 1; step >>= 1) idx += (y >= t[idx + step - 1]) ? step : 0;
    return idx;
}

template <int B, bool PROD, bool XF32, bool MF32>
__global__ void __launch_bounds__(kThreads, 1)
encode_dense128_kernel(const DevState st, const void* __restrict__ x, int64_t n, int64_t ld,
                       uint8_t* __restrict__ codes, uint8_t* __restrict__ qjl, float* __restrict__ norms,
                       float* __restrict__ rnorms) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    DenseSmem& sm = *reinterpret_cast<DenseSmem*>(smem_raw);
    const int tid = threadIdx.x;
    // vectors 4 vg .. +3 and 64 + 4 vg .. +3 (so that a warp's 16 vector groups read one
    // contiguous 256-byte run of a row of the tile), coordinates 8 og .. +7
    const int vg = tid & 15, og = tid >> 4;
    auto vec_of = [&](int a) { return (a < 4) ? 4 * vg + a : 64 + 4 * vg + (a - 4); };
    constexpr int kRow = 16 * B;              // code bytes per vector (none for B = 0)

    // stage Pi^T (and S^T) as fp32
    for (int i = tid; i < kD * kD; i += kThreads) {
        sm.piT[i] = MF32 ? reinterpret_cast<const float*>(st.piT)[i]
                         : bf16_bits_to_float(reinterpret_cast<const uint16_t*>(st.piT)[i]);
        if constexpr (PROD)
            sm.sT[i] = MF32 ? reinterpret_cast<const float*>(st.sT)[i]
                            : bf16_bits_to_float(reinterpret_cast<const uint16_t*>(st.sT)[i]);
    }
    if (tid < 16) {
        sm.c[tid] = (tid < st.L) ? st.c[tid] : 0.f;
        sm.t[tid] = (tid < st.L - 1) ? st.t[tid] : INFINITY;
    }
    __syncthreads();

    const int64_t ntiles = (n + kT - 1) / kT;
    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t v0 = tile * kT;
        // ---- stage the tile transposed: lane = vector (conflict-free stores along a row of
        // xt), warp w takes vectors 32 (w % 4) .. +31 and coordinates 64 (w / 4) .. +63;
        // ||x||^2 from the two halves ----
        {
            const int lane = tid & 31, warp = tid >> 5;
            const int v = 32 * (warp & 3) + lane, k0 = 64 * (warp >> 2);
            float ss = 0.f;
            if (v0 + v < n) {
#pragma unroll
                for (int c = 0; c < 64; c += 8) {
                    float e[8];
                    load_elems<8>(x, XF32 ? TQ_F32 : TQ_BF16, (v0 + v) * ld + k0 + c, e);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        sm.xt[(k0 + c + i) * kLd + v] = e[i];
                        ss = fmaf(e[i], e[i], ss);
                    }
                }
            } else {
#pragma unroll
                for (int c = 0; c < 64; ++c) sm.xt[(k0 + c) * kLd + v] = 0.f;
            }
            sm.rr[warp >> 2][v] = ss;   // (reused below for ||r||^2 once read)
        }
        __syncthreads();
        if (tid < kT) sm.nrm[tid] = sqrtf(sm.rr[0][tid] + sm.rr[1][tid]);
        // ---- Y = X Pi^T: acc[a][b] = y of vector vec_of(a), coordinate 8 og + b ----
        float acc[8][8];
#pragma unroll
        for (int a = 0; a < 8; ++a)
#pragma unroll
            for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
#pragma unroll 4
        for (int k = 0; k < kD; ++k) {
            const float4 x0 = *reinterpret_cast<const float4*>(&sm.xt[k * kLd + 4 * vg]);
            const float4 x1 = *reinterpret_cast<const float4*>(&sm.xt[k * kLd + 64 + 4 * vg]);
            const float4 p0 = *reinterpret_cast<const float4*>(&sm.piT[k * kD + 8 * og]);
            const float4 p1 = *reinterpret_cast<const float4*>(&sm.piT[k * kD + 8 * og + 4]);
            const float xa[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
            const float pb[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(xa[a], pb[b], acc[a][b]);
        }
        __syncthreads();   // every thread is done with the input tile
        // ---- quantize; residual into the tile buffer; packed codes ----
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            const int v = vec_of(a);
            const float nu = sm.nrm[v];
            const float sc = (nu > 0.f) ? 1.f / nu : 0.f;
            uint32_t word = 0u;   // the 8 codes of coordinates 8 og .. +7: 8 B bits
            float r2 = 0.f;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                const float y = acc[a][b] * sc;
                float r = y;   // B = 0: no MSE stage, the residual is y
                if constexpr (B > 0) {
                    const int c = cell<B>(sm.t, y);
                    word |= (uint32_t)c << (B * b);
                    r = (nu > 0.f) ? (y - sm.c[c]) : 0.f;
                }
                r2 = fmaf(r, r, r2);
                if constexpr (PROD) sm.xt[(8 * og + b) * kLd + v] = r;
            }
            // bytes og*B .. og*B+B-1 of the vector's code row
#pragma unroll
            for (int q = 0; q < B; ++q) sm.rows[v * kRow + og * B + q] = (uint8_t)(word >> (8 * q));
            if constexpr (PROD) sm.rr[og][v] = r2;
        }
        if constexpr (PROD) {
            __syncthreads();
            // ---- Z = R S^T: signs [(S r)_j >= 0] of coordinates 8 og .. +7 ----
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
#pragma unroll 4
            for (int k = 0; k < kD; ++k) {
                const float4 x0 = *reinterpret_cast<const float4*>(&sm.xt[k * kLd + 4 * vg]);
                const float4 x1 = *reinterpret_cast<const float4*>(&sm.xt[k * kLd + 64 + 4 * vg]);
                const float4 p0 = *reinterpret_cast<const float4*>(&sm.sT[k * kD + 8 * og]);
                const float4 p1 = *reinterpret_cast<const float4*>(&sm.sT[k * kD + 8 * og + 4]);
                const float xa[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                const float pb[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                for (int a = 0; a < 8; ++a)
#pragma unroll
                    for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(xa[a], pb[b], acc[a][b]);
            }
#pragma unroll
            for (int a = 0; a < 8; ++a) {
                uint32_t z = 0u;
#pragma unroll
                for (int b = 0; b < 8; ++b) z |= (acc[a][b] >= 0.f ? 1u : 0u) << b;
                sm.zrows[vec_of(a) * 16 + og] = (uint8_t)z;
            }
        }
        __syncthreads();
        // ---- write the tile: code rows, sign rows, norms ----
        const int nv = (int)((n - v0) < kT ? (n - v0) : kT);
        if constexpr (B > 0) {
            const uint4* src = reinterpret_cast<const uint4*>(sm.rows);
            uint4* dst = reinterpret_cast<uint4*>(codes + v0 * kRow);
            for (int i = tid; i < nv * kRow / 16; i += kThreads) dst[i] = src[i];
        }
        if constexpr (PROD) {
            const uint4* src = reinterpret_cast<const uint4*>(sm.zrows);
            uint4* dst = reinterpret_cast<uint4*>(qjl + v0 * 16);
            for (int i = tid; i < nv; i += kThreads) dst[i] = src[i];
        }
        if (tid < nv) {
            norms[v0 + tid] = sm.nrm[tid];
            if constexpr (PROD) {
                float s = 0.f;
#pragma unroll
                for (int g = 0; g < 16; ++g) s += sm.rr[g][tid];
                rnorms[v0 + tid] = sqrtf(s);
            }
        }
        __syncthreads();   // the buffers are reused by the next tile
    }
}

template <int B, bool PROD, bool XF32, bool MF32>
int launch_dense(const DevState& st, const void* x, int64_t n, int64_t ld, uint8_t* codes, uint8_t* qjl,
                 float* norms, float* rnorms, cudaStream_t s) {
    auto kern = encode_dense128_kernel<B, PROD, XF32, MF32>;
    const size_t smem = sizeof(DenseSmem);
    static int attr_set_for_device = -1;   // per instantiation
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_set_for_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return (int)e;
        attr_set_for_device = dev;
    }
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t ntiles = (n + kT - 1) / kT;
    const int grid = (int)std::min<int64_t>(ntiles, (int64_t)(sms > 0 ? sms : 148));
    kern<<<grid, kThreads, smem, s>>>(st, x, n, ld, codes, qjl, norms, rnorms);
    return (int)cudaGetLastError();
}

template <int B, bool PROD>
int launch_dense_t(const DevState& st, int dtype, const void* x, int64_t n, int64_t ld, uint8_t* codes, uint8_t* qjl,
                   float* norms, float* rnorms, cudaStream_t s) {
    const bool mf32 = st.mat_dtype == TQ_F32;
    if (dtype == TQ_F32)
        return mf32 ? launch_dense<B, PROD, true, true>(st, x, n, ld, codes, qjl, norms, rnorms, s)
                    : launch_dense<B, PROD, true, false>(st, x, n, ld, codes, qjl, norms, rnorms, s);
    return mf32 ? launch_dense<B, PROD, false, true>(st, x, n, ld, codes, qjl, norms, rnorms, s)
                : launch_dense<B, PROD, false, false>(st, x, n, ld, codes, qjl, norms, rnorms, s);
}

template <bool PROD>
int launch_dense_b(const DevState& st, int dtype, const void* x, int64_t n, int64_t ld, uint8_t* codes,
                   uint8_t* qjl, float* norms, float* rnorms, cudaStream_t s) {
    switch (st.b_mse) {
        case 0:
            if constexpr (PROD) return launch_dense_t<0, true>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
            return (int)cudaErrorInvalidValue;
        case 1: return launch_dense_t<1, PROD>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
        case 2: return launch_dense_t<2, PROD>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
        case 3: return launch_dense_t<3, PROD>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
        case 4: return launch_dense_t<4, PROD>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
        default: return (int)cudaErrorInvalidValue;
    }
}

}  // namespace

// True when the dense d = 128 encoder handles this configuration.
bool encode_dense128_supported(const DevState& st, int dtype, int64_t n, int64_t ld) {
    const bool bits_ok = (st.b_mse >= 1 && st.b_mse <= 4) || (st.b_mse == 0 && st.mode == TQ_PROD);
    return st.d == kD && st.rot == TQ_ROT_DENSE && bits_ok && n > 0 && ld >= kD && (dtype == TQ_F32 || dtype == TQ_BF16);
}

int launch_encode_dense128(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, uint8_t* codes,
                           uint8_t* qjl, float* norms, float* rnorms, void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    if (st.mode == TQ_PROD) return launch_dense_b<true>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
    return launch_dense_b<false>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
}

}  // namespace tq
