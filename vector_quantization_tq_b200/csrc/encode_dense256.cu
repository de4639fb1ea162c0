// Encoder for d = 256 with a dense rotation stored fp32 (Haar-random Pi, and S for prod), fp32
// or bf16 input, TurboQuant_mse or TurboQuant_prod with 0- to 4-bit MSE codes.
//
// TurboQuant review (Jump2Paper): Theorem 1 (store ||x||, rotate by Pi, Lloyd-Max cell per
// coordinate of the rotated unit vector), Definition 1 + Theorem 2 (QJL signs of S r, ||r||
// kept). As in the d = 128 tiled encoder, y = Pi x and S r are register-tiled products on the
// CUDA cores; here Pi^T and S^T (256 KiB each in fp32) do not fit in shared memory, so they
// stream through it in chunks of 32 rows (32 KiB), double-buffered with cp.async, one chunk
// ahead of the products:
//   a persistent block of 256 threads walks tiles of 64 vectors; the tile's input is staged
//   coordinate-major; thread t owns the 8 x 8 outputs of vectors 4 (t % 8) .. +3 and
//   32 + 4 (t % 8) .. +3 and coordinates 8 (t / 8) .. +7 (a warp's operand reads are one
//   128-byte run of each row); per k four 16-byte shared loads and 64 FMAs. Quantization,
//   residual and packing follow the d = 128 kernel; the tile's rows are written with 16-byte
//   stores.
#include <cuda_bf16.h>

#include "common.cuh"

namespace tq {

namespace {

constexpr int kD = 256;
constexpr int kT = 64;             // vectors per tile
constexpr int kThreads = 256;
constexpr int kLd = kT + 4;        // row stride (floats) of the transposed tile
constexpr int kKc = 32;            // rows of Pi^T / S^T per streamed chunk
constexpr int kChunks = kD / kKc;  // chunks per matrix

struct Dense256Smem {
    float ring[2][kKc * kD];       // streamed chunks of Pi^T or S^T
    float xt[kD * kLd];            // x tile transposed: xt[k][v]; then the residual r[k][v]
    float nrm[kT];
    float rr[32][kT];              // partial sums of squares: [coordinate group][vector]
    uint8_t rows[kT * 128];        // the tile's packed code rows (32 b bytes each)
    uint8_t zrows[kT * 32];        // the tile's packed sign rows
    float c[16];
    float t[16];
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// y (fp32) -> its cell #{k : t_k <= y} for L = 2^B levels (binary search, upper cell on a tie).
template <int B>
__device__ __forceinline__ int cell256(const float* t, float y) {
    static_assert(B >= 1, "a cell search needs at least two levels");
    int idx = 0;
#pragma unroll
    for (int step = 1 << (B - 1); step >= 1; step >>= 1) idx += (y >= t[idx + step - 1]) ? step : 0;
    return idx;
}

template <int B, bool PROD, bool XF32>
__global__ void __launch_bounds__(kThreads, 1)
encode_dense256_kernel(const DevState st, const void* __restrict__ x, int64_t n, int64_t ld,
                       uint8_t* __restrict__ codes, uint8_t* __restrict__ qjl, float* __restrict__ norms,
                       float* __restrict__ rnorms) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    Dense256Smem& sm = *reinterpret_cast<Dense256Smem*>(smem_raw);
    const int tid = threadIdx.x;
    const int vg = tid & 7, og = tid >> 3;
    auto vec_of = [&](int a) { return (a < 4) ? 4 * vg + a : 32 + 4 * vg + (a - 4); };
    constexpr int kRow = 32 * B;                 // code bytes per vector (none for B = 0)
    constexpr int kMats = PROD ? 2 : 1;          // Pi^T, then S^T
    const float* piT = reinterpret_cast<const float*>(st.piT);
    const float* sT = reinterpret_cast<const float*>(st.sT);

    if (tid < 16) {
        sm.c[tid] = (tid < st.L) ? st.c[tid] : 0.f;
        sm.t[tid] = (tid < st.L - 1) ? st.t[tid] : INFINITY;
    }
    // the chunk stream: per tile, chunks 0..7 of Pi^T (then of S^T); chunk j of the stream goes
    // to ring[j % 2]
    auto load_chunk = [&](int buf, int mat, int q) {
        const float4* src = reinterpret_cast<const float4*>((mat ? sT : piT) + (size_t)q * kKc * kD);
        float4* dst = reinterpret_cast<float4*>(sm.ring[buf]);
        for (int i = tid; i < kKc * kD / 4; i += kThreads) cp_async16(dst + i, src + i);
        cp_async_commit();
    };
    const int64_t ntiles = (n + kT - 1) / kT;
    if ((int64_t)blockIdx.x < ntiles) load_chunk(0, 0, 0);
    int buf = 0;   // ring buffer of the next chunk to use

    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t v0 = tile * kT;
        const bool last_tile = tile + gridDim.x >= ntiles;
        // ---- stage the tile transposed (lane = vector); ||x||^2 from four quarters ----
        {
            const int lane = tid & 31, warp = tid >> 5;
            const int v = 32 * (warp & 1) + lane, k0 = 64 * (warp >> 1);
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
            sm.rr[warp >> 1][v] = ss;
        }
        __syncthreads();
        if (tid < kT) sm.nrm[tid] = sqrtf((sm.rr[0][tid] + sm.rr[1][tid]) + (sm.rr[2][tid] + sm.rr[3][tid]));
#pragma unroll 1
        for (int mat = 0; mat < kMats; ++mat) {
            float acc[8][8];
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
#pragma unroll 1
            for (int q = 0; q < kChunks; ++q) {
                cp_async_wait0();
                __syncthreads();   // chunk q is in ring[buf]; everyone is done with the other buffer
                // the next chunk of the stream (this matrix, the next one, or the next tile's Pi^T)
                if (q + 1 < kChunks) load_chunk(buf ^ 1, mat, q + 1);
                else if (mat + 1 < kMats) load_chunk(buf ^ 1, mat + 1, 0);
                else if (!last_tile) load_chunk(buf ^ 1, 0, 0);
                const float* ch = sm.ring[buf];
#pragma unroll 4
                for (int kk = 0; kk < kKc; ++kk) {
                    const int k = q * kKc + kk;
                    const float4 x0 = *reinterpret_cast<const float4*>(&sm.xt[k * kLd + 4 * vg]);
                    const float4 x1 = *reinterpret_cast<const float4*>(&sm.xt[k * kLd + 32 + 4 * vg]);
                    const float4 p0 = *reinterpret_cast<const float4*>(&ch[kk * kD + 8 * og]);
                    const float4 p1 = *reinterpret_cast<const float4*>(&ch[kk * kD + 8 * og + 4]);
                    const float xa[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    const float pb[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                    for (int a = 0; a < 8; ++a)
#pragma unroll
                        for (int b = 0; b < 8; ++b) acc[a][b] = fmaf(xa[a], pb[b], acc[a][b]);
                }
                buf ^= 1;
            }
            __syncthreads();   // every thread is done with the tile buffer
            if (mat == 0) {
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
                            const int c = cell256<B>(sm.t, y);
                            word |= (uint32_t)c << (B * b);
                            r = (nu > 0.f) ? (y - sm.c[c]) : 0.f;
                        }
                        r2 = fmaf(r, r, r2);
                        if constexpr (PROD) sm.xt[(8 * og + b) * kLd + v] = r;
                    }
#pragma unroll
                    for (int qb = 0; qb < B; ++qb) sm.rows[v * kRow + og * B + qb] = (uint8_t)(word >> (8 * qb));
                    if constexpr (PROD) sm.rr[og][v] = r2;
                }
                __syncthreads();   // the residual is complete before S r reads it
            } else {
                // ---- signs [(S r)_j >= 0] of coordinates 8 og .. +7 ----
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    uint32_t z = 0u;
#pragma unroll
                    for (int b = 0; b < 8; ++b) z |= (acc[a][b] >= 0.f ? 1u : 0u) << b;
                    sm.zrows[vec_of(a) * 32 + og] = (uint8_t)z;
                }
                __syncthreads();
            }
        }
        // ---- write the tile: code rows, sign rows, norms ----
        const int nv = (int)((n - v0) < kT ? (n - v0) : kT);
        if constexpr (B > 0) {
            const uint4* src = reinterpret_cast<const uint4*>(sm.rows);
            uint4* dst = reinterpret_cast<uint4*>(codes + v0 * kRow);
            for (int i = tid; i < nv * kRow / 16; i += kThreads) dst[i] = src[i];
        }
        if constexpr (PROD) {
            const uint4* src = reinterpret_cast<const uint4*>(sm.zrows);
            uint4* dst = reinterpret_cast<uint4*>(qjl + v0 * 32);
            for (int i = tid; i < nv * 2; i += kThreads) dst[i] = src[i];
        }
        if (tid < nv) {
            norms[v0 + tid] = sm.nrm[tid];
            if constexpr (PROD) {
                float s = 0.f;
#pragma unroll 8
                for (int g = 0; g < 32; ++g) s += sm.rr[g][tid];
                rnorms[v0 + tid] = sqrtf(s);
            }
        }
        __syncthreads();   // the buffers are reused by the next tile
    }
    cp_async_wait0();
}

template <int B, bool PROD, bool XF32>
int launch_d256(const DevState& st, const void* x, int64_t n, int64_t ld, uint8_t* codes, uint8_t* qjl,
                float* norms, float* rnorms, cudaStream_t s) {
    auto kern = encode_dense256_kernel<B, PROD, XF32>;
    const size_t smem = sizeof(Dense256Smem);
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
int launch_d256_t(const DevState& st, int dtype, const void* x, int64_t n, int64_t ld, uint8_t* codes, uint8_t* qjl,
                  float* norms, float* rnorms, cudaStream_t s) {
    if (dtype == TQ_F32) return launch_d256<B, PROD, true>(st, x, n, ld, codes, qjl, norms, rnorms, s);
    return launch_d256<B, PROD, false>(st, x, n, ld, codes, qjl, norms, rnorms, s);
}

template <bool PROD>
int launch_d256_b(const DevState& st, int dtype, const void* x, int64_t n, int64_t ld, uint8_t* codes,
                  uint8_t* qjl, float* norms, float* rnorms, cudaStream_t s) {
    switch (st.b_mse) {
        case 0:
            if constexpr (PROD) return launch_d256_t<0, true>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
            return (int)cudaErrorInvalidValue;
        case 1: return launch_d256_t<1, PROD>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
        case 2: return launch_d256_t<2, PROD>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
        case 3: return launch_d256_t<3, PROD>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
        case 4: return launch_d256_t<4, PROD>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
        default: return (int)cudaErrorInvalidValue;
    }
}

}  // namespace

// True when the d = 256 streamed-matrix encoder handles this configuration (fp32 matrices).
bool encode_dense256_supported(const DevState& st, int dtype, int64_t n, int64_t ld) {
    const bool bits_ok = (st.b_mse >= 1 && st.b_mse <= 4) || (st.b_mse == 0 && st.mode == TQ_PROD);
    return st.d == kD && st.rot == TQ_ROT_DENSE && st.mat_dtype == TQ_F32 && bits_ok && n > 0 && ld >= kD &&
           (dtype == TQ_F32 || dtype == TQ_BF16);
}

int launch_encode_dense256(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, uint8_t* codes,
                           uint8_t* qjl, float* norms, float* rnorms, void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    if (st.mode == TQ_PROD) return launch_d256_b<true>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
    return launch_d256_b<false>(st, dtype, x, n, ld, codes, qjl, norms, rnorms, s);
}

}  // namespace tq
