// Distortion and inner-product error statistics of reconstructions (the distortion / bias
// sweep): D_mse = E||x - x~||^2 (Jump2Paper review, Theorem 1) and the inner-product error
// e = <q, x~> - <q, x> over query/vector pairs, whose mean is 0 for TurboQuant_prod
// (Theorem 2) and whose slope <q,x><q,x~> / <q,x>^2 is 1 - D_mse for TurboQuant_mse
// (the 2/pi bias at b = 1).
//
// A block stages 32 vectors (x and x~) and 64 queries at a time in shared memory (rows
// padded by one float, so the per-vector reads hit distinct banks); each thread owns one
// vector and 8 queries and accumulates both dot products in fp32, then the pair sums in
// fp64. Block sums go to the output with fp64 atomics (sums of many terms; order varies).
#include "common.cuh"

namespace tq {
namespace {

constexpr int kVB = 32;     // vectors per block tile
constexpr int kQC = 64;     // queries per chunk
constexpr int kThreads = 256;

__device__ __forceinline__ double block_sum_d(double v, double* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    double s = 0.0;
    if (threadIdx.x == 0)
        for (int i = 0; i < kThreads / 32; ++i) s += red[i];
    return s;
}

__global__ void __launch_bounds__(kThreads)
ip_stats_kernel(const float* __restrict__ x, const float* __restrict__ xt, int64_t n, int d,
                const float* __restrict__ q, int64_t nq, double* __restrict__ out) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int ld = d + 1;
    float* xs = reinterpret_cast<float*>(smem_raw);   // kVB x ld
    float* ts = xs + kVB * ld;                          // kVB x ld
    float* qs = ts + kVB * ld;                          // kQC x ld
    double* red = reinterpret_cast<double*>(qs + kQC * ld + 1);
    red = reinterpret_cast<double*>((reinterpret_cast<uintptr_t>(red) + 7) & ~uintptr_t(7));
    const int64_t v0 = (int64_t)blockIdx.x * kVB;
    const int nv = (int)((n - v0) < kVB ? (n - v0) : kVB);
    for (int i = threadIdx.x; i < kVB * d; i += kThreads) {
        const int v = i / d, j = i - v * d;
        xs[v * ld + j] = (v < nv) ? x[(v0 + v) * d + j] : 0.f;
        ts[v * ld + j] = (v < nv) ? xt[(v0 + v) * d + j] : 0.f;
    }
    const int v = threadIdx.x & 31;
    const int qg = threadIdx.x >> 5;   // 8 groups of 8 queries
    double s_e = 0.0, s_e2 = 0.0, s_ab = 0.0, s_a2 = 0.0;
    for (int64_t q0 = 0; q0 < nq; q0 += kQC) {
        const int nqc = (int)((nq - q0) < kQC ? (nq - q0) : kQC);
        __syncthreads();
        for (int i = threadIdx.x; i < kQC * d; i += kThreads) {
            const int r = i / d, j = i - r * d;
            qs[r * ld + j] = (r < nqc) ? q[(q0 + r) * d + j] : 0.f;
        }
        __syncthreads();
        float a[8], b[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = b[i] = 0.f;
        for (int j = 0; j < d; ++j) {
            const float xv = xs[v * ld + j], tv = ts[v * ld + j];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float qv = qs[(qg * 8 + i) * ld + j];
                a[i] = fmaf(qv, xv, a[i]);
                b[i] = fmaf(qv, tv, b[i]);
            }
        }
        if (v < nv) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                if (qg * 8 + i < nqc) {
                    const double e = (double)b[i] - (double)a[i];
                    s_e += e;
                    s_e2 += e * e;
                    s_ab += (double)a[i] * (double)b[i];
                    s_a2 += (double)a[i] * (double)a[i];
                }
            }
        }
    }
    double s_d = 0.0, s_x = 0.0;
    if (qg == 0 && v < nv) {
        for (int j = 0; j < d; ++j) {
            const double dx = (double)xs[v * ld + j] - (double)ts[v * ld + j];
            s_d += dx * dx;
            s_x += (double)xs[v * ld + j] * (double)xs[v * ld + j];
        }
    }
    const double sums[6] = {s_d, s_x, s_e, s_e2, s_ab, s_a2};
#pragma unroll
    for (int k = 0; k < 6; ++k) {
        const double t = block_sum_d(sums[k], red);
        if (threadIdx.x == 0) atomicAdd(out + k, t);
    }
}

}  // namespace

int launch_ip_stats(const float* x, const float* xt, int64_t n, int d, const float* q, int64_t nq, double* out,
                    void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(out, 0, 6 * sizeof(double), s);
    if (e != cudaSuccess) return (int)e;
    if (n == 0) return 0;
    const size_t smem = (size_t)(2 * kVB + kQC) * (d + 1) * sizeof(float) + 16 + (kThreads / 32) * sizeof(double);
    if (smem > 48 * 1024) {
        e = cudaFuncSetAttribute(ip_stats_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return (int)e;
    }
    const int64_t blocks = (n + kVB - 1) / kVB;
    if (blocks > (1ll << 31) - 1) return (int)cudaErrorInvalidConfiguration;
    ip_stats_kernel<<<(unsigned)blocks, kThreads, smem, s>>>(x, xt, n, d, q, nq, out);
    return (int)cudaGetLastError();
}

}  // namespace tq
