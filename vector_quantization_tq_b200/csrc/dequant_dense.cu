// Dequantization for d = 128 and d = 256 with a dense rotation stored fp32 (Haar-random Pi,
// and S for prod): x~ = ||x|| Pi^T (c[idx] + ||r|| sqrt(pi/2)/d S^T (2z - 1)).
//
// TurboQuant review (Jump2Paper): the inverse maps of Theorem 1 (centroids, then Pi^T, times
// the stored norm) and of Definition 1 / Theorem 2 (sqrt(pi/2)/d ||r|| S^T of the sign vector,
// added in the rotated domain). Both matrix products run over a tile of vectors on the CUDA
// cores, as in the tiled encoders:
//   a persistent block of 256 threads walks tiles of vectors (128 at d = 128, 64 at d = 256);
//   the operand tile is coordinate-major in shared memory (the signs as +-1 for prod, else the
//   centroids); S and Pi stream through shared memory in 32-row chunks, double-buffered with
//   cp.async one chunk ahead of the products; thread t owns the 8 x 8 outputs of 8 vectors and
//   8 coordinates (four 16-byte shared loads and 64 FMAs per row of the matrix). For prod the
//   first product t = S^T (2z - 1) stays in registers; each thread decodes the centroids of its
//   own 8 x 8 block (8 coordinates are b_mse whole bytes of the code row) and writes
//   c[idx] + a t back into the tile for the product with Pi; the rows go out as 32-byte runs.
#include "common.cuh"

namespace tq {

namespace {

constexpr int kThreads = 256;
constexpr int kKc = 32;   // matrix rows per streamed chunk

template <int D>
struct DqCfg {
    static constexpr int kT = (D == 128) ? 128 : 64;   // vectors per tile
    static constexpr int kVG = kT / 8;                   // vector groups (threads along the tile)
    static constexpr int kLd = kT + 4;                   // row stride (floats) of the operand tile
    static constexpr int kChunks = D / kKc;
    static_assert(kVG * (D / 8) == kThreads, "one 8 x 8 block per thread");
};

template <int D>
struct DqSmem {
    float ring[2][kKc * D];              // streamed chunks of S or Pi (row-major rows j, columns k)
    float vt[D * DqCfg<D>::kLd];         // operand tile vt[j][v]
    float c[kMaxLevels];
    float nrm[DqCfg<D>::kT];
    float ar[DqCfg<D>::kT];              // ||r|| sqrt(pi/2) / d
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The 8 codes of coordinates 8 og .. 8 og + 7 of a row: bytes og b .. og b + b - 1 (b <= 8).
__device__ __forceinline__ uint64_t code_bytes8(const uint8_t* row, int og, int b) {
    uint64_t w = 0;
    for (int q = 0; q < b; ++q) w |= (uint64_t)__ldg(row + og * b + q) << (8 * q);
    return w;
}

template <int D, bool PROD>
__global__ void __launch_bounds__(kThreads, 1)
dequant_dense_kernel(const DevState st, const uint8_t* __restrict__ codes, const uint8_t* __restrict__ qjl,
                     const float* __restrict__ norms, const float* __restrict__ rnorms, int64_t n, int64_t ldo,
                     float* __restrict__ out) {
    using Cfg = DqCfg<D>;
    constexpr int kT = Cfg::kT, kLd = Cfg::kLd, kChunks = Cfg::kChunks;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    DqSmem<D>& sm = *reinterpret_cast<DqSmem<D>*>(smem_raw);
    const int tid = threadIdx.x;
    const int vg = tid % Cfg::kVG, og = tid / Cfg::kVG;
    // vectors 4 vg .. +3 and kT/2 + 4 vg .. +3 (a warp's operand reads are one contiguous run of
    // a tile row), coordinates 8 og .. +7
    auto vec_of = [&](int a) { return (a < 4) ? 4 * vg + a : kT / 2 + 4 * vg + (a - 4); };
    const int b = st.b_mse;
    const uint64_t cmask = (b > 0) ? ((1ull << b) - 1ull) : 0ull;
    const float* pi = reinterpret_cast<const float*>(st.pi);
    const float* sm_s = reinterpret_cast<const float*>(st.s);

    for (int i = tid; i < kMaxLevels; i += kThreads) sm.c[i] = (i < st.L) ? st.c[i] : 0.f;
    // the chunk stream: per tile the chunks of S (prod), then those of Pi
    constexpr int kMats = PROD ? 2 : 1;
    auto load_chunk = [&](int buf, int mat, int q) {
        const float* m = (PROD && mat == 0) ? sm_s : pi;
        const float4* src = reinterpret_cast<const float4*>(m + (size_t)q * kKc * D);
        float4* dst = reinterpret_cast<float4*>(sm.ring[buf]);
        for (int i = tid; i < kKc * D / 4; i += kThreads) cp_async16(dst + i, src + i);
        cp_async_commit();
    };
    const int64_t ntiles = (n + kT - 1) / kT;
    load_chunk(0, 0, 0);
    int buf = 0;

    for (int64_t tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
        const int64_t v0 = tile * kT;
        const bool last_tile = tile + gridDim.x >= ntiles;
        if (tid < kT) {
            const bool ok = v0 + tid < n;
            sm.nrm[tid] = ok ? __ldg(norms + v0 + tid) : 0.f;
            if constexpr (PROD) sm.ar[tid] = ok ? __ldg(rnorms + v0 + tid) * st.qjl_scale : 0.f;
        }
        // ---- the first operand tile: +-1 signs (prod) or the centroids (mse) ----
#pragma unroll
        for (int a = 0; a < 8; ++a) {
            const int v = vec_of(a);
            const bool ok = v0 + v < n;
            if constexpr (PROD) {
                const uint32_t z = ok ? __ldg(qjl + (v0 + v) * st.qjl_bytes + og) : 0u;
#pragma unroll
                for (int j = 0; j < 8; ++j) sm.vt[(8 * og + j) * kLd + v] = ((z >> j) & 1u) ? 1.f : -1.f;
            } else {
                const uint64_t w = ok ? code_bytes8(codes + (v0 + v) * st.code_bytes, og, b) : 0ull;
#pragma unroll
                for (int j = 0; j < 8; ++j) sm.vt[(8 * og + j) * kLd + v] = sm.c[(w >> (b * j)) & cmask];
            }
        }
#pragma unroll 1
        for (int mat = 0; mat < kMats; ++mat) {
            float acc[8][8];
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int j = 0; j < 8; ++j) acc[a][j] = 0.f;
#pragma unroll 1
            for (int q = 0; q < kChunks; ++q) {
                cp_async_wait0();
                __syncthreads();   // chunk q is in ring[buf]; the other buffer and the tile are settled
                if (q + 1 < kChunks) load_chunk(buf ^ 1, mat, q + 1);
                else if (mat + 1 < kMats) load_chunk(buf ^ 1, mat + 1, 0);
                else if (!last_tile) load_chunk(buf ^ 1, 0, 0);
                const float* ch = sm.ring[buf];
#pragma unroll 4
                for (int kk = 0; kk < kKc; ++kk) {
                    const int k = q * kKc + kk;
                    const float4 x0 = *reinterpret_cast<const float4*>(&sm.vt[k * kLd + 4 * vg]);
                    const float4 x1 = *reinterpret_cast<const float4*>(&sm.vt[k * kLd + kT / 2 + 4 * vg]);
                    const float4 p0 = *reinterpret_cast<const float4*>(&ch[kk * D + 8 * og]);
                    const float4 p1 = *reinterpret_cast<const float4*>(&ch[kk * D + 8 * og + 4]);
                    const float xa[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    const float pb[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
                    for (int a = 0; a < 8; ++a)
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[a][j] = fmaf(xa[a], pb[j], acc[a][j]);
                }
                buf ^= 1;
            }
            if (PROD && mat == 0) {
                // ---- y = c[idx] + a t: this thread's block back into the tile for Pi^T ----
                __syncthreads();   // every thread is done reading the signs
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    const int v = vec_of(a);
                    const bool ok = v0 + v < n;
                    const uint64_t w = (ok && b > 0) ? code_bytes8(codes + (v0 + v) * st.code_bytes, og, b) : 0ull;
                    const float ar = sm.ar[v];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float cj = (b > 0) ? sm.c[(w >> (b * j)) & cmask] : 0.f;
                        sm.vt[(8 * og + j) * kLd + v] = fmaf(ar, acc[a][j], cj);
                    }
                }
            } else {
                // ---- x~ = ||x|| Pi^T y: 32 bytes per vector ----
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    const int v = vec_of(a);
                    if (v0 + v < n) {
                        const float nu = sm.nrm[v];
                        float4* o = reinterpret_cast<float4*>(out + (v0 + v) * ldo + 8 * og);
                        o[0] = make_float4(nu * acc[a][0], nu * acc[a][1], nu * acc[a][2], nu * acc[a][3]);
                        o[1] = make_float4(nu * acc[a][4], nu * acc[a][5], nu * acc[a][6], nu * acc[a][7]);
                    }
                }
            }
        }
        __syncthreads();   // the tile and the per-vector scalars are rewritten by the next tile
    }
    cp_async_wait0();
}

template <int D, bool PROD>
int launch_dq(const DevState& st, const uint8_t* codes, const uint8_t* qjl, const float* norms, const float* rnorms,
              int64_t n, int64_t ldo, float* out, cudaStream_t s) {
    auto kern = dequant_dense_kernel<D, PROD>;
    const size_t smem = sizeof(DqSmem<D>);
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
    const int64_t ntiles = (n + DqCfg<D>::kT - 1) / DqCfg<D>::kT;
    const int grid = (int)std::min<int64_t>(ntiles, (int64_t)(sms > 0 ? sms : 148));
    kern<<<grid, kThreads, smem, s>>>(st, codes, qjl, norms, rnorms, n, ldo, out);
    return (int)cudaGetLastError();
}

}  // namespace

// True when the tiled dequantizer handles this configuration (dense fp32 matrices, d = 128 or
// 256, whole output rows with 16-byte aligned starts).
bool dequant_dense_supported(const DevState& st, int64_t n, const int32_t* chan, int64_t ldo) {
    return (st.d == 128 || st.d == 256) && st.rot == TQ_ROT_DENSE && st.mat_dtype == TQ_F32 && chan == nullptr &&
           n > 0 && ldo >= st.d && ldo % 4 == 0 && st.b_mse >= 0 && st.b_mse <= 8;
}

int launch_dequant_dense(const DevState& st, const uint8_t* codes, const uint8_t* qjl, const float* norms,
                         const float* rnorms, int64_t n, int64_t ldo, float* out, void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    const bool prod = qjl != nullptr;
    if (st.d == 128) return prod ? launch_dq<128, true>(st, codes, qjl, norms, rnorms, n, ldo, out, s)
                                 : launch_dq<128, false>(st, codes, qjl, norms, rnorms, n, ldo, out, s);
    return prod ? launch_dq<256, true>(st, codes, qjl, norms, rnorms, n, ldo, out, s)
                : launch_dq<256, false>(st, codes, qjl, norms, rnorms, n, ldo, out, s);
}

}  // namespace tq
