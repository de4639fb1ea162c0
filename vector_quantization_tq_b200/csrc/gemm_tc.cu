// Dense projections on the tensor core for large d (TurboQuant with a dense Haar rotation
// and a dense QJL matrix; Jump2Paper review: Pi and S are d x d, and the rotation is a
// plain matrix product). Used for d >= 512 with bf16-stored Pi and S and bf16 input.
//
// C[M x N] = A[M x K] * B[N x K]^T, A and B bf16 K-major in global memory, fp32 accumulate.
// Persistent CTA (one per SM) of 10 warps walking 128 x BN output tiles (N tile fastest, so
// the CTAs that share an A tile run together and A comes from DRAM once):
//   warp 0  TMA producer: K-steps of 64 through a shared-memory ring, continuing into the next
//           tile without draining;
//   warp 1  MMA issuer: 4 x tcgen05.mma (M128 N=BN K16) per stage into one of two TMEM
//           accumulators (tiles alternate), commit frees the stage;
//   warps 2-9 epilogue: two warps per TMEM lane quadrant, each thread one output row and half
//           of the tile's columns, 32 at a time, while the MMAs of the next tile run into the
//           other accumulator.
// Epilogues:
//   kStoreF32  C in fp32 (query preparation).
//   kRotate    y = acc / ||x||, b-bit Lloyd-Max cell, residual r = y - c[idx] written as a
//              bf16 pair (hi, lo = bf16(r - hi)) for the next product, partial ||r||^2.
//   kSigns     QJL bits [acc >= 0] of S r, and ||r|| from the partials.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace tq {

namespace {
__device__ int g_tq_device_error = 0;
}  // namespace

namespace {

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kGemmThreads = 320;

enum EpiKind { kStoreF32 = 0, kRotate = 1, kSigns = 2 };

// Ring depth 4 (the TMA latency from L2 is about three steps' MMAs); the quantize epilogue
// keeps 4 KB per warp of staging for its residual stores.
template <int EPI>
struct GemmCfg {
    static constexpr int kStages = 4;
    static constexpr int kStageBytes = (EPI == kRotate) ? 8 * 4096 : 16;
};

struct GemmParams {
    int M, N, K;
    int b_kwrap;              // B's K coordinate is taken modulo b_kwrap (B reused along K)
    // kStoreF32
    float* c;
    int ldc;
    // kRotate / kSigns
    const float* norms;       // ||x|| per row
    uint8_t* codes;           // [M][code_bytes]
    int code_bytes;
    int b_mse;
    uint16_t* r2;             // [M][2N] bf16 bits: hi in [0, N), lo in [N, 2N)
    float* rho_part;          // [M][N / BN]
    int n_tiles;
    uint8_t* qjl;             // [M][N/8]
    float* rnorms;
    float t[16];
    float c_cent[16];
};

template <int BN, int EPI>
struct __align__(1024) GemmSmem {
    uint8_t a[GemmCfg<EPI>::kStages][kBM * kBK * 2];
    uint8_t b[GemmCfg<EPI>::kStages][BN * kBK * 2];
    uint8_t stage[GemmCfg<EPI>::kStageBytes];   // kRotate: 4 KB of residual staging per epilogue warp
    uint64_t full[GemmCfg<EPI>::kStages];
    uint64_t empty[GemmCfg<EPI>::kStages];
    uint64_t acc_full[2];      // the tile's MMAs are done (commit)
    uint64_t acc_empty[2];     // the epilogue has read the accumulator (one arrival per warp)
    float rr_half[2][kBM];     // the second column half's partial ||r||^2 per row, by tile parity
    uint32_t tmem_base;
    int abort;
};

// Barrier over the eight epilogue warps (named barrier 2) that returns the OR of `pred`.
__device__ __forceinline__ bool epi_sync_or(bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "barrier.cta.red.or.pred po, 2, 256, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred)
        : "memory");
    return r != 0;
}

// BQ: code width of the kRotate epilogue (compile-time, so the code words stay in registers).
template <int BN, int EPI, int BQ>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tma_a, const __grid_constant__ CUtensorMap tma_b,
               const GemmParams p) {
    using Cfg = GemmCfg<EPI>;
    constexpr int kStages = Cfg::kStages;
    extern __shared__ uint8_t smem_raw[];
    GemmSmem<BN, EPI>& sm = *reinterpret_cast<GemmSmem<BN, EPI>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                                ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntn = p.N / BN;
    const int64_t ntiles = (int64_t)((p.M + kBM - 1) / kBM) * ntn;
    const int ksteps = p.K / kBK;
    constexpr uint32_t kCols = 2 * BN;      // two accumulators
    static_assert(BN % 64 == 0 && 2 * BN <= 512, "two accumulators of BN columns; whole chunks per column half");

    if (threadIdx.x == 0) {
        ptx::prefetch_tmap(&tma_a);
        ptx::prefetch_tmap(&tma_b);
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&sm.full[s], 1);
            ptx::mbar_init(&sm.empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&sm.acc_full[a], 1);
            ptx::mbar_init(&sm.acc_empty[a], 8);   // one arrival per epilogue warp
        }
        sm.abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(&sm.tmem_base, kCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ---- TMA producer: the K steps of every tile of this CTA, one ring position each ----
        if (lane == 0) {
            int64_t g = 0;
            for (int64_t t = blockIdx.x; t < ntiles && !sm.abort; t += gridDim.x) {
                const int m0 = (int)(t / ntn) * kBM, n0 = (int)(t % ntn) * BN;
                for (int ks = 0; ks < ksteps; ++ks, ++g) {
                    const int s = (int)(g % kStages);
                    if (g >= kStages && !ptx::mbar_wait(&sm.empty[s], (uint32_t)(((g / kStages) - 1) & 1))) {
                        atomicExch(&sm.abort, 1);
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(&sm.full[s], (kBM + BN) * kBK * 2);
                    ptx::tma_load_2d(sm.a[s], &tma_a, ks * kBK, m0, &sm.full[s]);
                    ptx::tma_load_2d(sm.b[s], &tma_b, (ks * kBK) % p.b_kwrap, n0, &sm.full[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ---- MMA issue: tile i accumulates into columns [BN (i % 2), BN (i % 2) + BN) ----
        if (lane == 0) {
            const uint32_t idesc = ptx::idesc_bf16_f32(kBM, BN);
            int64_t g = 0, i = 0;
            for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
                const int acc = (int)(i & 1);
                if (i >= 2 && !ptx::mbar_wait(&sm.acc_empty[acc], (uint32_t)(((i >> 1) - 1) & 1)))
                    atomicExch(&sm.abort, 1);
                if (sm.abort) break;
                ptx::tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
                for (int ks = 0; ks < ksteps; ++ks, ++g) {
                    const int s = (int)(g % kStages);
                    if (!ptx::mbar_wait(&sm.full[s], (uint32_t)((g / kStages) & 1))) {
                        atomicExch(&sm.abort, 1);
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_addr(sm.a[s]);
                    const uint32_t b_addr = ptx::smem_addr(sm.b[s]);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        ptx::mma_ss(d_tmem, ptx::smem_desc_kmajor_sw128(a_addr + kk * 32),
                                    ptx::smem_desc_kmajor_sw128(b_addr + kk * 32), idesc, (ks | kk) ? 1u : 0u);
                    ptx::mma_commit(&sm.empty[s]);
                }
                if (sm.abort) break;
                ptx::mma_commit(&sm.acc_full[acc]);   // arrives once every MMA above has completed
            }
        }
    } else {
        // ---- epilogue: warps 2..9; lane quadrant warp % 4, column half (warp - 2) / 4 ----
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;
        const int row = quad * 32 + lane;
        const uint32_t t_quad = tmem + ((uint32_t)(quad * 32) << 16);
        int64_t i = 0;
        bool failed = false;
        for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
            const int acc_i = (int)(i & 1);
            const int m0 = (int)(t / ntn) * kBM, nt = (int)(t % ntn), n0 = nt * BN;
            const int m = m0 + row;
            bool ok = true;
            if (lane == 0) ok = ptx::mbar_wait(&sm.acc_full[acc_i], (uint32_t)((i >> 1) & 1));
            // the eight epilogue warps stop together (they meet at a named barrier per tile)
            if (epi_sync_or(!ok || sm.abort)) {
                failed = true;
                break;
            }
            ptx::tc_fence_after();
            const uint32_t t_lane = t_quad + (uint32_t)(acc_i * BN);
            float inv_nu = 0.f;
            if constexpr (EPI == kRotate) {
                const float nu = (m < p.M) ? __ldg(p.norms + m) : 0.f;
                inv_nu = (nu > 0.f) ? 1.f / nu : 0.f;
            }
            float rr = 0.f;
#pragma unroll 1
            for (int c = half * (BN / 64); c < (half + 1) * (BN / 64); ++c) {
                uint32_t acc[32];
                ptx::tmem_ld32(t_lane + c * 32, acc);
                ptx::tmem_wait_ld();
                if (EPI != kRotate && m >= p.M) continue;   // the quantize pass stages every row
                const int ncol = n0 + c * 32;
                if constexpr (EPI == kStoreF32) {
                    float4* dst = reinterpret_cast<float4*>(p.c + (size_t)m * p.ldc + ncol);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        dst[j] = make_float4(__uint_as_float(acc[4 * j]), __uint_as_float(acc[4 * j + 1]),
                                             __uint_as_float(acc[4 * j + 2]), __uint_as_float(acc[4 * j + 3]));
                } else if constexpr (EPI == kRotate) {
                    constexpr int b = BQ;
                    uint32_t cw[4] = {0u, 0u, 0u, 0u};   // 32 codes of b <= 4 bits
                    uint32_t hi[16], lo[16];
#pragma unroll
                    for (int j = 0; j < 32; j += 2) {
                        float r2[2];
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const float y = __uint_as_float(acc[j + e]) * inv_nu;
                            uint32_t code = 0;
                            float cv = p.c_cent[0];
                            for (int k = 0; k < (1 << b) - 1; ++k)
                                if (y >= p.t[k]) {
                                    code = k + 1;
                                    cv = p.c_cent[k + 1];
                                }
                            const int bit = (j + e) * b;
                            cw[bit >> 5] |= code << (bit & 31);
                            if ((bit & 31) + b > 32) cw[(bit >> 5) + 1] |= code >> (32 - (bit & 31));
                            r2[e] = (inv_nu > 0.f) ? y - cv : 0.f;
                            rr = fmaf(r2[e], r2[e], rr);
                        }
                        const __nv_bfloat162 h = __float22bfloat162_rn(make_float2(r2[0], r2[1]));
                        const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h);
                        const float l0 = r2[0] - __uint_as_float(hb << 16);
                        const float l1 = r2[1] - __uint_as_float(hb & 0xffff0000u);
                        const __nv_bfloat162 l = __float22bfloat162_rn(make_float2(l0, l1));
                        hi[j >> 1] = hb;
                        lo[j >> 1] = *reinterpret_cast<const uint32_t*>(&l);
                    }
                    // The chunk's residual (64 bytes of hi and of lo per row) is staged in this
                    // warp's 4 KB, each row's 16-byte slots rotated by (row / 2) % 4 so that a
                    // quarter-warp's writes fall into different banks; the warp then stores
                    // 64-byte row pieces (two whole sectors), eight rows per instruction, instead
                    // of 16 bytes per row.
                    uint8_t* stg = sm.stage + (warp - 2) * 4096;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int slot = (j ^ ((lane >> 1) & 3)) * 16;
                        *reinterpret_cast<uint4*>(stg + lane * 64 + slot) =
                            make_uint4(hi[4 * j], hi[4 * j + 1], hi[4 * j + 2], hi[4 * j + 3]);
                        *reinterpret_cast<uint4*>(stg + 2048 + lane * 64 + slot) =
                            make_uint4(lo[4 * j], lo[4 * j + 1], lo[4 * j + 2], lo[4 * j + 3]);
                    }
                    __syncwarp();
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int r8 = 8 * k + (lane >> 2), sl = lane & 3;   // row of the warp, 16-byte slot
                        const int64_t mr = m0 + quad * 32 + r8;
                        const int off = r8 * 64 + ((sl ^ ((r8 >> 1) & 3)) * 16);
                        const uint4 vh = *reinterpret_cast<const uint4*>(stg + off);
                        const uint4 vl = *reinterpret_cast<const uint4*>(stg + 2048 + off);
                        if (mr < p.M) {
                            uint16_t* rowp = p.r2 + (size_t)mr * 2 * p.N;
                            *reinterpret_cast<uint4*>(rowp + ncol + sl * 8) = vh;
                            *reinterpret_cast<uint4*>(rowp + p.N + ncol + sl * 8) = vl;
                        }
                    }
                    __syncwarp();   // the staging area is rewritten by the next chunk
                    if (m < p.M) {
                        uint32_t* cdst = reinterpret_cast<uint32_t*>(p.codes + (size_t)m * p.code_bytes) + (ncol / 32) * b;
                        for (int w = 0; w < b; ++w) cdst[w] = cw[w];
                    }
                } else {   // kSigns
                    uint32_t neg = 0u;
#pragma unroll
                    for (int j = 31; j >= 0; --j) neg = __funnelshift_l(acc[j], neg, 1);
                    // (S r)_j >= 0 -> 1; a zero residual gives +-0 products: treat as >= 0
                    uint32_t z = ~neg;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (acc[j] == 0x80000000u) z |= 1u << j;
                    reinterpret_cast<uint32_t*>(p.qjl + (size_t)m * (p.N / 8))[ncol / 32] = z;
                }
            }
            // the accumulator is free for tile i + 2 once every epilogue warp has read it
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0)
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(ptx::smem_addr(&sm.acc_empty[acc_i]))
                             : "memory");
            if constexpr (EPI == kSigns) {
                if (half == 0 && nt == 0 && m < p.M) {
                    float sq = 0.f;
                    for (int k = 0; k < p.n_tiles; ++k) sq += p.rho_part[(size_t)m * p.n_tiles + k];
                    p.rnorms[m] = sqrtf(sq);
                }
            }
            if constexpr (EPI == kRotate) {
                // the row's partial ||r||^2 over this N tile: both column halves (the buffer
                // alternates with the tile, so one barrier per tile orders its writes and reads)
                if (half == 1) sm.rr_half[acc_i][row] = rr;
                asm volatile("bar.sync 1, 256;" ::: "memory");   // the eight epilogue warps
                if (half == 0 && m < p.M) p.rho_part[(size_t)m * p.n_tiles + nt] = rr + sm.rr_half[acc_i][row];
            }
        }
        if (failed && lane == 0) atomicExch(&g_tq_device_error, 1);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kCols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

// 2-D bf16 tensor map over [rows][cols] (row stride ld elements), box 64 x box_rows, 128B swizzle.
int make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
    EncodeTiledFn enc = tiled_fn();
    if (!enc) return (int)cudaErrorNotSupported;
    const cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? 0 : (int)cudaErrorInvalidValue;
}

template <int BN, int EPI, int BQ = 0>
int run_gemm(const void* A, int64_t lda, const void* B, int64_t ldb, const GemmParams& p, cudaStream_t s) {
    if (p.K % kBK != 0 || p.N % BN != 0) return (int)cudaErrorInvalidValue;
    CUtensorMap ta, tb;
    int e = make_map(&ta, A, p.M, p.K, lda, kBM);
    if (e) return e;
    e = make_map(&tb, B, p.N, p.K, ldb, BN);
    if (e) return e;
    auto kern = gemm_tc_kernel<BN, EPI, BQ>;
    const size_t smem = sizeof(GemmSmem<BN, EPI>) + 1024;
    static int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t ce = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (ce != cudaSuccess) return (int)ce;
        attr_dev = dev;
    }
    const int64_t ntiles = (int64_t)((p.M + kBM - 1) / kBM) * (p.N / BN);
    int sms = 0;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = (int)std::min<int64_t>(ntiles, (int64_t)(sms > 0 ? sms : 148));
    kern<<<grid, kGemmThreads, smem, s>>>(ta, tb, p);
    return (int)cudaGetLastError();
}

// ||x|| of bf16 rows (d elements, row stride ld), one warp per row.
__global__ void __launch_bounds__(256) row_norms_bf16(const uint16_t* __restrict__ x, int64_t n, int d, int64_t ld,
                                                      float* __restrict__ out) {
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= n) return;
    const uint16_t* r = x + row * ld;
    float s = 0.f;
    for (int j = (threadIdx.x & 31) * 8; j < d; j += 256) {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(r + j));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float a = __uint_as_float(w[k] << 16), b = __uint_as_float(w[k] & 0xffff0000u);
            s = fmaf(a, a, s);
            s = fmaf(b, b, s);
        }
    }
    s = warp_sum(s);
    if ((threadIdx.x & 31) == 0) out[row] = sqrtf(s);
}

}  // namespace

// True when the dense tensor-core encoder handles this configuration.
bool encode_gemm_supported(const DevState& st, int dtype, int64_t n, int64_t ld) {
    return st.rot == TQ_ROT_DENSE && st.mat_dtype == TQ_BF16 && dtype == TQ_BF16 && st.d >= 512 &&
           st.d % 256 == 0 && st.b_mse >= 1 && st.b_mse <= 4 && n > 0 && n < ((int64_t)1 << 31) && ld >= st.d;
}

// Prod encode with the randomized Hadamard rotation at d >= 512 (bf16 S and input): the
// rotation, codes and residual run on the CUDA cores (general encoder writing [r_hi | r_lo]
// and ||r||^2), S r and its signs on the tensor core (the kSigns pass below).
bool encode_rht_gemm_supported(const DevState& st, int dtype, int64_t n, int64_t ld) {
    return st.rot == TQ_ROT_RHT && st.mode == TQ_PROD && st.mat_dtype == TQ_BF16 && dtype == TQ_BF16 &&
           st.d >= 512 && st.d % 256 == 0 && st.b_mse <= 4 && n > 0 && n < ((int64_t)1 << 31) && ld >= st.d;
}

// Signs of S r and ||r|| from the residual workspace (r2, rho_part) of n vectors.
int launch_signs_gemm(const DevState& st, int64_t n, uint8_t* qjl, float* rnorms, void* ws, void* stream) {
    const int d = st.d;
    GemmParams p = {};
    p.M = (int)n;
    p.N = d;
    p.K = 2 * d;
    p.b_kwrap = d;
    p.rho_part = reinterpret_cast<float*>(reinterpret_cast<uint16_t*>(ws) + (size_t)n * 2 * d);
    p.n_tiles = d / 256;
    p.qjl = qjl;
    p.rnorms = rnorms;
    return run_gemm<256, kSigns>(ws, 2 * d, st.s, d, p, (cudaStream_t)stream);
}

// Dense tensor-core encode: ||x||, y = Pi x / ||x|| (codes + residual), then signs of S r.
// Workspace: R = [r_hi | r_lo] bf16 [n][2d] and partial ||r||^2 [n][d/256].
size_t encode_gemm_ws_bytes(int d, int64_t n) {
    const size_t per = (size_t)d * 4 + 4 * (size_t)(d / 256);
    return ((size_t)n * per + 1023) & ~(size_t)1023;
}

int launch_encode_gemm(const DevState& st, const void* x, int64_t n, int64_t ld, uint8_t* codes, uint8_t* qjl,
                       float* norms, float* rnorms, void* ws, void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    const int d = st.d;
    uint16_t* r2 = reinterpret_cast<uint16_t*>(ws);
    float* rho_part = reinterpret_cast<float*>(r2 + (size_t)n * 2 * d);
    row_norms_bf16<<<(unsigned)((n + 7) / 8), 256, 0, s>>>(reinterpret_cast<const uint16_t*>(x), n, d, ld, norms);
    int e = (int)cudaGetLastError();
    if (e) return e;
    GemmParams p = {};
    p.M = (int)n;
    p.N = d;
    p.K = d;
    p.b_kwrap = d;
    p.norms = norms;
    p.codes = codes;
    p.code_bytes = st.code_bytes;
    p.b_mse = st.b_mse;
    p.r2 = r2;
    p.rho_part = rho_part;
    p.n_tiles = d / 256;
    p.qjl = qjl;
    p.rnorms = rnorms;
    for (int i = 0; i < 16; ++i) {
        p.t[i] = (i < st.L - 1) ? st.t[i] : 0.f;
        p.c_cent[i] = (i < st.L) ? st.c[i] : 0.f;
    }
    // y = X Pi^T: B = Pi, row-major [out][in], i.e. K-major in `in`.
    switch (st.b_mse) {
        case 1: e = run_gemm<256, kRotate, 1>(x, ld, st.pi, d, p, s); break;
        case 2: e = run_gemm<256, kRotate, 2>(x, ld, st.pi, d, p, s); break;
        case 3: e = run_gemm<256, kRotate, 3>(x, ld, st.pi, d, p, s); break;
        default: e = run_gemm<256, kRotate, 4>(x, ld, st.pi, d, p, s); break;
    }
    if (e || st.mode != TQ_PROD) return e;
    // S r over K = 2d: A = [r_hi | r_lo], B = S reused for both halves of K.
    p.K = 2 * d;
    e = run_gemm<256, kSigns>(r2, 2 * d, st.s, d, p, s);
    return e;
}

// C = A B^T in fp32 for small M (query preparation): A [M][K], B [N][K] bf16.
int launch_gemm_f32(const void* A, int64_t lda, const void* B, int64_t ldb, int M, int N, int K, int b_kwrap,
                    float* C, int ldc, void* stream) {
    GemmParams p = {};
    p.M = M;
    p.N = N;
    p.K = K;
    p.b_kwrap = b_kwrap;
    p.c = C;
    p.ldc = ldc;
    return run_gemm<256, kStoreF32>(A, lda, B, ldb, p, (cudaStream_t)stream);
}

int take_device_error_gemm(int* flag) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_tq_device_error, sizeof(int));
    if (e != cudaSuccess) return (int)e;
    if (v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_tq_device_error, &zero, sizeof(int));
        if (e != cudaSuccess) return (int)e;
    }
    *flag = v;
    return 0;
}

}  // namespace tq
