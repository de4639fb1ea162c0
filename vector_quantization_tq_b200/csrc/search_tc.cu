// Top-k search over 1-bit TurboQuant_prod codes (b = 2: 1-bit MSE + 1-bit QJL) on the
// tensor core (Jump2Paper review: nearest-neighbour search by the unbiased inner-product
// estimate). With a 2-level symmetric codebook c[idx] = +-c1 the estimate is
//     est(q, x) = ||x|| ( c1 <q', sigma> + ||r|| sqrt(pi/2)/d <u, s> ),   q' = Pi q, u = S q',
// with sigma, s in {-1, +1}^d the two bit planes: two dot products with +-1 vectors, i.e. a
// GEMM of the queries [q' | u] (bf16, nq x 2d) against the keys' planes expanded to +-1.
//
// CTA: 128 queries x a run of key tiles of 256. Warp roles:
//   warp 0      TMA producer of the query tile (K-steps of 64 through a 3-stage ring);
//   warp 1      MMA issuer: K-steps of the first d coordinates accumulate <q', sigma> in TMEM
//               columns [0, 256), the next d accumulate <u, s> in [256, 512);
//   warps 2-9   epilogue: two threads per query (keys 0-127 and 128-255 of a tile), est for
//               their keys, a running top-16 each in registers (both lists go to the merge);
//   warps 10-17 expanders: each K-step's 64 bits per key become 64 bf16 +-1 values in shared
//               memory (arithmetic: one multiply and one logic op per pair of values), one key
//               per thread, with the key bits fetched a few steps ahead.
// Each CTA writes its k best (value, index) per query; a merge launch picks the final k.
#include <cuda.h>
#include <cuda_bf16.h>

#include <climits>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace tq {

namespace {
__device__ int g_tq_device_error = 0;
}  // namespace

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kStages = 3;
constexpr int kThreads = 576;   // 18 warps: TMA, MMA, 8 epilogue, 8 expanders
constexpr int kTopMax = 16;
constexpr int kCand = 32;   // candidates an epilogue thread buffers before merging them into its top list
constexpr int kEpiWarp0 = 2, kExpWarp0 = 10;

struct SearchParams {
    int nq;
    int64_t n;
    int d;
    int k;
    int tiles_per_cta;
    const uint8_t* codes;     // [n][d/8], 1 bit per coordinate
    const uint8_t* qjl;       // [n][d/8]
    const float* norms;
    const float* rnorms;
    float c1;
    float qjl_scale;
    float* cand_v;            // [nq][gridDim.y][k]
    int64_t* cand_i;
};

struct __align__(1024) SearchSmem {
    uint8_t a[kStages][kBM * kBK * 2];   // queries, 128B-swizzled (TMA)
    uint8_t b[kStages][kBN * kBK * 2];   // keys as +-1, K-major core matrices
    float nu[kBN];
    float g2[kBN];
    float candv[kCand][2 * kBM];         // per epilogue thread (column): estimates above its threshold
    int candi[kCand][2 * kBM];           // and their keys
    uint64_t afull[kStages];
    uint64_t bfull[kStages];
    uint64_t empty[kStages];
    uint64_t done;
    uint64_t tfree;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ void named_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// Barrier over `n` threads that also returns the OR of `pred` across them (uniform result).
__device__ __forceinline__ bool named_sync_or(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "barrier.cta.red.or.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__global__ void __launch_bounds__(kThreads, 1)
search_tc_kernel(const __grid_constant__ CUtensorMap tma_q, const SearchParams p) {
    extern __shared__ uint8_t smem_raw[];
    SearchSmem& sm = *reinterpret_cast<SearchSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kBM;
    const int64_t ntile_total = (p.n + kBN - 1) / kBN;
    const int64_t tile_begin = (int64_t)blockIdx.y * p.tiles_per_cta;
    const int64_t tile_end = (tile_begin + p.tiles_per_cta < ntile_total) ? tile_begin + p.tiles_per_cta : ntile_total;
    const int ks_per_tile = 2 * p.d / kBK;
    const int ks_half = p.d / kBK;

    if (threadIdx.x == 0) {
        ptx::prefetch_tmap(&tma_q);
        for (int s = 0; s < kStages; ++s) {
            ptx::mbar_init(&sm.afull[s], 1);
            ptx::mbar_init(&sm.bfull[s], 8);   // one arrival per expander warp
            ptx::mbar_init(&sm.empty[s], 1);
        }
        ptx::mbar_init(&sm.done, 1);
        ptx::mbar_init(&sm.tfree, 1);
        sm.abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(&sm.tmem_base, 512);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ---- query tiles by TMA ----
        if (lane == 0) {
            int64_t g = 0;
            for (int64_t t = tile_begin; t < tile_end && !sm.abort; ++t) {
                for (int ks = 0; ks < ks_per_tile; ++ks, ++g) {
                    const int s = (int)(g % kStages);
                    const int64_t r = g / kStages;
                    if (r > 0 && !ptx::mbar_wait(&sm.empty[s], (uint32_t)((r - 1) & 1))) {
                        atomicExch(&sm.abort, 1);
                        break;
                    }
                    ptx::mbar_arrive_expect_tx(&sm.afull[s], kBM * kBK * 2);
                    ptx::tma_load_2d(sm.a[s], &tma_q, ks * kBK, m0, &sm.afull[s]);
                }
            }
        }
    } else if (warp == 1) {
        // ---- MMA issue ----
        if (lane == 0) {
            const uint32_t idesc = ptx::idesc_bf16_f32(kBM, kBN);
            int64_t g = 0;
            int64_t it = 0;
            for (int64_t t = tile_begin; t < tile_end; ++t, ++it) {
                if (it > 0 && !ptx::mbar_wait(&sm.tfree, (uint32_t)((it - 1) & 1))) {
                    atomicExch(&sm.abort, 1);
                }
                if (sm.abort) break;
                for (int ks = 0; ks < ks_per_tile; ++ks, ++g) {
                    const int s = (int)(g % kStages);
                    const uint32_t par = (uint32_t)((g / kStages) & 1);
                    if (!ptx::mbar_wait(&sm.afull[s], par) || !ptx::mbar_wait(&sm.bfull[s], par)) {
                        atomicExch(&sm.abort, 1);
                        break;
                    }
                    ptx::tc_fence_after();
                    const bool second = ks >= ks_half;
                    const uint32_t d_col = second ? 256u : 0u;
                    const bool first = (ks == 0) || (ks == ks_half);
                    const uint32_t a_addr = ptx::smem_addr(sm.a[s]);
                    const uint32_t b_addr = ptx::smem_addr(sm.b[s]);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        ptx::mma_ss(tmem + d_col, ptx::smem_desc_kmajor_sw128(a_addr + kk * 32),
                                    ptx::smem_desc_kmajor(b_addr + kk * 2 * (kBN * 16), kBN * 16, 128), idesc,
                                    (first && kk == 0) ? 0u : 1u);
                    ptx::mma_commit(&sm.empty[s]);
                }
                if (sm.abort) break;
                ptx::mma_commit(&sm.done);
            }
        }
    } else if (warp >= kExpWarp0) {
        // ---- expanders: key bits -> +-1 bf16 ----
        // K-step g of the CTA (tile tile_begin + g / ks_per_tile, step g % ks_per_tile) needs 8
        // bytes of one bit plane for each of the tile's 256 keys; each thread handles one key.
        // The bytes of four consecutive steps are contiguous in the key's row (d is a multiple of
        // 256, so a group of four never crosses the plane or the tile), so a thread fetches them
        // with two 16-byte loads one group ahead of the expansion.
        const int e = threadIdx.x - kExpWarp0 * 32;   // key within the tile, 0..255
        const int64_t nsteps = (tile_end - tile_begin) * ks_per_tile;
        // The groups are fetched in order, so the fetch position (tile, step) advances by four
        // per call instead of being divided out of the step index.
        const int row_bytes = p.d / 8;
        int64_t f_tile = tile_begin;   // tile and step of the next fetch
        int f_ks = 0;
        auto fetch = [&](uint4& lo, uint4& hi) {
            lo = make_uint4(0u, 0u, 0u, 0u);
            hi = lo;
            if (f_tile >= tile_end) return;
            const uint8_t* plane = (f_ks < ks_half) ? p.codes : p.qjl;
            const int byte0 = ((f_ks < ks_half) ? f_ks : f_ks - ks_half) * (kBK / 8);
            const int64_t key = f_tile * kBN + e;
            if (key < p.n) {
                const uint4* src = reinterpret_cast<const uint4*>(plane + key * row_bytes + byte0);
                lo = __ldg(src);
                hi = __ldg(src + 1);
            }
            f_ks += 4;
            if (f_ks == ks_per_tile) {
                f_ks = 0;
                ++f_tile;
            }
        };
        // expand step g from `bits` into its stage; false when the CTA stops. Each warp waits for
        // the stage on its own and arrives on bfull once its keys are written (8 arrivals).
        auto expand = [&](int64_t g, const uint2 bits) -> bool {
            const int s = (int)(g % kStages);
            const int64_t r = g / kStages;
            bool ok = true;
            if (r > 0) ok = ptx::mbar_wait(&sm.empty[s], (uint32_t)((r - 1) & 1));
            if (!ok) atomicExch(&sm.abort, 1);
            if (!__all_sync(0xffffffffu, ok && !sm.abort)) return false;
            {
                uint8_t* dst = sm.b[s] + (e >> 3) * 128 + (e & 7) * 16;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    // byte j of the step's 64 bits -> 8 bf16 values, +1 for a set bit: word k holds
                    // bits 2k (low half) and 2k+1 (high half); one multiply places both sign bits
                    // (bit 15 and bit 31), one logic op masks them into -1.0 / -1.0
                    const uint32_t x = __byte_perm(j < 4 ? bits.x : bits.y, 0u, 0x4440u | (j & 3));
                    uint4 v;
                    v.x = (x * 0x40008000u & 0x80008000u) ^ 0xBF80BF80u;
                    v.y = (x * 0x10002000u & 0x80008000u) ^ 0xBF80BF80u;
                    v.z = (x * 0x04000800u & 0x80008000u) ^ 0xBF80BF80u;
                    v.w = (x * 0x01000200u & 0x80008000u) ^ 0xBF80BF80u;
                    *reinterpret_cast<uint4*>(dst + j * (kBN * 16)) = v;
                }
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if ((threadIdx.x & 31) == 0) {
                // arrive (no transaction bytes): plain arrive on the barrier
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(ptx::smem_addr(&sm.bfull[s])) : "memory");
            }
            return true;
        };
        uint4 nlo, nhi;
        fetch(nlo, nhi);
        bool run = true;
        for (int64_t g0 = 0; g0 < nsteps && run; g0 += 4) {
            const uint4 clo = nlo, chi = nhi;
            fetch(nlo, nhi);   // steps g0 + 4 .. g0 + 7
            run = expand(g0, make_uint2(clo.x, clo.y)) && expand(g0 + 1, make_uint2(clo.z, clo.w)) &&
                  expand(g0 + 2, make_uint2(chi.x, chi.y)) && expand(g0 + 3, make_uint2(chi.z, chi.w));
        }
    } else {
        // ---- epilogue: warps 2..9, two threads per query (one per half of the tile's keys) ----
        const int quad = warp & 3;
        const int half = (warp - kEpiWarp0) >> 2;
        const int row = quad * 32 + lane;
        const int col = half * kBM + row;   // this thread's column of the candidate buffer
        const int m = m0 + row;
        const int et = threadIdx.x - kEpiWarp0 * 32;   // 0..255 within the epilogue group
        float best_v[kTopMax];
        int best_i[kTopMax];   // key index (n < 2^31)
#pragma unroll
        for (int i = 0; i < kTopMax; ++i) {
            best_v[i] = -INFINITY;
            best_i[i] = INT_MAX;
        }
        // Estimates above the current k-th best go to the query's candidate buffer (in key
        // order); the buffer is merged into the sorted list once per tile, after the tile's
        // accumulator has been released (so the merge overlaps the next tile's MMAs), or by the
        // whole warp when some lane's buffer could overflow. The result does not depend on when
        // the merges happen: the threshold is never above the list's k-th best, and the list
        // takes keys in key order with strict comparisons (ties stay with the lower key).
        float thr = -INFINITY;
        int cnt = 0;
        auto merge = [&]() {
            for (int i = 0; i < cnt; ++i) {
                const float est = sm.candv[i][col];
                if (est > best_v[kTopMax - 1]) {
                    best_v[kTopMax - 1] = est;
                    best_i[kTopMax - 1] = sm.candi[i][col];
#pragma unroll
                    for (int j = kTopMax - 1; j > 0; --j) {
                        if (best_v[j] > best_v[j - 1]) {
                            const float tv = best_v[j];
                            best_v[j] = best_v[j - 1];
                            best_v[j - 1] = tv;
                            const int ti = best_i[j];
                            best_i[j] = best_i[j - 1];
                            best_i[j - 1] = ti;
                        }
                    }
                }
            }
            cnt = 0;
            thr = best_v[kTopMax - 1];
        };
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        int64_t it = 0;
        bool failed = false;
        for (int64_t t = tile_begin; t < tile_end; ++t, ++it) {
            // per-key scales of this tile
            for (int i = et; i < kBN; i += 256) {
                const int64_t key = t * kBN + i;
                sm.nu[i] = (key < p.n) ? __ldg(p.norms + key) : 0.f;
                sm.g2[i] = (key < p.n) ? __ldg(p.rnorms + key) * p.qjl_scale : 0.f;
            }
            bool ok = true;
            if (et == 0) ok = ptx::mbar_wait(&sm.done, (uint32_t)(it & 1));
            if (et == 0 && !ok) atomicExch(&sm.abort, 1);
            if (named_sync_or(2, 256, et == 0 && (!ok || sm.abort))) {
                failed = true;
                break;
            }
            ptx::tc_fence_after();
#pragma unroll 1
            for (int c = half * (kBN / 16); c < (half + 1) * (kBN / 16); ++c) {
                // room for this group's 8 keys: the whole warp merges together (a merge taken by
                // one lane at a time ran once per lane, serialised, while the first tile filled
                // the buffers)
                if (__any_sync(0xffffffffu, cnt > kCand - 8)) merge();
                uint32_t a1[8], a2[8];
                ptx::tmem_ld8(t_lane + c * 8, a1);
                ptx::tmem_ld8(t_lane + 256 + c * 8, a2);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int kl = c * 8 + j;
                    const int64_t key = t * kBN + kl;
                    const float est = sm.nu[kl] * fmaf(sm.g2[kl], __uint_as_float(a2[j]), p.c1 * __uint_as_float(a1[j]));
                    if (key < p.n && est > thr) {
                        sm.candv[cnt][col] = est;
                        sm.candi[cnt][col] = (int)key;
                        ++cnt;
                    }
                }
            }
            ptx::tc_fence_before();
            named_sync(2, 256);   // every epilogue thread is done with TMEM and sm.nu / sm.g2
            if (et == 0)
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(ptx::smem_addr(&sm.tfree)) : "memory");
            merge();   // while the next tile's MMAs run
        }
        if (failed) {
            if (et == 0) atomicExch(&g_tq_device_error, 1);
        } else if (m < p.nq) {
            const int64_t o = (((int64_t)m * gridDim.y + blockIdx.y) * 2 + half) * p.k;
#pragma unroll
            for (int i = 0; i < kTopMax; ++i)
                if (i < p.k) {
                    p.cand_v[o + i] = best_v[i];
                    p.cand_i[o + i] = (best_i[i] == INT_MAX) ? INT64_MAX : (int64_t)best_i[i];
                }
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, 512);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn tiled_fn_s() {
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

// fp32 rows -> [hi | lo] bf16 rows (hi = bf16(v), lo = bf16(v - hi)), or -> bf16 rows.
__global__ void split_rows_kernel(const float* __restrict__ in, int64_t rows, int d, uint16_t* __restrict__ out,
                                  int with_lo) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * d) return;
    const int64_t r = i / d;
    const int j = (int)(i - r * d);
    const float v = in[i];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const uint16_t hb = *reinterpret_cast<const uint16_t*>(&h);
    const int64_t ld = with_lo ? 2 * d : d;
    out[r * ld + j] = hb;
    if (with_lo) {
        const __nv_bfloat16 l = __float2bfloat16_rn(v - __bfloat162float(h));
        out[r * ld + d + j] = *reinterpret_cast<const uint16_t*>(&l);
    }
}

// Queries as the GEMM operand: [bf16(q') | bf16(u)] rows of 2d.
__global__ void pack_queries_kernel(const float* __restrict__ qp, const float* __restrict__ u, int64_t rows, int d,
                                    uint16_t* __restrict__ out) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= rows * d) return;
    const int64_t r = i / d;
    const int j = (int)(i - r * d);
    const __nv_bfloat16 a = __float2bfloat16_rn(qp[i]);
    const __nv_bfloat16 b = __float2bfloat16_rn(u[i]);
    out[r * 2 * d + j] = *reinterpret_cast<const uint16_t*>(&a);
    out[r * 2 * d + d + j] = *reinterpret_cast<const uint16_t*>(&b);
}

}  // namespace

int launch_gemm_f32(const void* A, int64_t lda, const void* B, int64_t ldb, int M, int N, int K, int b_kwrap,
                    float* C, int ldc, void* stream);
int launch_search_merge(int64_t nq, int64_t ncand, int k, const float* cand_v, const int64_t* cand_i, int64_t* idx,
                        float* vals, void* stream);

namespace {
// q' = Pi q for the randomized Hadamard rotation: one block per query (signs, the Sylvester
// or Kronecker transform in shared memory, 1/sqrt(d)).
__global__ void __launch_bounds__(256)
rht_rows_kernel(const DevState st, const void* __restrict__ q, int qdtype, float* __restrict__ qp) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float* v = reinterpret_cast<float*>(smem_raw);
    const int d = st.d;
    const int64_t r = blockIdx.x;
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
        const float x = (qdtype == TQ_F32) ? __ldg(reinterpret_cast<const float*>(q) + r * d + j)
                                           : bf16_bits_to_float(__ldg(reinterpret_cast<const uint16_t*>(q) + r * d + j));
        v[j] = rht_neg(st, j) ? -x : x;
    }
    __syncthreads();
    if ((d & (d - 1)) == 0) {
        for (int h = 1; h < d; h <<= 1) {
            for (int p = threadIdx.x; p < d / 2; p += blockDim.x) {
                const int j = (p / h) * 2 * h + (p % h);
                const float a = v[j], b = v[j + h];
                v[j] = a + b;
                v[j + h] = a - b;
            }
            __syncthreads();
        }
    } else {
        kron_hadamard(v, d, st.h12, false, threadIdx.x, blockDim.x, [] { __syncthreads(); });
    }
    for (int j = threadIdx.x; j < d; j += blockDim.x) qp[r * d + j] = v[j] * st.rsqrt_d;
}
}  // namespace

bool search_tc_supported(const DevState& st, int qdtype, int k) {
    return k <= kTopMax && st.mode == TQ_PROD && st.b_mse == 1 && st.mat_dtype == TQ_BF16 &&
           st.d >= 512 && st.d % 256 == 0 && k <= kTopMax && (qdtype == TQ_BF16 || qdtype == TQ_F32);
}

namespace {
int search_ctas_y(int64_t n) {
    const int64_t tiles = (n + kBN - 1) / kBN;
    const int64_t per = 16;   // key tiles per CTA (4096 keys)
    return (int)((tiles + per - 1) / per);
}
}  // namespace

size_t search_tc_ws_bytes(const DevState& st, int64_t nq, int64_t n, int k) {
    const size_t d = st.d;
    size_t b = 0;
    auto add = [&](size_t bytes) { b += (bytes + 1023) & ~(size_t)1023; };
    add(nq * d * 4);          // q'
    add(nq * d * 4);          // u
    add(nq * 2 * d * 2);      // split / packed bf16 operand
    add(nq * 2 * d * 2);      // packed queries
    const size_t nc = (size_t)nq * search_ctas_y(n) * 2 * k;   // two lists per (query, CTA)
    add(nc * 4);
    add(nc * 8);
    return b;
}

int launch_search_tc(const DevState& st, const void* q, int qdtype, int64_t nq, const uint8_t* codes,
                     const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, int k, int64_t* idx,
                     float* vals, void* ws, void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    const int d = st.d;
    unsigned char* w = reinterpret_cast<unsigned char*>(ws);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        void* r = w + off;
        off += (bytes + 1023) & ~(size_t)1023;
        return r;
    };
    float* qp = reinterpret_cast<float*>(take(nq * d * 4));
    float* u = reinterpret_cast<float*>(take(nq * d * 4));
    uint16_t* split = reinterpret_cast<uint16_t*>(take(nq * 2 * d * 2));
    uint16_t* qpack = reinterpret_cast<uint16_t*>(take(nq * 2 * d * 2));
    const int cy = search_ctas_y(n);
    const size_t nc = (size_t)nq * cy * 2 * k;
    float* cand_v = reinterpret_cast<float*>(take(nc * 4));
    int64_t* cand_i = reinterpret_cast<int64_t*>(take(nc * 8));
    const int threads = 256;
    const unsigned blocks = (unsigned)((nq * d + threads - 1) / threads);
    int e;
    // q' = Pi q
    if (st.rot == TQ_ROT_RHT) {
        rht_rows_kernel<<<(unsigned)nq, 256, d * sizeof(float), s>>>(st, q, qdtype, qp);
        e = (int)cudaGetLastError();
    } else if (qdtype == TQ_BF16) {
        e = launch_gemm_f32(q, d, st.pi, d, (int)nq, d, d, d, qp, d, stream);
    } else {
        split_rows_kernel<<<blocks, threads, 0, s>>>(reinterpret_cast<const float*>(q), nq, d, split, 1);
        e = launch_gemm_f32(split, 2 * d, st.pi, d, (int)nq, d, 2 * d, d, qp, d, stream);
    }
    if (e) return e;
    // u = S q' (q' split into bf16 hi + lo)
    split_rows_kernel<<<blocks, threads, 0, s>>>(qp, nq, d, split, 1);
    e = launch_gemm_f32(split, 2 * d, st.s, d, (int)nq, d, 2 * d, d, u, d, stream);
    if (e) return e;
    pack_queries_kernel<<<blocks, threads, 0, s>>>(qp, u, nq, d, qpack);
    if ((e = (int)cudaGetLastError())) return e;
    // search GEMM + per-CTA top-k
    EncodeTiledFn enc = tiled_fn_s();
    if (!enc) return (int)cudaErrorNotSupported;
    CUtensorMap tm;
    const cuuint64_t gdim[2] = {(cuuint64_t)(2 * d), (cuuint64_t)nq};
    const cuuint64_t gstride[1] = {(cuuint64_t)(2 * d) * 2};
    const cuuint32_t box[2] = {64, kBM};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, qpack, gdim, gstride, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
        return (int)cudaErrorInvalidValue;
    SearchParams p;
    p.nq = (int)nq;
    p.n = n;
    p.d = d;
    p.k = k;
    p.tiles_per_cta = 16;
    p.codes = codes;
    p.qjl = qjl;
    p.norms = norms;
    p.rnorms = rnorms;
    p.c1 = st.c[1];
    p.qjl_scale = st.qjl_scale;
    p.cand_v = cand_v;
    p.cand_i = cand_i;
    const size_t smem = sizeof(SearchSmem) + 1024;
    static int attr_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_dev != dev) {
        cudaError_t ce = cudaFuncSetAttribute(search_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (ce != cudaSuccess) return (int)ce;
        attr_dev = dev;
    }
    dim3 grid((unsigned)((nq + kBM - 1) / kBM), (unsigned)cy);
    search_tc_kernel<<<grid, kThreads, smem, s>>>(tm, p);
    if ((e = (int)cudaGetLastError())) return e;
    return launch_search_merge(nq, (int64_t)cy * 2 * k, k, cand_v, cand_i, idx, vals, stream);
}

int take_device_error_search(int* flag) {
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
