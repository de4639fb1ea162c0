// Tensor-core encoder for d = 128 with the randomized Hadamard rotation and bf16 input
// (TurboQuant_prod with S stored bf16, or TurboQuant_mse).
//
// TurboQuant review (Jump2Paper): Theorem 1 (rotate, per-coordinate Lloyd-Max code),
// Definition 1 + Theorem 2 (QJL signs of S r on the residual, ||r|| kept); AI Trends
// summary of the TurboQuant video (L2 normalise + RHT).
//
// Layout of the work: a CTA of 128 threads owns tiles of 128 vectors; thread t is vector t
// of the tile, which is also TMEM lane t of the MMA accumulator.
//   1. TMA (128-byte swizzle) brings the tile's bf16 rows into shared memory, two stages
//      deep, so the next tile streams in while this one is computed.
//   2. Each thread reads its row, flips the RHT signs on the packed bf16 bits, converts to
//      fp32, takes ||x||, runs the 7-stage Walsh-Hadamard butterfly in registers (paired
//      fp32 adds), scales by 1/(sqrt(d) ||x||), quantizes against the Lloyd-Max boundaries,
//      and writes codes and norms.
//   3. prod: the residual r = y - c[idx] is split as r = hi + lo (both bf16, lo = bf16(r - hi))
//      and written to TMEM as the MMA A operand; one thread issues 16 tcgen05.mma
//      (K = 128 for hi, then for lo) against S held in shared memory (K-major core
//      matrices), accumulating S r in fp32 in TMEM. The split keeps the error of S r at
//      about 2^-16 |S||r|, so a sign is decided as fp32 arithmetic on r would decide it.
//   4. Each thread reads its 128 accumulator columns back (tcgen05.ld) and packs the signs
//      [(S r)_j >= 0] into 16 bytes.
// Every wait is bounded; on a timeout the kernel records an error word and returns.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace tq {

namespace {
__device__ int g_tq_device_error = 0;
}  // namespace

namespace {

constexpr int kTile = 128;
constexpr int kD = 128;
constexpr uint32_t kTmemCols = 256;   // [0,128) accumulator, [128,192) A hi, [192,256) A lo

struct TcParams {
    uint8_t* codes;
    uint8_t* qjl;
    float* norms;
    float* rnorms;
    const uint16_t* s;        // S, bf16, row-major [128][128]
    int64_t n;
    float rsqrt_d;
    float t[16];              // boundaries
    float c[16];              // centroids
    uint32_t sgn[64];         // XOR mask per bf16 pair: bit 15 / bit 31 flip elements 2i / 2i+1
};

struct __align__(1024) TcSmem {
    uint8_t x[2][2][kTile * 128];   // [stage][half]: 128 rows x 128 bytes, 128B-swizzled
    uint8_t s[kD * kD * 2];         // S as the B operand: K-major core matrices
    uint64_t bar_x[2];
    uint64_t bar_mma;
    uint32_t tmem_base;
    int pad;
};

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// Walsh-Hadamard butterfly over 128 values held as 64 float2 (v[i] = elements 2i, 2i+1).
__device__ __forceinline__ void fwht128(float2 (&v)[64]) {
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        const float a = v[i].x, b = v[i].y;
        v[i] = f2(a + b, a - b);
    }
    const float2 m1 = f2(-1.f, -1.f);
#pragma unroll
    for (int k = 1; k < 64; k <<= 1) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            if ((i & k) == 0) {
                const float2 a = v[i], b = v[i + k];
                v[i] = __fadd2_rn(a, b);
                v[i + k] = __ffma2_rn(b, m1, a);
            }
        }
    }
}

template <int B>
__device__ __forceinline__ void put_code(uint32_t (&cw)[4 * (B > 0 ? B : 1)], int j, uint32_t code) {
    const int bit = j * B;
    const int w = bit >> 5, sh = bit & 31;
    cw[w] |= code << sh;
    if (sh + B > 32) cw[w + 1] |= code >> (32 - sh);
}

template <int B, bool PROD>
__global__ void __launch_bounds__(kTile, 2)
encode_tc_kernel(const __grid_constant__ CUtensorMap tmap, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    TcSmem& sm = *reinterpret_cast<TcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int64_t ntiles = (p.n + kTile - 1) / kTile;

    if (tid == 0) {
        ptx::prefetch_tmap(&tmap);
        ptx::mbar_init(&sm.bar_x[0], 1);
        ptx::mbar_init(&sm.bar_x[1], 1);
        ptx::mbar_init(&sm.bar_mma, 1);
        ptx::fence_mbar_init();
    }
    if constexpr (PROD) {
        if (warp == 0) {
            ptx::tmem_alloc(&sm.tmem_base, kTmemCols);
            ptx::tmem_relinquish();
        }
        // S into shared memory: chunk c (8 values along K) of row n at c*2048 + (n/8)*128 + (n%8)*16
        for (int i = tid; i < kD * 16; i += kTile) {
            const int row = i >> 4, c = i & 15;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.s + row * kD + c * 8));
            *reinterpret_cast<uint4*>(sm.s + c * 2048 + (row >> 3) * 128 + (row & 7) * 16) = v;
        }
        ptx::fence_proxy_async_smem();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = PROD ? sm.tmem_base : 0u;
    const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);

    auto issue = [&](int stg, int64_t tile) {
        ptx::mbar_arrive_expect_tx(&sm.bar_x[stg], 2 * kTile * 128);
        ptx::tma_load_2d(sm.x[stg][0], &tmap, 0, (int)(tile * kTile), &sm.bar_x[stg]);
        ptx::tma_load_2d(sm.x[stg][1], &tmap, 64, (int)(tile * kTile), &sm.bar_x[stg]);
    };
    uint32_t pending = 0u;   // bit s: a load into stage s is in flight
    const int64_t t0 = blockIdx.x;
    if (t0 < ntiles) {
        if (tid == 0) issue(0, t0);
        pending |= 1u;
    }
    if (t0 + gridDim.x < ntiles) {
        if (tid == 0) issue(1, t0 + gridDim.x);
        pending |= 2u;
    }
    uint32_t xphase = 0u;    // bit s: parity of the next phase of stage s
    uint32_t mphase = 0u;
    bool failed = false;
    const uint32_t idesc = ptx::idesc_bf16_f32(128, 128);
    const uint32_t s_addr = ptx::smem_addr(sm.s);

    int it = 0;
    for (int64_t tile = t0; tile < ntiles; tile += gridDim.x, ++it) {
        const int stg = it & 1;
        const bool ok = ptx::mbar_wait(&sm.bar_x[stg], (xphase >> stg) & 1u);
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        xphase ^= 1u << stg;
        pending &= ~(1u << stg);
        // ---- read this thread's row (undo the 128-byte swizzle) ----
        uint32_t w[64];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint8_t* base = sm.x[stg][h] + tid * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 q = *reinterpret_cast<const uint4*>(base + ((c ^ (tid & 7)) << 4));
                w[h * 32 + c * 4 + 0] = q.x;
                w[h * 32 + c * 4 + 1] = q.y;
                w[h * 32 + c * 4 + 2] = q.z;
                w[h * 32 + c * 4 + 3] = q.w;
            }
        }
        __syncthreads();   // every thread has its row: the stage can be refilled
        const int64_t nxt = tile + 2 * (int64_t)gridDim.x;
        if (nxt < ntiles) {
            if (tid == 0) issue(stg, nxt);
            pending |= 1u << stg;
        }
        // ---- signs, fp32, norm ----
        float2 v[64];
        float2 ss = f2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 64; ++i) {
            const uint32_t u = w[i] ^ p.sgn[i];
            v[i] = f2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
            ss = __ffma2_rn(v[i], v[i], ss);
        }
        const float nu = sqrtf(ss.x + ss.y);
        fwht128(v);
        const float sc = (nu > 0.f) ? p.rsqrt_d / nu : 0.f;   // y = sc * (H D x)

        // ---- quantize, residual ----
        constexpr int NW = 4 * (B > 0 ? B : 1);
        uint32_t cw[NW];
#pragma unroll
        for (int i = 0; i < NW; ++i) cw[i] = 0u;
        float2 rr2 = f2(0.f, 0.f);
        if constexpr (B <= 2) {
            // Symmetric codebooks with 2 or 4 levels, decided on the unscaled coordinate:
            // sign plane N (1 = negative) and, for 4 levels, plane M (1 = |y| below t_2).
            // Cells (B = 2): y < -t2 | -t2 <= y < 0 | 0 <= y < t2 | t2 <= y.
            const float T2 = (B == 2 && nu > 0.f) ? p.t[2] / sc : INFINITY;
            const float cs = (nu > 0.f) ? p.c[B == 2 ? 2 : 1] : 0.f;
            const float cb = (nu > 0.f) ? p.c[B == 2 ? 3 : 1] : 0.f;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint32_t np = 0u, mp = 0u;
#pragma unroll
                for (int q = 15; q >= 0; --q) {
                    const int i = g * 16 + q;
                    float r[2];
#pragma unroll
                    for (int e = 1; e >= 0; --e) {
                        const float y = e ? v[i].y : v[i].x;
                        const uint32_t yb = __float_as_uint(y);
                        np = __funnelshift_l(yb, np, 1);
                        float mag = cs;
                        if constexpr (B == 2) {
                            const float dd = fabsf(y) - T2;
                            mp = __funnelshift_l(__float_as_uint(dd), mp, 1);
                            mag = (dd < 0.f) ? cs : cb;
                        }
                        const float smag = __uint_as_float(__float_as_uint(mag) | (yb & 0x80000000u));
                        r[e] = fmaf(y, sc, -smag);
                    }
                    v[i] = f2(r[0], r[1]);
                    rr2 = __ffma2_rn(v[i], v[i], rr2);
                }
                if constexpr (B == 1) {
                    cw[g] = ~np;                       // code = 1 for y >= 0
                } else {
                    const uint32_t hi_bit = ~np;              // bit 1: y >= 0
                    const uint32_t lo_bit = ~(np ^ mp);       // bit 0: negative XOR small, inverted
                    auto spread = [](uint32_t x) {
                        x &= 0xffffu;
                        x = (x | (x << 8)) & 0x00ff00ffu;
                        x = (x | (x << 4)) & 0x0f0f0f0fu;
                        x = (x | (x << 2)) & 0x33333333u;
                        x = (x | (x << 1)) & 0x55555555u;
                        return x;
                    };
                    cw[2 * g] = spread(lo_bit) | (spread(hi_bit) << 1);
                    cw[2 * g + 1] = spread(lo_bit >> 16) | (spread(hi_bit >> 16) << 1);
                }
            }
        } else {
            const float2 sc2 = f2(sc, sc);
#pragma unroll
            for (int i = 0; i < 64; ++i) v[i] = __fmul2_rn(v[i], sc2);
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                float r[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float y = e ? v[i].y : v[i].x;
                    uint32_t code = 0;
                    float cv = p.c[0];
#pragma unroll
                    for (int k = 0; k < (1 << B) - 1; ++k) {
                        if (y >= p.t[k]) {
                            code = k + 1;
                            cv = p.c[k + 1];
                        }
                    }
                    put_code<B>(cw, 2 * i + e, code);
                    r[e] = (nu > 0.f) ? (y - cv) : 0.f;
                }
                v[i] = f2(r[0], r[1]);
                rr2 = __ffma2_rn(v[i], v[i], rr2);
            }
        }
        const int64_t row = tile * kTile + tid;
        if (row < p.n) {
            uint4* co = reinterpret_cast<uint4*>(p.codes + row * (16 * B));
#pragma unroll
            for (int q = 0; q < B; ++q) co[q] = make_uint4(cw[4 * q], cw[4 * q + 1], cw[4 * q + 2], cw[4 * q + 3]);
            p.norms[row] = nu;
            if constexpr (PROD) p.rnorms[row] = sqrtf(rr2.x + rr2.y);
        }
        if constexpr (PROD) {
            // ---- A = [hi | lo] into TMEM columns 128.. ----
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                uint32_t hi[32], lo[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const float2 r = v[part * 32 + q];
                    const __nv_bfloat162 h = __float22bfloat162_rn(r);
                    const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h);
                    const float2 hf = f2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xffff0000u));
                    const float2 l = __ffma2_rn(hf, f2(-1.f, -1.f), r);
                    const __nv_bfloat162 lb = __float22bfloat162_rn(l);
                    hi[q] = hb;
                    lo[q] = *reinterpret_cast<const uint32_t*>(&lb);
                }
                ptx::tmem_st32(t_lane + 128 + part * 32, hi);
                ptx::tmem_st32(t_lane + 192 + part * 32, lo);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncthreads();
            if (tid == 0) {
                ptx::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ts(tmem, tmem + 128 + kk * 8,
                                ptx::smem_desc_kmajor(s_addr + kk * 2 * 2048, 2048, 128), idesc, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ts(tmem, tmem + 192 + kk * 8,
                                ptx::smem_desc_kmajor(s_addr + kk * 2 * 2048, 2048, 128), idesc, 1u);
                ptx::mma_commit(&sm.bar_mma);
            }
            const bool mok = ptx::mbar_wait(&sm.bar_mma, mphase);
            if (__syncthreads_or(!mok)) {
                failed = true;
                break;
            }
            mphase ^= 1u;
            ptx::tc_fence_after();
            // ---- signs of S r ----
            uint32_t zw[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t acc[32];
                ptx::tmem_ld32(t_lane + q * 32, acc);
                ptx::tmem_wait_ld();
                uint32_t neg = 0u;   // sign bits, collected so that bit j is column j
#pragma unroll
                for (int j = 31; j >= 0; --j) neg = __funnelshift_l(acc[j], neg, 1);
                zw[q] = (nu > 0.f) ? ~neg : 0xffffffffu;   // r = 0 -> S r = 0 -> all signs +1
            }
            ptx::tc_fence_before();
            if (row < p.n) *reinterpret_cast<uint4*>(p.qjl + row * 16) = make_uint4(zw[0], zw[1], zw[2], zw[3]);
        }
    }
    if (failed) {
        if (tid == 0) atomicExch(&g_tq_device_error, 1);
        // let copies in flight land before the shared memory goes away (bounded)
        for (int s2 = 0; s2 < 2; ++s2)
            if ((pending >> s2) & 1u) (void)ptx::mbar_wait(&sm.bar_x[s2], (xphase >> s2) & 1u);
        if (PROD) (void)ptx::mbar_wait(&sm.bar_mma, mphase, 100000000ull);
    }
    __syncthreads();
    if constexpr (PROD) {
        if (warp == 0) {
            ptx::tc_fence_after();
            ptx::tmem_dealloc(tmem, kTmemCols);
        }
    }
}

// ------------------------------------------------------------------------------------
// Two threads per vector (b_mse = 1 or 2): 256 threads per 128-vector tile. Warp w serves
// vectors 32*(w%4) .. +31 (its TMEM lane quadrant) and coordinates 64*(w/4) .. +63. Both
// threads of a vector read the whole bf16 row, so the stride-64 butterfly stage is taken
// at load time (y_j = x_j +- x_{j+64}) and the remaining six stages stay in registers.
// Halving the per-thread state keeps registers under 128, so two CTAs (16 warps) fit
// on an SM; the two halves meet only through ||r||^2 (shared memory) and the MMA.
// ------------------------------------------------------------------------------------
struct __align__(1024) TcSmem2 {
    uint8_t x[2][2][kTile * 128];   // [stage][half]: 128 rows x 128 bytes, 128B-swizzled
    uint8_t s[kD * kD * 2];         // S as the B operand: K-major core matrices
    float rr[2][kTile];             // per half: partial ||r||^2
    uint64_t bar_x[2];
    uint64_t bar_mma;
    uint32_t tmem_base;
    int pad;
};

__device__ __forceinline__ uint32_t spread16(uint32_t x) {
    x &= 0xffffu;
    x = (x | (x << 8)) & 0x00ff00ffu;
    x = (x | (x << 4)) & 0x0f0f0f0fu;
    x = (x | (x << 2)) & 0x33333333u;
    x = (x | (x << 1)) & 0x55555555u;
    return x;
}

template <int B, bool PROD>
__global__ void __launch_bounds__(2 * kTile, 2)
encode_tc2_kernel(const __grid_constant__ CUtensorMap tmap, const TcParams p) {
    static_assert(B == 1 || B == 2, "two-thread layout covers 1- and 2-bit codes");
    extern __shared__ uint8_t smem_raw[];
    TcSmem2& sm = *reinterpret_cast<TcSmem2*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int quad = warp & 3;
    const int half = warp >> 2;
    const int vrow = quad * 32 + (tid & 31);   // vector within the tile = TMEM lane
    const int64_t ntiles = (p.n + kTile - 1) / kTile;

    if (tid == 0) {
        ptx::prefetch_tmap(&tmap);
        ptx::mbar_init(&sm.bar_x[0], 1);
        ptx::mbar_init(&sm.bar_x[1], 1);
        ptx::mbar_init(&sm.bar_mma, 1);
        ptx::fence_mbar_init();
    }
    if constexpr (PROD) {
        if (warp == 0) {
            ptx::tmem_alloc(&sm.tmem_base, kTmemCols);
            ptx::tmem_relinquish();
        }
        for (int i = tid; i < kD * 16; i += 2 * kTile) {
            const int row = i >> 4, c = i & 15;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.s + row * kD + c * 8));
            *reinterpret_cast<uint4*>(sm.s + c * 2048 + (row >> 3) * 128 + (row & 7) * 16) = v;
        }
        ptx::fence_proxy_async_smem();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = PROD ? sm.tmem_base : 0u;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);

    auto issue = [&](int stg, int64_t tile) {
        ptx::mbar_arrive_expect_tx(&sm.bar_x[stg], 2 * kTile * 128);
        ptx::tma_load_2d(sm.x[stg][0], &tmap, 0, (int)(tile * kTile), &sm.bar_x[stg]);
        ptx::tma_load_2d(sm.x[stg][1], &tmap, 64, (int)(tile * kTile), &sm.bar_x[stg]);
    };
    uint32_t pending = 0u, xphase = 0u, mphase = 0u;
    const int64_t t0 = blockIdx.x;
    if (t0 < ntiles) {
        if (tid == 0) issue(0, t0);
        pending |= 1u;
    }
    if (t0 + gridDim.x < ntiles) {
        if (tid == 0) issue(1, t0 + gridDim.x);
        pending |= 2u;
    }
    bool failed = false;
    const uint32_t idesc = ptx::idesc_bf16_f32(128, 128);
    const uint32_t s_addr = ptx::smem_addr(sm.s);
    const float2 hs = half ? f2(-1.f, -1.f) : f2(1.f, 1.f);

    int it = 0;
    for (int64_t tile = t0; tile < ntiles; tile += gridDim.x, ++it) {
        const int stg = it & 1;
        const bool ok = ptx::mbar_wait(&sm.bar_x[stg], (xphase >> stg) & 1u);
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        xphase ^= 1u << stg;
        pending &= ~(1u << stg);
        // ---- read x_j and x_{j+64} (8 at a time), signs, fp32, stride-64 stage ----
        float2 v[32];
        float2 ss = f2(0.f, 0.f);
        {
            const uint8_t* b0 = sm.x[stg][0] + vrow * 128;
            const uint8_t* b1 = sm.x[stg][1] + vrow * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int off = (c ^ (vrow & 7)) << 4;
                const uint4 qa = *reinterpret_cast<const uint4*>(b0 + off);
                const uint4 qb = *reinterpret_cast<const uint4*>(b1 + off);
                const uint32_t wa[4] = {qa.x, qa.y, qa.z, qa.w};
                const uint32_t wb[4] = {qb.x, qb.y, qb.z, qb.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t ua = wa[e] ^ p.sgn[4 * c + e];
                    const uint32_t ub = wb[e] ^ p.sgn[32 + 4 * c + e];
                    const float2 xa = f2(__uint_as_float(ua << 16), __uint_as_float(ua & 0xffff0000u));
                    const float2 xb = f2(__uint_as_float(ub << 16), __uint_as_float(ub & 0xffff0000u));
                    ss = __ffma2_rn(xa, xa, ss);
                    ss = __ffma2_rn(xb, xb, ss);
                    v[4 * c + e] = __ffma2_rn(xb, hs, xa);
                }
            }
        }
        __syncthreads();   // both halves have read the stage: refill it
        const int64_t nxt = tile + 2 * (int64_t)gridDim.x;
        if (nxt < ntiles) {
            if (tid == 0) issue(stg, nxt);
            pending |= 1u << stg;
        }
        const float nu = sqrtf(ss.x + ss.y);
        // ---- remaining butterfly stages (strides 1..32) on the local 64 values ----
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float a = v[i].x, b = v[i].y;
            v[i] = f2(a + b, a - b);
        }
#pragma unroll
        for (int k = 1; k < 32; k <<= 1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if ((i & k) == 0) {
                    const float2 a = v[i], b = v[i + k];
                    v[i] = __fadd2_rn(a, b);
                    v[i + k] = __ffma2_rn(b, f2(-1.f, -1.f), a);
                }
            }
        }
        const float sc = (nu > 0.f) ? p.rsqrt_d / nu : 0.f;
        // ---- quantize on the unscaled coordinate; residual ----
        const float T2 = (B == 2 && nu > 0.f) ? p.t[2] / sc : INFINITY;
        const float cs = (nu > 0.f) ? p.c[B == 2 ? 2 : 1] : 0.f;
        const float cb = (nu > 0.f) ? p.c[B == 2 ? 3 : 1] : 0.f;
        uint32_t cw[2 * B];
        float2 rr2 = f2(0.f, 0.f);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            uint32_t np = 0u, mp = 0u;
#pragma unroll
            for (int q = 15; q >= 0; --q) {
                const int i = g * 16 + q;
                float r[2];
#pragma unroll
                for (int e = 1; e >= 0; --e) {
                    const float y = e ? v[i].y : v[i].x;
                    const uint32_t yb = __float_as_uint(y);
                    np = __funnelshift_l(yb, np, 1);
                    float mag = cs;
                    if constexpr (B == 2) {
                        const float dd = fabsf(y) - T2;
                        mp = __funnelshift_l(__float_as_uint(dd), mp, 1);
                        mag = (dd < 0.f) ? cs : cb;
                    }
                    const float smag = __uint_as_float(__float_as_uint(mag) | (yb & 0x80000000u));
                    r[e] = fmaf(y, sc, -smag);
                }
                v[i] = f2(r[0], r[1]);
                rr2 = __ffma2_rn(v[i], v[i], rr2);
            }
            if constexpr (B == 1) {
                cw[g] = ~np;
            } else {
                const uint32_t hb = ~np, lb = ~(np ^ mp);
                cw[2 * g] = spread16(lb) | (spread16(hb) << 1);
                cw[2 * g + 1] = spread16(lb >> 16) | (spread16(hb >> 16) << 1);
            }
        }
        const int64_t row = tile * kTile + vrow;
        if (row < p.n) {
            if constexpr (B == 2)
                *reinterpret_cast<uint4*>(p.codes + row * 32 + half * 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            else
                *reinterpret_cast<uint2*>(p.codes + row * 16 + half * 8) = make_uint2(cw[0], cw[1]);
            if (half == 0) p.norms[row] = nu;
        }
        if constexpr (PROD) {
            sm.rr[half][vrow] = rr2.x + rr2.y;
#pragma unroll
            for (int part = 0; part < 1; ++part) {
                uint32_t hi[32], lo[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const float2 r = v[q];
                    const __nv_bfloat162 h = __float22bfloat162_rn(r);
                    const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h);
                    const float2 hf = f2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xffff0000u));
                    const float2 l = __ffma2_rn(hf, f2(-1.f, -1.f), r);
                    const __nv_bfloat162 lb = __float22bfloat162_rn(l);
                    hi[q] = hb;
                    lo[q] = *reinterpret_cast<const uint32_t*>(&lb);
                }
                ptx::tmem_st32(t_lane + 128 + half * 32, hi);
                ptx::tmem_st32(t_lane + 192 + half * 32, lo);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncthreads();
            if (half == 0 && row < p.n) p.rnorms[row] = sqrtf(sm.rr[0][vrow] + sm.rr[1][vrow]);
            if (tid == 0) {
                ptx::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ts(tmem, tmem + 128 + kk * 8,
                                ptx::smem_desc_kmajor(s_addr + kk * 2 * 2048, 2048, 128), idesc, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ts(tmem, tmem + 192 + kk * 8,
                                ptx::smem_desc_kmajor(s_addr + kk * 2 * 2048, 2048, 128), idesc, 1u);
                ptx::mma_commit(&sm.bar_mma);
            }
            const bool mok = ptx::mbar_wait(&sm.bar_mma, mphase);
            if (__syncthreads_or(!mok)) {
                failed = true;
                break;
            }
            mphase ^= 1u;
            ptx::tc_fence_after();
            uint32_t zw[2];
            {
                uint32_t a0[32], a1[32];
                ptx::tmem_ld32(t_lane + half * 64, a0);
                ptx::tmem_ld32(t_lane + half * 64 + 32, a1);
                ptx::tmem_wait_ld();
                uint32_t n0 = 0u, n1 = 0u;
#pragma unroll
                for (int j = 31; j >= 0; --j) {
                    n0 = __funnelshift_l(a0[j], n0, 1);
                    n1 = __funnelshift_l(a1[j], n1, 1);
                }
                zw[0] = (nu > 0.f) ? ~n0 : 0xffffffffu;
                zw[1] = (nu > 0.f) ? ~n1 : 0xffffffffu;
            }
            ptx::tc_fence_before();
            if (row < p.n) *reinterpret_cast<uint2*>(p.qjl + row * 16 + half * 8) = make_uint2(zw[0], zw[1]);
        }
    }
    if (failed) {
        if (tid == 0) atomicExch(&g_tq_device_error, 1);
        for (int s2 = 0; s2 < 2; ++s2)
            if ((pending >> s2) & 1u) (void)ptx::mbar_wait(&sm.bar_x[s2], (xphase >> s2) & 1u);
        if (PROD) (void)ptx::mbar_wait(&sm.bar_mma, mphase, 100000000ull);
    }
    __syncthreads();
    if constexpr (PROD) {
        if (warp == 0) {
            ptx::tc_fence_after();
            ptx::tmem_dealloc(tmem, kTmemCols);
        }
    }
}

// ------------------------------------------------------------------------------------
// Rotation on the tensor core (b_mse = 1 or 2). The randomized Hadamard transform is the
// dense product y = (H diag(eps)) x: with x bf16 (exact) and H diag(eps) = +-1 (exact in
// bf16), one K = 128 MMA straight from the 128B-swizzled TMA tile gives H D x in fp32 in
// TMEM, with exact products and fp32 sums as in the register butterfly. The threads then
// only read y back, quantize, split the residual and read the signs of S r.
// Two threads per vector as in encode_tc2_kernel; TMEM columns [0,128) hold y and then
// S r, [128,256) the residual operand (hi, lo).
// ------------------------------------------------------------------------------------
struct __align__(1024) TcSmem3 {
    uint8_t x[2][kTile * 128];      // [half]: 128 rows x 128 bytes, 128B-swizzled
    uint8_t hd[kD * kD * 2];        // H diag(eps) as the B operand: K-major core matrices
    uint8_t s[kD * kD * 2];         // S as the B operand
    float ssq[2][kTile];            // per half: partial ||H D x||^2
    float rsq[2][kTile];            // per half: partial ||r||^2
    uint64_t bar_x;
    uint64_t bar_h;
    uint64_t bar_s;
    uint32_t tmem_base;
    int pad;
};

template <int B, bool PROD>
__global__ void __launch_bounds__(2 * kTile, 2)
encode_tc3_kernel(const __grid_constant__ CUtensorMap tmap, const TcParams p) {
    static_assert(B == 1 || B == 2, "two-thread layout covers 1- and 2-bit codes");
    extern __shared__ uint8_t smem_raw[];
    TcSmem3& sm = *reinterpret_cast<TcSmem3*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int quad = warp & 3;
    const int half = warp >> 2;
    const int vrow = quad * 32 + (tid & 31);
    const int64_t ntiles = (p.n + kTile - 1) / kTile;

    if (tid == 0) {
        ptx::prefetch_tmap(&tmap);
        ptx::mbar_init(&sm.bar_x, 1);
        ptx::mbar_init(&sm.bar_h, 1);
        ptx::mbar_init(&sm.bar_s, 1);
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(&sm.tmem_base, kTmemCols);
        ptx::tmem_relinquish();
    }
    // H diag(eps): entry (n, k) = (-1)^popcount(n & k) * eps_k, at chunk k/8 of row n.
    for (int i = tid; i < kD * kD; i += 2 * kTile) {
        const int n = i >> 7, k = i & 127;
        const uint32_t neg = (__popc(n & k) & 1) ^ ((p.sgn[k >> 1] >> ((k & 1) ? 31 : 15)) & 1u);
        const uint16_t v = neg ? 0xBF80u : 0x3F80u;
        *reinterpret_cast<uint16_t*>(sm.hd + (k >> 3) * 2048 + (n >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2) = v;
    }
    if constexpr (PROD) {
        for (int i = tid; i < kD * 16; i += 2 * kTile) {
            const int row = i >> 4, c = i & 15;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.s + row * kD + c * 8));
            *reinterpret_cast<uint4*>(sm.s + c * 2048 + (row >> 3) * 128 + (row & 7) * 16) = v;
        }
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);

    auto issue = [&](int64_t tile) {
        ptx::mbar_arrive_expect_tx(&sm.bar_x, 2 * kTile * 128);
        ptx::tma_load_2d(sm.x[0], &tmap, 0, (int)(tile * kTile), &sm.bar_x);
        ptx::tma_load_2d(sm.x[1], &tmap, 64, (int)(tile * kTile), &sm.bar_x);
    };
    bool pending = false;
    const int64_t t0 = blockIdx.x;
    if (t0 < ntiles) {
        if (tid == 0) issue(t0);
        pending = true;
    }
    uint32_t xph = 0u, hph = 0u, sph = 0u;
    bool failed = false, hmma_pending = false, smma_pending = false;
    const uint32_t idesc = ptx::idesc_bf16_f32(128, 128);
    const uint32_t s_addr = ptx::smem_addr(sm.s);
    const uint32_t hd_addr = ptx::smem_addr(sm.hd);
    const uint32_t x_addr0 = ptx::smem_addr(sm.x[0]);
    const uint32_t x_addr1 = ptx::smem_addr(sm.x[1]);

    for (int64_t tile = t0; tile < ntiles; tile += gridDim.x) {
        // One thread waits for the tile, runs y = (H D) x on the tensor core and waits for
        // it; the others park on the block barrier instead of spinning.
        bool ok = true;
        if (tid == 0) {
            ok = ptx::mbar_wait(&sm.bar_x, xph);
            if (ok) {
                ptx::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a = ((kk < 4) ? x_addr0 : x_addr1) + (kk & 3) * 32;
                    ptx::mma_ss(tmem, ptx::smem_desc_kmajor_sw128(a),
                                ptx::smem_desc_kmajor(hd_addr + kk * 2 * 2048, 2048, 128), idesc,
                                kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(&sm.bar_h);
                ok = ptx::mbar_wait(&sm.bar_h, hph);
                if (!ok) hmma_pending = true;
            }
        }
        if (__syncthreads_or(!ok)) {
            failed = true;
            break;
        }
        xph ^= 1u;
        hph ^= 1u;
        pending = false;
        ptx::tc_fence_after();
        const int64_t nxt = tile + gridDim.x;
        if (nxt < ntiles) {   // the MMA has read the tile: refill the buffer
            if (tid == 0) issue(nxt);
            pending = true;
        }
        float2 v[32];
        {
            uint32_t a0[32], a1[32];
            ptx::tmem_ld32(t_lane + half * 64, a0);
            ptx::tmem_ld32(t_lane + half * 64 + 32, a1);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                v[i] = f2(__uint_as_float(a0[2 * i]), __uint_as_float(a0[2 * i + 1]));
                v[16 + i] = f2(__uint_as_float(a1[2 * i]), __uint_as_float(a1[2 * i + 1]));
            }
        }
        float2 ss = f2(0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = __ffma2_rn(v[i], v[i], ss);
        sm.ssq[half][vrow] = ss.x + ss.y;
        ptx::tc_fence_before();
        __syncthreads();
        // ||H D x||^2 = d ||x||^2
        const float nu = sqrtf(sm.ssq[0][vrow] + sm.ssq[1][vrow]) * p.rsqrt_d;
        const float sc = (nu > 0.f) ? p.rsqrt_d / nu : 0.f;
        const float T2 = (B == 2 && nu > 0.f) ? p.t[2] / sc : INFINITY;
        const float cs = (nu > 0.f) ? p.c[B == 2 ? 2 : 1] : 0.f;
        const float cb = (nu > 0.f) ? p.c[B == 2 ? 3 : 1] : 0.f;
        uint32_t cw[2 * B];
        float2 rr2 = f2(0.f, 0.f);
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            uint32_t np = 0u, mp = 0u;
#pragma unroll
            for (int q = 15; q >= 0; --q) {
                const int i = g * 16 + q;
                float r[2];
#pragma unroll
                for (int e = 1; e >= 0; --e) {
                    const float y = e ? v[i].y : v[i].x;
                    const uint32_t yb = __float_as_uint(y);
                    np = __funnelshift_l(yb, np, 1);
                    float mag = cs;
                    if constexpr (B == 2) {
                        const float dd = fabsf(y) - T2;
                        mp = __funnelshift_l(__float_as_uint(dd), mp, 1);
                        mag = (dd < 0.f) ? cs : cb;
                    }
                    const float smag = __uint_as_float(__float_as_uint(mag) | (yb & 0x80000000u));
                    r[e] = fmaf(y, sc, -smag);
                }
                v[i] = f2(r[0], r[1]);
                rr2 = __ffma2_rn(v[i], v[i], rr2);
            }
            if constexpr (B == 1) {
                cw[g] = ~np;
            } else {
                const uint32_t hb = ~np, lb = ~(np ^ mp);
                cw[2 * g] = spread16(lb) | (spread16(hb) << 1);
                cw[2 * g + 1] = spread16(lb >> 16) | (spread16(hb >> 16) << 1);
            }
        }
        const int64_t row = tile * kTile + vrow;
        if (row < p.n) {
            if constexpr (B == 2)
                *reinterpret_cast<uint4*>(p.codes + row * 32 + half * 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            else
                *reinterpret_cast<uint2*>(p.codes + row * 16 + half * 8) = make_uint2(cw[0], cw[1]);
            if (half == 0) p.norms[row] = nu;
        }
        if constexpr (PROD) {
            sm.rsq[half][vrow] = rr2.x + rr2.y;
            {
                uint32_t hi[32], lo[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const float2 r = v[q];
                    const __nv_bfloat162 h = __float22bfloat162_rn(r);
                    const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h);
                    const float2 hf = f2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xffff0000u));
                    const float2 l = __ffma2_rn(hf, f2(-1.f, -1.f), r);
                    const __nv_bfloat162 lb = __float22bfloat162_rn(l);
                    hi[q] = hb;
                    lo[q] = *reinterpret_cast<const uint32_t*>(&lb);
                }
                ptx::tmem_st32(t_lane + 128 + half * 32, hi);
                ptx::tmem_st32(t_lane + 192 + half * 32, lo);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncthreads();
            if (half == 0 && row < p.n) p.rnorms[row] = sqrtf(sm.rsq[0][vrow] + sm.rsq[1][vrow]);
            bool sok = true;
            if (tid == 0) {
                ptx::tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ts(tmem, tmem + 128 + kk * 8,
                                ptx::smem_desc_kmajor(s_addr + kk * 2 * 2048, 2048, 128), idesc, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ts(tmem, tmem + 192 + kk * 8,
                                ptx::smem_desc_kmajor(s_addr + kk * 2 * 2048, 2048, 128), idesc, 1u);
                ptx::mma_commit(&sm.bar_s);
                sok = ptx::mbar_wait(&sm.bar_s, sph);
                if (!sok) smma_pending = true;
            }
            if (__syncthreads_or(!sok)) {
                failed = true;
                break;
            }
            sph ^= 1u;
            ptx::tc_fence_after();
            uint32_t zw[2];
            {
                uint32_t a0[32], a1[32];
                ptx::tmem_ld32(t_lane + half * 64, a0);
                ptx::tmem_ld32(t_lane + half * 64 + 32, a1);
                ptx::tmem_wait_ld();
                uint32_t n0 = 0u, n1 = 0u;
#pragma unroll
                for (int j = 31; j >= 0; --j) {
                    n0 = __funnelshift_l(a0[j], n0, 1);
                    n1 = __funnelshift_l(a1[j], n1, 1);
                }
                zw[0] = (nu > 0.f) ? ~n0 : 0xffffffffu;
                zw[1] = (nu > 0.f) ? ~n1 : 0xffffffffu;
            }
            if (row < p.n) *reinterpret_cast<uint2*>(p.qjl + row * 16 + half * 8) = make_uint2(zw[0], zw[1]);
        }
        ptx::tc_fence_before();
    }
    if (failed) {
        if (tid == 0) atomicExch(&g_tq_device_error, 1);
        if (tid == 0) {
            if (pending) (void)ptx::mbar_wait(&sm.bar_x, xph);
            if (hmma_pending) (void)ptx::mbar_wait(&sm.bar_h, hph, 100000000ull);
            if (smma_pending) (void)ptx::mbar_wait(&sm.bar_s, sph, 100000000ull);
        }
    }
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------------------------
// Pipelined tensor-core encoder (b_mse = 1 or 2). One persistent CTA per SM owns all 512
// TMEM columns. Warp 16 streams tiles of 128 vectors with TMA (kT4Stages deep) and issues
// the MMAs; warps 0..15 quantize, four warps per group of 32 vectors (TMEM lane quadrant
// warp % 4), each thread taking 32 of its vector's 128 coordinates. The tensor core runs
// y = (H D) x for tile k+1 and S r for tile k-1 while the warps quantize tile k.
// TMEM columns: Y [0,128) y; D [128,256) S r; HL0 [256,384), HL1 [384,512) the residual
// operand of tiles k even / odd (hi in the first 64 columns, lo in the next 64).
// Arithmetic per coordinate is that of encode_tc3_kernel: the same fp32 rotation sums, the
// level decision |y| sc < t against the Lloyd-Max boundary, the bf16 hi + lo residual and
// the sign of S r read from the fp32 accumulator.
// ------------------------------------------------------------------------------------
constexpr int kT4Stages = 3;
constexpr uint32_t kT4Cols = 512;
constexpr int kT4P = 2;   // threads per vector (each takes 128 / kT4P coordinates)
template <int P>
struct T4 {
    static constexpr int kWarps = 4 * P;                // quantizing warps
    static constexpr int kThreads = (kWarps + 1) * 32;  // + the TMA / MMA warp
    static constexpr int kC = kD / P;                   // coordinates per thread
};

struct __align__(1024) TcSmem4 {
    uint8_t x[kT4Stages][2][kTile * 128];   // [stage][half]: 128 rows x 128 bytes, 128B-swizzled
    uint8_t hd[kD * kD * 2];                // H diag(eps), B operand (K-major core matrices)
    uint8_t s[kD * kD * 2];                 // S, B operand
    float ssq[2][4][kTile];                 // [tile parity][part]: partial ||H D x||^2
    float rsq[2][4][kTile];                 // [tile parity][part]: partial ||r||^2 (up to 4 parts)
    uint64_t bar_x[kT4Stages];              // tile landed
    uint64_t bar_xfree[kT4Stages];          // the rotation MMA has read the stage
    uint64_t bar_h;                         // y of the current tile is in TMEM
    uint64_t bar_yfree;                     // all quantizing warps have read y
    uint64_t bar_hl[2];                     // residual operand written and S r of the previous tile read
    uint64_t bar_s;                         // S r is in TMEM
    uint32_t tmem_base;
    int abort;
};

template <int B, bool PROD, int P>
__global__ void __launch_bounds__(T4<P>::kThreads, 1)
encode_tc4_kernel(const __grid_constant__ CUtensorMap tmap, const TcParams p) {
    static_assert(B == 1 || B == 2, "the pipelined encoder covers 1- and 2-bit codes");
    static_assert(P == 2 || P == 4, "two or four threads per vector");
    constexpr int kWarps = T4<P>::kWarps, kThreads = T4<P>::kThreads, C = T4<P>::kC, NCH = C / 32;
    extern __shared__ uint8_t smem_raw[];
    TcSmem4& sm = *reinterpret_cast<TcSmem4*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    volatile int* abort_flag = &sm.abort;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int64_t ntiles = (p.n + kTile - 1) / kTile;
    const int64_t mytiles = (ntiles > (int64_t)blockIdx.x) ? (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

    if (tid == 0) {
        ptx::prefetch_tmap(&tmap);
        for (int i = 0; i < kT4Stages; ++i) {
            ptx::mbar_init(&sm.bar_x[i], 1);
            ptx::mbar_init(&sm.bar_xfree[i], 1);
        }
        ptx::mbar_init(&sm.bar_h, 1);
        ptx::mbar_init(&sm.bar_yfree, kWarps);
        ptx::mbar_init(&sm.bar_hl[0], kWarps);
        ptx::mbar_init(&sm.bar_hl[1], kWarps);
        ptx::mbar_init(&sm.bar_s, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(&sm.tmem_base, kT4Cols);
        ptx::tmem_relinquish();
    }
    // H diag(eps): entry (n, k) = (-1)^popcount(n & k) * eps_k, at chunk k/8 of row n.
    for (int i = tid; i < kD * kD; i += kThreads) {
        const int n = i >> 7, k = i & 127;
        const uint32_t neg = (__popc(n & k) & 1) ^ ((p.sgn[k >> 1] >> ((k & 1) ? 31 : 15)) & 1u);
        *reinterpret_cast<uint16_t*>(sm.hd + (k >> 3) * 2048 + (n >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2) =
            neg ? 0xBF80u : 0x3F80u;
    }
    if constexpr (PROD) {
        for (int i = tid; i < kD * 16; i += kThreads) {
            const int row = i >> 4, c = i & 15;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.s + row * kD + c * 8));
            *reinterpret_cast<uint4*>(sm.s + c * 2048 + (row >> 3) * 128 + (row & 7) * 16) = v;
        }
    }
    ptx::fence_proxy_async_smem();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == kWarps) {
        // ---------------- producer: TMA + MMA issue (one thread) ----------------
        if (lane == 0) {
            const uint32_t idesc = ptx::idesc_bf16_f32(128, 128);
            const uint32_t s_addr = ptx::smem_addr(sm.s);
            const uint32_t hd_addr = ptx::smem_addr(sm.hd);
            uint32_t tma_pend = 0u, tma_par = 0u;   // per stage: load in flight / its phase parity
            int h_st = -1;
            uint32_t h_par = 0u;
            bool s_issued = false;
            uint32_t s_par = 0u;
            auto load = [&](int64_t j) {
                const int st = (int)(j % kT4Stages);
                const int row0 = (int)((blockIdx.x + j * gridDim.x) * kTile);
                ptx::mbar_arrive_expect_tx(&sm.bar_x[st], 2 * kTile * 128);
                ptx::tma_load_2d(sm.x[st][0], &tmap, 0, row0, &sm.bar_x[st]);
                ptx::tma_load_2d(sm.x[st][1], &tmap, 64, row0, &sm.bar_x[st]);
                tma_pend |= 1u << st;
                tma_par = (tma_par & ~(1u << st)) | ((uint32_t)((j / kT4Stages) & 1) << st);
            };
            auto issue_s = [&](int64_t j) -> bool {
                if (!ptx::mbar_wait(&sm.bar_hl[j & 1], (uint32_t)(j >> 1) & 1u) || *abort_flag) return false;
                ptx::tc_fence_after();
                const uint32_t hl = tmem + 256u + (uint32_t)(j & 1) * 128u;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ts(tmem + 128u, hl + kk * 8, ptx::smem_desc_kmajor(s_addr + kk * 2 * 2048, 2048, 128),
                                idesc, kk > 0 ? 1u : 0u);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ts(tmem + 128u, hl + 64 + kk * 8,
                                ptx::smem_desc_kmajor(s_addr + kk * 2 * 2048, 2048, 128), idesc, 1u);
                ptx::mma_commit(&sm.bar_s);
                s_issued = true;
                s_par = (uint32_t)(j & 1);
                return true;
            };
            for (int64_t j = 0; j < mytiles && j < kT4Stages; ++j) load(j);
            bool ok = true;
            for (int64_t k = 0; k < mytiles; ++k) {
                const int st = (int)(k % kT4Stages);
                const uint32_t xpar = (uint32_t)((k / kT4Stages) & 1);
                ok = ptx::mbar_wait(&sm.bar_x[st], xpar);
                if (!ok) break;
                tma_pend &= ~(1u << st);
                if (k > 0) {
                    ok = ptx::mbar_wait(&sm.bar_yfree, (uint32_t)((k - 1) & 1)) && !*abort_flag;
                    if (!ok) break;
                }
                ptx::tc_fence_after();
                const uint32_t xa0 = ptx::smem_addr(sm.x[st][0]), xa1 = ptx::smem_addr(sm.x[st][1]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ss(tmem, ptx::smem_desc_kmajor_sw128(((kk < 4) ? xa0 : xa1) + (kk & 3) * 32),
                                ptx::smem_desc_kmajor(hd_addr + kk * 2 * 2048, 2048, 128), idesc, kk > 0 ? 1u : 0u);
                ptx::mma_commit(&sm.bar_h);
                ptx::mma_commit(&sm.bar_xfree[st]);
                h_st = st;
                h_par = xpar;
                if (PROD && k > 0) {
                    ok = issue_s(k - 1);
                    if (!ok) break;
                }
                if (k + kT4Stages < mytiles) {
                    ok = ptx::mbar_wait(&sm.bar_xfree[st], xpar);
                    if (!ok) break;
                    load(k + kT4Stages);
                }
            }
            if (ok && PROD && mytiles > 0) ok = issue_s(mytiles - 1);
            if (!ok) {
                *abort_flag = 1;
                atomicExch(&g_tq_device_error, 1);
            }
            // Drain: every copy and MMA this thread started has finished before the CTA
            // releases TMEM and shared memory.
            for (int st = 0; st < kT4Stages; ++st)
                if ((tma_pend >> st) & 1u) (void)ptx::mbar_wait(&sm.bar_x[st], (tma_par >> st) & 1u);
            if (h_st >= 0) (void)ptx::mbar_wait(&sm.bar_xfree[h_st], h_par);
            if (s_issued) (void)ptx::mbar_wait(&sm.bar_s, s_par);
        }
    } else {
        // ---------------- quantizing warps ----------------
        // warp w: lane quadrant w % 4 (vectors 32 (w % 4) ..), part w / 4 (coordinates
        // C part .. C part + C - 1 of each of those vectors)
        const int quad = warp & 3, part = warp >> 2;
        const int vrow = quad * 32 + lane;
        const int bar_id = 1 + quad;   // named barrier of the P warps sharing these vectors
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        const float t2 = p.t[2];
        int64_t prev_row = -1;
        bool prev_nz = false;
        bool fail = false;
        // Signs of S r (in D) for vector `srow`: [(S r)_j >= 0], all ones for a zero vector.
        auto emit_signs = [&](uint32_t parity, int64_t srow, bool snz) -> bool {
            bool sok = true;
            if (lane == 0) sok = ptx::mbar_wait(&sm.bar_s, parity);
            sok = __shfl_sync(0xffffffffu, sok ? 1 : 0, 0) != 0;
            ptx::tc_fence_after();
            uint32_t zw[NCH];
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                uint32_t d[32];
                ptx::tmem_ld32(t_lane + 128 + part * C + ch * 32, d);
                ptx::tmem_wait_ld();
                uint32_t z0 = 0u, z1 = 0u;
#pragma unroll
                for (int j = 15; j >= 0; --j) {
                    z0 = __funnelshift_l(d[j], z0, 1);
                    z1 = __funnelshift_l(d[j + 16], z1, 1);
                }
                zw[ch] = snz ? ~(z0 | (z1 << 16)) : 0xffffffffu;
            }
            if (sok && srow < p.n) {
                uint8_t* dst = p.qjl + srow * 16 + part * (C / 8);
                if constexpr (NCH == 2) *reinterpret_cast<uint2*>(dst) = make_uint2(zw[0], zw[1]);
                else *reinterpret_cast<uint32_t*>(dst) = zw[0];
            }
            return sok;
        };
        for (int64_t k = 0; k < mytiles; ++k) {
            const int kb = (int)(k & 1);
            const int64_t row = (blockIdx.x + k * gridDim.x) * kTile + vrow;
            bool ok = true;
            if (lane == 0) ok = ptx::mbar_wait(&sm.bar_h, (uint32_t)(k & 1));
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            ptx::tc_fence_after();
            uint32_t a[C];
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                uint32_t (&ac)[32] = *reinterpret_cast<uint32_t(*)[32]>(a + ch * 32);
                ptx::tmem_ld32(t_lane + part * C + ch * 32, ac);
            }
            ptx::tmem_wait_ld();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&sm.bar_yfree);
            float2 q0 = f2(0.f, 0.f), q1 = f2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < C / 4; ++i) {
                const float2 u0 = f2(__uint_as_float(a[4 * i]), __uint_as_float(a[4 * i + 1]));
                const float2 u1 = f2(__uint_as_float(a[4 * i + 2]), __uint_as_float(a[4 * i + 3]));
                q0 = __ffma2_rn(u0, u0, q0);
                q1 = __ffma2_rn(u1, u1, q1);
            }
            sm.ssq[kb][part][vrow] = (q0.x + q0.y) + (q1.x + q1.y);
            if (ptx::bar_sync_or(bar_id, 32 * P, !ok || *abort_flag)) {
                fail = true;
                break;
            }
            // ||H D x||^2 = d ||x||^2; the normalised rotated coordinate is y / ||H D x||
            float ssq = sm.ssq[kb][0][vrow] + sm.ssq[kb][1][vrow];
            if constexpr (P == 4) ssq += sm.ssq[kb][2][vrow] + sm.ssq[kb][3][vrow];
            const bool nz = ssq > 0.f;
            const float sc = nz ? rsqrtf(ssq) : 0.f;
            const float cs = nz ? p.c[B == 2 ? 2 : 1] : 0.f;   // inner level (b = 2) / the level (b = 1)
            const float cb = nz ? p.c[B == 2 ? 3 : 1] : 0.f;   // outer level
            const float dcb = cs - cb;
            // Code bits in chains of 16 coordinates: np (y < 0), mp (inner level). Coordinates
            // go in pairs through f32x2 arithmetic: ys = y sc; inner iff ys^2 < t2^2; the residual
            // is r = ys - sign(y) c, c the inner or outer level.
            uint32_t np[C / 16], mp[C / 16];
#pragma unroll
            for (int g = 0; g < C / 16; ++g) np[g] = mp[g] = 0u;
            float2 r2[C / 2];
            const float2 sc2 = f2(sc, sc);
            const float2 nt2 = f2(-t2 * t2, -t2 * t2);
            const float2 dcb2 = f2(dcb, dcb), cb2 = f2(cb, cb);
#pragma unroll
            for (int i = 7; i >= 0; --i) {
#pragma unroll
                for (int g = C / 16 - 1; g >= 0; --g) {
                    const int pi = 8 * g + i;   // coordinates 2 pi, 2 pi + 1
                    const uint32_t yb0 = a[2 * pi], yb1 = a[2 * pi + 1];
                    const float2 ys = __fmul2_rn(f2(__uint_as_float(yb0), __uint_as_float(yb1)), sc2);
                    np[g] = __funnelshift_l(yb1, np[g], 1);   // bit: y < 0
                    np[g] = __funnelshift_l(yb0, np[g], 1);
                    float2 mag = cb2;
                    if constexpr (B == 2) {
                        const float2 dd = __ffma2_rn(ys, ys, nt2);   // < 0: inner level
                        mp[g] = __funnelshift_l(__float_as_uint(dd.y), mp[g], 1);
                        mp[g] = __funnelshift_l(__float_as_uint(dd.x), mp[g], 1);
                        // exactly 1 (inner) or 0: a nonzero dd is far above the subnormal range
                        const float2 st = f2(__saturatef(dd.x * -0x1p126f), __saturatef(dd.y * -0x1p126f));
                        mag = __ffma2_rn(st, dcb2, cb2);
                    }
                    // -sign(y) c
                    const float2 nsm = f2(__uint_as_float(__float_as_uint(mag.x) | (~yb0 & 0x80000000u)),
                                          __uint_as_float(__float_as_uint(mag.y) | (~yb1 & 0x80000000u)));
                    r2[pi] = __fadd2_rn(ys, nsm);
                }
            }
            if (row < p.n) {
                uint32_t cw[B * C / 32];
#pragma unroll
                for (int h2 = 0; h2 < C / 32; ++h2) {
                    const uint32_t n32 = np[2 * h2] | (np[2 * h2 + 1] << 16);
                    if constexpr (B == 2) {
                        const uint32_t m32 = mp[2 * h2] | (mp[2 * h2 + 1] << 16);
                        const uint32_t hb = ~n32, lb = ~(n32 ^ m32);
                        cw[2 * h2] = spread16(lb) | (spread16(hb) << 1);
                        cw[2 * h2 + 1] = spread16(lb >> 16) | (spread16(hb >> 16) << 1);
                    } else {
                        cw[h2] = ~n32;
                    }
                }
                uint8_t* dst = p.codes + row * (B * 16) + part * (B * C / 8);
                if constexpr (B * C / 32 == 4) *reinterpret_cast<uint4*>(dst) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
                else if constexpr (B * C / 32 == 2) *reinterpret_cast<uint2*>(dst) = make_uint2(cw[0], cw[1]);
                else *reinterpret_cast<uint32_t*>(dst) = cw[0];
                if (part == 0) p.norms[row] = sqrtf(ssq) * p.rsqrt_d;
            }
            if constexpr (PROD) {
                float2 e0 = f2(0.f, 0.f), e1 = f2(0.f, 0.f);
                uint32_t hi[C / 2], lo[C / 2];
#pragma unroll
                for (int i = 0; i < C / 2; ++i) {
                    const float2 rp = r2[i];
                    if (i & 1) e1 = __ffma2_rn(rp, rp, e1);
                    else e0 = __ffma2_rn(rp, rp, e0);
                    const __nv_bfloat162 h = __float22bfloat162_rn(rp);
                    const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h);
                    const float2 hf = f2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xffff0000u));
                    const float2 l = __ffma2_rn(hf, f2(-1.f, -1.f), rp);
                    const __nv_bfloat162 lb = __float22bfloat162_rn(l);
                    hi[i] = hb;
                    lo[i] = *reinterpret_cast<const uint32_t*>(&lb);
                }
                sm.rsq[kb][part][vrow] = (e0.x + e0.y) + (e1.x + e1.y);
                const uint32_t hl = t_lane + 256u + (uint32_t)kb * 128u;
                if constexpr (C / 2 == 32) {
                    ptx::tmem_st32(hl + part * 32, hi);
                    ptx::tmem_st32(hl + 64 + part * 32, lo);
                } else {
                    ptx::tmem_st16(hl + part * 16, *reinterpret_cast<uint32_t(*)[16]>(hi));
                    ptx::tmem_st16(hl + 64 + part * 16, *reinterpret_cast<uint32_t(*)[16]>(lo));
                }
                ptx::tmem_wait_st();
                bool sok = true;
                if (k > 0) sok = emit_signs((uint32_t)((k - 1) & 1), prev_row, prev_nz);   // previous tile
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&sm.bar_hl[kb]);
                if (ptx::bar_sync_or(bar_id, 32 * P, !sok || *abort_flag)) {
                    fail = true;
                    break;
                }
                if (part == 0 && row < p.n) {
                    float rs = sm.rsq[kb][0][vrow] + sm.rsq[kb][1][vrow];
                    if constexpr (P == 4) rs += sm.rsq[kb][2][vrow] + sm.rsq[kb][3][vrow];
                    p.rnorms[row] = sqrtf(rs);
                }
                prev_row = row;
                prev_nz = nz;
            }
        }
        if constexpr (PROD) {
            if (!fail && mytiles > 0 && !emit_signs((uint32_t)((mytiles - 1) & 1), prev_row, prev_nz)) fail = true;
        }
        if (fail) {
            *abort_flag = 1;
            if (lane == 0) atomicExch(&g_tq_device_error, 1);
        }
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, kT4Cols);
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled_fn() {
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

int sm_count() {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

template <int B, bool PROD>
int launch_tc(const DevState& st, const void* x, int64_t n, int64_t ld, uint8_t* codes, uint8_t* qjl, float* norms,
              float* rnorms, cudaStream_t stream) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return (int)cudaErrorNotSupported;
    CUtensorMap tmap;
    const cuuint64_t gdim[2] = {(cuuint64_t)kD, (cuuint64_t)n};
    const cuuint64_t gstride[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {64, kTile};
    const cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return (int)cudaErrorInvalidValue;
    TcParams p;
    p.codes = codes;
    p.qjl = qjl;
    p.norms = norms;
    p.rnorms = rnorms;
    p.s = reinterpret_cast<const uint16_t*>(st.s);
    p.n = n;
    p.rsqrt_d = st.rsqrt_d;
    for (int i = 0; i < 16; ++i) {
        p.t[i] = (i < st.L - 1) ? st.t[i] : 0.f;
        p.c[i] = (i < st.L) ? st.c[i] : 0.f;
    }
    for (int i = 0; i < 64; ++i) {
        const bool n0 = (st.signs[(2 * i) >> 5] >> ((2 * i) & 31)) & 1u;
        const bool n1 = (st.signs[(2 * i + 1) >> 5] >> ((2 * i + 1) & 31)) & 1u;
        p.sgn[i] = (n0 ? 0x8000u : 0u) | (n1 ? 0x80000000u : 0u);
    }
    constexpr bool kTwo = (B == 1 || B == 2);
    const size_t smem = (kTwo ? sizeof(TcSmem4) : sizeof(TcSmem)) + 1024;
    auto kern = kTwo ? encode_tc4_kernel<(B <= 2 ? B : 2), PROD, kT4P> : encode_tc_kernel<B, PROD>;
    static int attr_set_for_device = -1;   // per instantiation
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_set_for_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return (int)e;
        attr_set_for_device = dev;
    }
    const int64_t ntiles = (n + kTile - 1) / kTile;
    const int grid = (int)std::min<int64_t>(ntiles, (int64_t)sm_count() * (kTwo ? 1 : 2));
    kern<<<grid, kTwo ? T4<kT4P>::kThreads : kTile, smem, stream>>>(tmap, p);
    return (int)cudaGetLastError();
}

}  // namespace

// True when the tensor-core encoder handles this configuration.
bool encode_tc_supported(const DevState& st, int dtype, int64_t n, int64_t ld) {
    if (st.d != kD || st.rot != TQ_ROT_RHT || dtype != TQ_BF16) return false;
    if (n <= 0 || n >= (int64_t)1 << 31 || ld < kD) return false;
    if (st.mode == TQ_PROD) return st.mat_dtype == TQ_BF16 && st.b_mse >= 1 && st.b_mse <= 3;
    return st.b_mse >= 1 && st.b_mse <= 4;
}

int launch_encode_tc(const DevState& st, const void* x, int64_t n, int64_t ld, uint8_t* codes, uint8_t* qjl,
                     float* norms, float* rnorms, void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    if (st.mode == TQ_PROD) {
        switch (st.b_mse) {
            case 1: return launch_tc<1, true>(st, x, n, ld, codes, qjl, norms, rnorms, s);
            case 2: return launch_tc<2, true>(st, x, n, ld, codes, qjl, norms, rnorms, s);
            case 3: return launch_tc<3, true>(st, x, n, ld, codes, qjl, norms, rnorms, s);
            default: return (int)cudaErrorInvalidValue;
        }
    }
    switch (st.b_mse) {
        case 1: return launch_tc<1, false>(st, x, n, ld, codes, qjl, norms, rnorms, s);
        case 2: return launch_tc<2, false>(st, x, n, ld, codes, qjl, norms, rnorms, s);
        case 3: return launch_tc<3, false>(st, x, n, ld, codes, qjl, norms, rnorms, s);
        case 4: return launch_tc<4, false>(st, x, n, ld, codes, qjl, norms, rnorms, s);
        default: return (int)cudaErrorInvalidValue;
    }
}

namespace {
// A wait that can only run out: one thread waits on the first phase of an mbarrier nothing
// arrives on, gives up after limit_ns and records the error word, as every bounded wait of
// the library does on a timeout.
__global__ void expired_wait_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        ptx::mbar_init(&bar, 1);
        ptx::fence_mbar_init();
        if (!ptx::mbar_wait(&bar, 0u, limit_ns)) atomicExch(&g_tq_device_error, 1);
    }
}
}  // namespace

int launch_expired_wait(uint64_t limit_ns, void* stream) {
    expired_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(limit_ns);
    return (int)cudaGetLastError();
}

// Reads and clears the error words of all kernels with bounded waits (one word per
// translation unit: the library is built without relocatable device code).
int read_device_error(int* flag) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_tq_device_error, sizeof(int));
    if (e != cudaSuccess) return (int)e;
    if (v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_tq_device_error, &zero, sizeof(int));
        if (e != cudaSuccess) return (int)e;
    }
    int g = 0, s = 0;
    int rc = take_device_error_gemm(&g);
    if (rc) return rc;
    rc = take_device_error_search(&s);
    if (rc) return rc;
    *flag = v | g | s;
    return 0;
}

}  // namespace tq
