// Tensor-core encoders for d = 128 with the randomized Hadamard rotation and bf16 input
// (TurboQuant_prod with S stored bf16, or TurboQuant_mse).
//
// TurboQuant review (Jump2Paper): Theorem 1 (rotate, per-coordinate Lloyd-Max code),
// Definition 1 + Theorem 2 (QJL signs of S r on the residual, ||r|| kept); AI Trends
// summary of the TurboQuant video (L2 normalise + RHT).
//
// Two kernels:
//   encode_duo_kernel (b_mse = 1, 2): the rotation y = (H diag(eps)) x and S r both run on the
//     tensor core; two teams of warps per SM alternate between quantizing and waiting for
//     the MMAs (described at the kernel).
//   encode_tc_kernel (b_mse = 3, 4): a CTA of 128 threads owns tiles of 128 vectors; thread t
//     is vector t of the tile, which is also TMEM lane t of the MMA accumulator.
//     1. TMA (128-byte swizzle) brings the tile's bf16 rows into shared memory, two stages
//        deep, so the next tile streams in while this one is computed.
//     2. Each thread reads its row, flips the RHT signs on the packed bf16 bits, converts to
//        fp32, takes ||x||, runs the 7-stage Walsh-Hadamard butterfly in registers (paired
//        fp32 adds), scales by 1/(sqrt(d) ||x||), quantizes against the Lloyd-Max
//        boundaries, and writes codes and norms.
//     3. prod: the residual r = y - c[idx] is split as r = hi + lo (both bf16,
//        lo = bf16(r - hi)) and written to TMEM as the MMA A operand; one thread issues 16
//        tcgen05.mma (K = 128 for hi, then for lo) against S held in shared memory (K-major
//        core matrices), accumulating S r in fp32 in TMEM. The split keeps the error of S r
//        at about 2^-16 |S||r|, so a sign is decided as fp32 arithmetic on r would decide it.
//     4. Each thread reads its 128 accumulator columns back (tcgen05.ld) and packs the signs
//        [(S r)_j >= 0] into 16 bytes.
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
// Two-team tensor-core encoder (b_mse = 1 or 2). One persistent CTA per SM owns all 512
// TMEM columns and runs two independent pipelines ("teams") over alternate tiles of 128
// vectors. The two quantizing warps that share an SM sub-partition (and a TMEM lane
// quadrant) belong to different teams and so are at different points of their tiles:
// while one waits for the tensor core, the other computes, and no warp waits for another.
//   team t: warps 4t .. 4t+3 quantize (warp 4t+q owns TMEM lanes 32q .. 32q+31: one thread
//   per vector, all 128 coordinates); lane 0 of warp 8+t streams the team's tiles with TMA
//   (two stages) and issues its MMAs.
//   TMEM columns of team t: two regions of 128, [256t, 256t+128) and [256t+128, 256t+256).
//   For tile i the region i % 2 (Y) holds y = (H D) x and then S r, the other (HL) the
//   residual operand (hi in 64 columns, lo in 64); the roles swap every tile (mse keeps y in
//   the first region).
// Per tile: rotation MMA into Y; the warps read y twice (||y||^2, then 32 coordinates at a
// time: level bits, codes, and the residual split r = hi + lo, both bf16, written to HL); the
// S r MMA (16 MMAs: K = 128 for hi, then for lo; A from TMEM) accumulates into Y in fp32; the
// warps read the signs. The next tile's rotation goes to this tile's HL region as soon as S r
// has read it, so it runs while the warps read the signs. The split keeps the error of S r
// at about 2^-16 |S| |r|, so a sign is decided as fp32 arithmetic on r would decide it. The
// two producers are coupled so that the teams' quantize passes alternate (one team computes
// while the other waits for the tensor core).
// ------------------------------------------------------------------------------------
constexpr int kDuoThreads = 10 * 32;   // 8 quantizing warps + 2 producer warps
constexpr uint32_t kDuoCols = 512;

struct __align__(1024) TcSmemDuo {
    uint8_t x[2][2][2][kTile * 128];   // [team][stage][half]: 128 rows x 128 bytes, 128B-swizzled
    uint8_t hd[kD * kD * 2];           // H diag(eps), B operand (K-major core matrices)
    uint8_t s[kD * kD * 2];            // S, B operand
    uint64_t bar_x[2][2];              // [team][stage]: tile landed
    uint64_t bar_xfree[2][2];          // [team][stage]: the rotation MMA has read the stage
    uint64_t bar_y[2];                 // y of the team's current tile is in Y_t
    uint64_t bar_hl[2];                // residual written and y read (one arrival per warp)
    uint64_t bar_d[2];                 // S r is in Y_t
    uint64_t bar_free[2];              // mse: Y_t read to the end (one arrival per warp)
    uint64_t bar_mid[2];               // half of the quantize pass done (one arrival per warp)
    uint32_t tmem_base;
    int abort;
};

// Sign word of 32 accumulator columns: bit j = [v_j >= 0] read from the fp32 sign bit.
__device__ __forceinline__ uint32_t sign_word(const uint32_t (&d)[32]) {
    uint32_t z0 = 0u, z1 = 0u;
#pragma unroll
    for (int j = 15; j >= 0; --j) {
        z0 = __funnelshift_l(d[j], z0, 1);
        z1 = __funnelshift_l(d[j + 16], z1, 1);
    }
    return ~(z0 | (z1 << 16));
}

// The coordinates of a tile in one or two groups (an outlier-channel split): group 0 holds
// the first m32 chunks of 32 output coordinates, group 1 the rest. Without a split, group 0
// is everything and the rotation operand is H diag(eps) built from TcParams::sgn.
struct DuoGroups {
    const uint16_t* pmat;   // split: rotation operand [128 outputs][128 channels] bf16, else null
    int m32;                // chunks in group 0
    uint8_t* codes[2];
    uint8_t* qjl[2];
    float* norms[2];
    float* rnorms[2];
    int code_bytes[2];      // row strides of the planes
    int qjl_bytes[2];
    float t2[2];            // b = 2: boundary between the inner and outer level
    float cs[2];            // inner level (b = 2) / the level (b = 1)
    float cb[2];            // outer level
    float rsqrt_d[2];       // 1 / sqrt(group dimension): ||x_g|| = ||y_g|| / sqrt(d_g)
};

// Quantizes 32 coordinates y (fp32 bits) of one vector at BC bits: code words w0 (and w1 for
// BC = 2), and for prod the residual r = ys - sign(y) c split into bf16 hi + lo and its squares
// added to e0 / e1. Level bits go into one chain per 16 coordinates with funnel shifts: BC = 2
// puts (y < 0, inner) of coordinate j at bits 2j+1, 2j; BC = 1 the bit y < 0 at bit j. Pairs of
// coordinates go through f32x2 arithmetic: ys = y sc; inner iff ys^2 < t2^2.
template <int BC, bool PROD>
__device__ __forceinline__ void duo_quant_chunk(const uint32_t (&y)[32], float2 sc2, float2 nt2, float2 dcb2,
                                                float2 cb2, uint32_t& w0, uint32_t& w1, float2& e0, float2& e1,
                                                uint32_t (&hi)[16], uint32_t (&lo)[16]) {
    uint32_t wd[2] = {0u, 0u};
    float2 r2[16];
#pragma unroll
    for (int ii = 7; ii >= 0; --ii) {
#pragma unroll
        for (int g = 1; g >= 0; --g) {
            const int pi = 8 * g + ii;   // coordinates 2 pi, 2 pi + 1 of the chunk
            const uint32_t yb0 = y[2 * pi], yb1 = y[2 * pi + 1];
            const float2 ys = __fmul2_rn(f2(__uint_as_float(yb0), __uint_as_float(yb1)), sc2);
            float2 mag = cb2;
            if constexpr (BC == 2) {
                const float2 dd = __ffma2_rn(ys, ys, nt2);   // < 0: inner level
                wd[g] = __funnelshift_l(yb1, wd[g], 1);
                wd[g] = __funnelshift_l(__float_as_uint(dd.y), wd[g], 1);
                wd[g] = __funnelshift_l(yb0, wd[g], 1);
                wd[g] = __funnelshift_l(__float_as_uint(dd.x), wd[g], 1);
                // exactly 1 (inner) or 0: a nonzero dd is far above the subnormal range
                const float2 stp = f2(__saturatef(dd.x * -0x1p126f), __saturatef(dd.y * -0x1p126f));
                mag = __ffma2_rn(stp, dcb2, cb2);
            } else {
                wd[g] = __funnelshift_l(yb1, wd[g], 1);
                wd[g] = __funnelshift_l(yb0, wd[g], 1);
            }
            // -sign(y) c
            const float2 nsm = f2(__uint_as_float(__float_as_uint(mag.x) | (~yb0 & 0x80000000u)),
                                  __uint_as_float(__float_as_uint(mag.y) | (~yb1 & 0x80000000u)));
            r2[pi] = __fadd2_rn(ys, nsm);
        }
    }
    if constexpr (BC == 2) {
        // code = 2 [y >= 0] + [y >= 0] xnor [inner]: index of the level, LSB first
        w0 = (~wd[0] & 0xAAAAAAAAu) | (~(wd[0] ^ (wd[0] >> 1)) & 0x55555555u);
        w1 = (~wd[1] & 0xAAAAAAAAu) | (~(wd[1] ^ (wd[1] >> 1)) & 0x55555555u);
    } else {
        w0 = ~(wd[0] | (wd[1] << 16));
    }
    if constexpr (PROD) {
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float2 rp = r2[k];
            if (k & 1) e1 = __ffma2_rn(rp, rp, e1);
            else e0 = __ffma2_rn(rp, rp, e0);
            const __nv_bfloat162 h = __float22bfloat162_rn(rp);
            const uint32_t hb = *reinterpret_cast<const uint32_t*>(&h);
            const float2 hf = f2(__uint_as_float(hb << 16), __uint_as_float(hb & 0xffff0000u));
            const float2 l = __ffma2_rn(hf, f2(-1.f, -1.f), rp);
            const __nv_bfloat162 lb = __float22bfloat162_rn(l);
            hi[k] = hb;
            lo[k] = *reinterpret_cast<const uint32_t*>(&lb);
        }
    }
}

template <int B0, int B1, bool PROD, bool SPLIT>
__global__ void __launch_bounds__(384, 1)   // 384: caps registers at 168 (three warps per sub-partition)
encode_duo_kernel(const __grid_constant__ CUtensorMap tmap, const TcParams p, const DuoGroups gp) {
    static_assert((B0 == 1 || B0 == 2) && (B1 == 1 || B1 == 2), "the two-team encoder covers 1- and 2-bit codes");
    static_assert(SPLIT || B0 == B1, "one code width without a split");
    extern __shared__ uint8_t smem_raw[];
    TcSmemDuo& sm = *reinterpret_cast<TcSmemDuo*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    volatile int* abort_flag = &sm.abort;
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int64_t ntiles = (p.n + kTile - 1) / kTile;
    const int64_t mytiles = (ntiles > (int64_t)blockIdx.x) ? (ntiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

    if (tid == 0) {
        ptx::prefetch_tmap(&tmap);
        for (int t = 0; t < 2; ++t) {
            for (int s = 0; s < 2; ++s) {
                ptx::mbar_init(&sm.bar_x[t][s], 1);
                ptx::mbar_init(&sm.bar_xfree[t][s], 1);
            }
            ptx::mbar_init(&sm.bar_y[t], 1);
            ptx::mbar_init(&sm.bar_hl[t], 4);
            ptx::mbar_init(&sm.bar_d[t], 1);
            ptx::mbar_init(&sm.bar_free[t], 4);
            ptx::mbar_init(&sm.bar_mid[t], 4);
        }
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0) {
        ptx::tmem_alloc(&sm.tmem_base, kDuoCols);
        ptx::tmem_relinquish();
    }
    if constexpr (SPLIT) {
        // the groups' rotations as one operand (row n = output coordinate, K = input channel)
        for (int i = tid; i < kD * 16; i += kDuoThreads) {
            const int row = i >> 4, c = i & 15;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(gp.pmat + row * kD + c * 8));
            *reinterpret_cast<uint4*>(sm.hd + c * 2048 + (row >> 3) * 128 + (row & 7) * 16) = v;
        }
    } else {
        // H diag(eps): entry (n, k) = (-1)^popcount(n & k) * eps_k, at chunk k/8 of row n.
        for (int i = tid; i < kD * kD; i += kDuoThreads) {
            const int n = i >> 7, k = i & 127;
            const uint32_t neg = (__popc(n & k) & 1) ^ ((p.sgn[k >> 1] >> ((k & 1) ? 31 : 15)) & 1u);
            *reinterpret_cast<uint16_t*>(sm.hd + (k >> 3) * 2048 + (n >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2) =
                neg ? 0xBF80u : 0x3F80u;
        }
    }
    if constexpr (PROD) {
        for (int i = tid; i < kD * 16; i += kDuoThreads) {
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

    if (warp >= 8) {
        // ---------------- producer of team t: TMA + MMA issue (one thread) ----------------
        const int t = warp - 8;
        const int64_t nt = (mytiles > t) ? (mytiles - t + 1) / 2 : 0;   // team tiles: local t, t+2, ...
        if (lane == 0) {
            const uint32_t idesc = ptx::idesc_bf16_f32(128, 128);
            const uint32_t s_addr = ptx::smem_addr(sm.s);
            const uint32_t hd_addr = ptx::smem_addr(sm.hd);
            const uint32_t tbase = tmem + 256u * (uint32_t)t;
            uint32_t tma_pend = 0u, tma_par = 0u;   // per stage: load in flight / its phase parity
            bool y_issued = false, d_issued = false;
            uint32_t y_par = 0u, d_par = 0u;
            auto load = [&](int64_t i) {
                const int st = (int)(i & 1);
                const int row0 = (int)((blockIdx.x + (t + 2 * i) * gridDim.x) * kTile);
                ptx::mbar_arrive_expect_tx(&sm.bar_x[t][st], 2 * kTile * 128);
                ptx::tma_load_2d(sm.x[t][st][0], &tmap, 0, row0, &sm.bar_x[t][st]);
                ptx::tma_load_2d(sm.x[t][st][1], &tmap, 64, row0, &sm.bar_x[t][st]);
                tma_pend |= 1u << st;
                tma_par = (tma_par & ~(1u << st)) | ((uint32_t)((i >> 1) & 1) << st);
            };
            for (int64_t i = 0; i < nt && i < 2; ++i) load(i);
            bool ok = true;
            for (int64_t i = 0; i < nt; ++i) {
                const int st = (int)(i & 1);
                const uint32_t xpar = (uint32_t)((i >> 1) & 1);
                ok = ptx::mbar_wait(&sm.bar_x[t][st], xpar);
                if (!ok) break;
                tma_pend &= ~(1u << st);
                // prod: the team's two regions swap roles every tile (y / S r of tile i in region
                // i % 2, its residual in the other); the rotation may overwrite region i % 2 as
                // soon as S r of tile i - 1 (which read it) is done. mse: one region, free once
                // the warps have read it.
                const uint32_t ycol = tbase + (PROD ? 128u * (uint32_t)(i & 1) : 0u);
                const uint32_t hl = tbase + (PROD ? 128u * (uint32_t)((i + 1) & 1) : 128u);
                if (i > 0) {
                    ok = ptx::mbar_wait(PROD ? &sm.bar_d[t] : &sm.bar_free[t], (uint32_t)((i - 1) & 1)) &&
                         !*abort_flag;
                    if (!ok) break;
                }
                if constexpr (PROD) {
                    // Stagger the teams: team 1's tile i starts when team 0 is half way through
                    // quantizing its tile i, team 0's tile i when team 1 is half way through its
                    // tile i - 1. One team computes while the other waits for the tensor core.
                    if (t == 1 || i > 0) {
                        ok = ptx::mbar_wait(&sm.bar_mid[t ^ 1], (uint32_t)((t == 1 ? i : i - 1) & 1)) && !*abort_flag;
                        if (!ok) break;
                    }
                }
                ptx::tc_fence_after();
                const uint32_t xa0 = ptx::smem_addr(sm.x[t][st][0]), xa1 = ptx::smem_addr(sm.x[t][st][1]);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_ss(ycol, ptx::smem_desc_kmajor_sw128(((kk < 4) ? xa0 : xa1) + (kk & 3) * 32),
                                ptx::smem_desc_kmajor(hd_addr + kk * 2 * 2048, 2048, 128), idesc, kk > 0 ? 1u : 0u);
                ptx::mma_commit(&sm.bar_xfree[t][st]);
                ptx::mma_commit(&sm.bar_y[t]);
                y_issued = true;
                y_par = (uint32_t)(i & 1);
                if (i + 2 < nt) {   // refill the stage once the rotation has read it
                    ok = ptx::mbar_wait(&sm.bar_xfree[t][st], xpar);
                    if (!ok) break;
                    load(i + 2);
                }
                if constexpr (PROD) {
                    ok = ptx::mbar_wait(&sm.bar_hl[t], (uint32_t)(i & 1)) && !*abort_flag;
                    if (!ok) break;
                    ptx::tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        ptx::mma_ts(ycol, hl + kk * 8, ptx::smem_desc_kmajor(s_addr + kk * 2 * 2048, 2048, 128),
                                    idesc, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        ptx::mma_ts(ycol, hl + 64 + kk * 8,
                                    ptx::smem_desc_kmajor(s_addr + kk * 2 * 2048, 2048, 128), idesc, 1u);
                    ptx::mma_commit(&sm.bar_d[t]);
                    d_issued = true;
                    d_par = (uint32_t)(i & 1);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                atomicExch(&g_tq_device_error, 1);
            }
            // Drain: every copy and MMA this thread started has finished before the CTA
            // releases TMEM and shared memory.
            for (int st = 0; st < 2; ++st)
                if ((tma_pend >> st) & 1u) (void)ptx::mbar_wait(&sm.bar_x[t][st], (tma_par >> st) & 1u);
            if (y_issued) (void)ptx::mbar_wait(&sm.bar_y[t], y_par);   // committed after the stage release
            if (d_issued) (void)ptx::mbar_wait(&sm.bar_d[t], d_par);
        }
    } else {
        // ---------------- quantizing warps of team t ----------------
        const int t = warp >> 2, quad = warp & 3;
        const int64_t nt = (mytiles > t) ? (mytiles - t + 1) / 2 : 0;
        const int vrow = quad * 32 + lane;
        const uint32_t t_lane = tmem + ((uint32_t)(quad * 32) << 16);
        const uint32_t tbase = t_lane + 256u * (uint32_t)t;
        const int m32 = SPLIT ? gp.m32 : 4;   // chunks of group 0
        bool fail = false;
        // MMA results (read through tcgen05.ld after a tcgen05 fence): one lane waits, and the
        // warp barrier orders the other lanes after it.
        auto wait_bar = [&](uint64_t* bar, uint32_t par) -> bool {
            bool ok = true;
            if (lane == 0) ok = ptx::mbar_wait(bar, par) && !*abort_flag;
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            __syncwarp();
            return ok;
        };
        for (int64_t i = 0; i < nt; ++i) {
            const int64_t row = (blockIdx.x + (t + 2 * i) * gridDim.x) * kTile + vrow;
            // y (then S r) and the residual: regions i % 2 and (i + 1) % 2 for prod
            const uint32_t ycol = tbase + (PROD ? 128u * (uint32_t)(i & 1) : 0u);
            const uint32_t hlc = tbase + (PROD ? 128u * (uint32_t)((i + 1) & 1) : 128u);
            if (!wait_bar(&sm.bar_y[t], (uint32_t)(i & 1))) {
                fail = true;
                break;
            }
            ptx::tc_fence_after();
            // ||y_g||^2 per group (||H D x||^2 = d ||x||^2); the normalised rotated coordinate
            // is y / ||y_g||. qc: sums per chunk of 32 coordinates.
            constexpr bool kSignsOnly = (!SPLIT && B0 == 1 && !PROD);   // the code is the sign of y: one pass
            float qc[4];
            uint32_t cw[8];   // code words in chunk order: chunk c at cw[2c] (and cw[2c + 1] at 2 bits)
            float2 q0 = f2(0.f, 0.f), q1 = f2(0.f, 0.f);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t a0[32], a1[32];
                ptx::tmem_ld32(ycol + h * 64, a0);
                ptx::tmem_ld32(ycol + h * 64 + 32, a1);
                ptx::tmem_wait_ld();
                if constexpr (SPLIT) q0 = q1 = f2(0.f, 0.f);   // per chunk
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const float2 u0 = f2(__uint_as_float(a0[2 * k]), __uint_as_float(a0[2 * k + 1]));
                    const float2 u1 = f2(__uint_as_float(a1[2 * k]), __uint_as_float(a1[2 * k + 1]));
                    q0 = __ffma2_rn(u0, u0, q0);
                    q1 = __ffma2_rn(u1, u1, q1);
                }
                qc[2 * h] = q0.x + q0.y;
                qc[2 * h + 1] = q1.x + q1.y;
                if constexpr (kSignsOnly) {
                    cw[4 * h] = sign_word(a0);   // bit j = [y_j >= 0] = the 1-bit code
                    cw[4 * h + 2] = sign_word(a1);
                }
            }
            float ssq[2] = {0.f, 0.f};
            if constexpr (SPLIT) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    ssq[0] += (c < m32) ? qc[c] : 0.f;
                    ssq[1] += (c < m32) ? 0.f : qc[c];
                }
            } else {
                ssq[0] = (q0.x + q0.y) + (q1.x + q1.y);
            }
            if constexpr (kSignsOnly) {   // y is read to the end: the next rotation may go
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&sm.bar_free[t]);
            }
            bool nz[2];
            float sc[2], cs[2], cb[2], t2[2];
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                nz[g] = ssq[g] > 0.f;
                sc[g] = nz[g] ? rsqrtf(ssq[g]) : 0.f;
                cs[g] = nz[g] ? gp.cs[g] : 0.f;
                cb[g] = nz[g] ? gp.cb[g] : 0.f;
                t2[g] = gp.t2[g];
            }
            float rs[2] = {0.f, 0.f};   // ||r_g||^2
            float2 e0 = f2(0.f, 0.f), e1 = f2(0.f, 0.f);   // ||r||^2 in pairs (per chunk for a split)
            // 32 coordinates at a time, each at its group's width, scale and levels.
#pragma unroll
            for (int c = 0; c < (kSignsOnly ? 0 : 4); ++c) {
                uint32_t y[32];
                ptx::tmem_ld32(ycol + 32 * c, y);
                ptx::tmem_wait_ld();
                const bool g1 = SPLIT && c >= m32;   // the chunk's group (selects, no indexing)
                const float scg = g1 ? sc[1] : sc[0], csg = g1 ? cs[1] : cs[0], cbg = g1 ? cb[1] : cb[0];
                const float t2g = g1 ? t2[1] : t2[0];
                const float2 sc2 = f2(scg, scg);
                const float2 nt2 = f2(-t2g * t2g, -t2g * t2g);
                const float2 dcb2 = f2(csg - cbg, csg - cbg), cb2 = f2(cbg, cbg);
                uint32_t hi[16], lo[16];
                if constexpr (SPLIT) e0 = e1 = f2(0.f, 0.f);
                if (PROD && c == 1) {   // half way: the other team's next rotation may go
                    __syncwarp();
                    if (lane == 0) ptx::mbar_arrive(&sm.bar_mid[t]);
                }
                if (!g1)
                    duo_quant_chunk<B0, PROD>(y, sc2, nt2, dcb2, cb2, cw[2 * c], cw[2 * c + 1], e0, e1, hi, lo);
                else
                    duo_quant_chunk<B1, PROD>(y, sc2, nt2, dcb2, cb2, cw[2 * c], cw[2 * c + 1], e0, e1, hi, lo);
                if constexpr (PROD) {
                    if constexpr (SPLIT) {
                        const float ec = (e0.x + e0.y) + (e1.x + e1.y);
                        rs[0] += g1 ? 0.f : ec;
                        rs[1] += g1 ? ec : 0.f;
                    }
                    ptx::tmem_st16(hlc + 16 * c, hi);
                    ptx::tmem_st16(hlc + 64 + 16 * c, lo);
                }
            }
            if constexpr (PROD && !SPLIT) rs[0] = (e0.x + e0.y) + (e1.x + e1.y);
            if constexpr (PROD) ptx::tmem_wait_st();
            if constexpr (!kSignsOnly) {
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(PROD ? &sm.bar_hl[t] : &sm.bar_free[t]);
            }
            if (row < p.n) {
                if constexpr (!SPLIT) {
                    if constexpr (B0 == 2) {
                        uint4* dst = reinterpret_cast<uint4*>(gp.codes[0] + row * 32);
                        dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
                        dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
                    } else {
                        *reinterpret_cast<uint4*>(gp.codes[0] + row * 16) = make_uint4(cw[0], cw[2], cw[4], cw[6]);
                    }
                } else {
                    uint32_t* dst0 = reinterpret_cast<uint32_t*>(gp.codes[0] + row * gp.code_bytes[0]);
                    uint32_t* dst1 = reinterpret_cast<uint32_t*>(gp.codes[1] + row * gp.code_bytes[1]);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if (c < m32) {
                            if constexpr (B0 == 2) {
                                dst0[2 * c] = cw[2 * c];
                                dst0[2 * c + 1] = cw[2 * c + 1];
                            } else {
                                dst0[c] = cw[2 * c];
                            }
                        } else {
                            if constexpr (B1 == 2) {
                                dst1[2 * (c - m32)] = cw[2 * c];
                                dst1[2 * (c - m32) + 1] = cw[2 * c + 1];
                            } else {
                                dst1[c - m32] = cw[2 * c];
                            }
                        }
                    }
                    gp.norms[1][row] = sqrtf(ssq[1]) * gp.rsqrt_d[1];
                }
                gp.norms[0][row] = sqrtf(ssq[0]) * gp.rsqrt_d[0];
            }
            if constexpr (PROD) {
                if (row < p.n) {
                    gp.rnorms[0][row] = sqrtf(rs[0]);
                    if constexpr (SPLIT) gp.rnorms[1][row] = sqrtf(rs[1]);
                }
                // signs of S r, all ones for a zero vector (group)
                if (!wait_bar(&sm.bar_d[t], (uint32_t)(i & 1))) {
                    fail = true;
                    break;
                }
                ptx::tc_fence_after();
                uint32_t zw[4];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t d0[32], d1[32];
                    ptx::tmem_ld32(ycol + h * 64, d0);
                    ptx::tmem_ld32(ycol + h * 64 + 32, d1);
                    ptx::tmem_wait_ld();
                    zw[2 * h] = sign_word(d0);
                    zw[2 * h + 1] = sign_word(d1);
                }
                if (row < p.n) {
                    if constexpr (!SPLIT) {
                        *reinterpret_cast<uint4*>(gp.qjl[0] + row * 16) =
                            nz[0] ? make_uint4(zw[0], zw[1], zw[2], zw[3]) : make_uint4(~0u, ~0u, ~0u, ~0u);
                    } else {
                        uint32_t* q0 = reinterpret_cast<uint32_t*>(gp.qjl[0] + row * gp.qjl_bytes[0]);
                        uint32_t* q1 = reinterpret_cast<uint32_t*>(gp.qjl[1] + row * gp.qjl_bytes[1]);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            if (c < m32) q0[c] = nz[0] ? zw[c] : ~0u;
                            else q1[c - m32] = nz[1] ? zw[c] : ~0u;
                        }
                    }
                }
            }
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
        ptx::tmem_dealloc(tmem, kDuoCols);
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

// Levels of group g of the two-team encoder from a state with b_mse 1 or 2.
void duo_levels(const DevState& st, DuoGroups& gp, int g) {
    gp.t2[g] = (st.b_mse == 2) ? st.t[2] : 0.f;
    gp.cs[g] = st.c[st.b_mse == 2 ? 2 : 1];
    gp.cb[g] = st.c[st.b_mse == 2 ? 3 : 1];
    gp.rsqrt_d[g] = st.rsqrt_d;
}

bool make_tmap(CUtensorMap* tmap, const void* x, int64_t n, int64_t ld) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)kD, (cuuint64_t)n};
    const cuuint64_t gstride[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {64, kTile};
    const cuuint32_t estride[2] = {1, 1};
    return enc(tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), gdim, gstride, box, estride,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int B0, int B1, bool PROD, bool SPLIT>
int launch_duo(const CUtensorMap& tmap, const TcParams& p, const DuoGroups& gp, cudaStream_t stream) {
    auto kern = encode_duo_kernel<B0, B1, PROD, SPLIT>;
    const size_t smem = sizeof(TcSmemDuo) + 1024;
    static int attr_set_for_device = -1;   // per instantiation
    int dev = 0;
    cudaGetDevice(&dev);
    if (attr_set_for_device != dev) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return (int)e;
        attr_set_for_device = dev;
    }
    const int64_t ntiles = (p.n + kTile - 1) / kTile;
    const int grid = (int)std::min<int64_t>(ntiles, (int64_t)sm_count());
    kern<<<grid, kDuoThreads, smem, stream>>>(tmap, p, gp);
    return (int)cudaGetLastError();
}

template <int B, bool PROD>
int launch_tc(const DevState& st, const void* x, int64_t n, int64_t ld, uint8_t* codes, uint8_t* qjl, float* norms,
              float* rnorms, cudaStream_t stream) {
    CUtensorMap tmap;
    if (!encode_tiled_fn()) return (int)cudaErrorNotSupported;
    if (!make_tmap(&tmap, x, n, ld)) return (int)cudaErrorInvalidValue;
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
    if constexpr (B == 1 || B == 2) {
        DuoGroups gp = {};
        gp.pmat = nullptr;
        gp.m32 = 4;
        for (int g = 0; g < 2; ++g) {   // group 1 is empty without a split
            gp.codes[g] = codes;
            gp.qjl[g] = qjl;
            gp.norms[g] = norms;
            gp.rnorms[g] = rnorms;
            gp.code_bytes[g] = st.code_bytes;
            gp.qjl_bytes[g] = st.qjl_bytes;
            duo_levels(st, gp, g);
        }
        return launch_duo<B, B, PROD, false>(tmap, p, gp, stream);
    } else {
        auto kern = encode_tc_kernel<B, PROD>;
        const size_t smem = sizeof(TcSmem) + 1024;
        static int attr_set_for_device = -1;   // per instantiation
        int dev = 0;
        cudaGetDevice(&dev);
        if (attr_set_for_device != dev) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return (int)e;
            attr_set_for_device = dev;
        }
        const int64_t ntiles = (n + kTile - 1) / kTile;
        const int grid = (int)std::min<int64_t>(ntiles, (int64_t)sm_count() * 2);
        kern<<<grid, kTile, smem, stream>>>(tmap, p);
        return (int)cudaGetLastError();
    }
}

template <int B0, bool PROD>
int launch_split_b1(int b1, const CUtensorMap& tmap, const TcParams& p, const DuoGroups& gp, cudaStream_t s) {
    if (b1 == 1) return launch_duo<B0, 1, PROD, true>(tmap, p, gp, s);
    return launch_duo<B0, 2, PROD, true>(tmap, p, gp, s);
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

// The outlier-channel split of a 128-channel bf16 input on the two-team encoder: group 0
// (state so, the first m output coordinates) and group 1 (si, the other 128 - m). pmat is the
// two groups' rotations as one [128][128] bf16 operand (each row a Hadamard row times the
// group's signs, placed at the group's channels), sbd the block-diagonal [128][128] S.
bool split_tc_supported(const DevState& so, const DevState& si, int m) {
    const bool prod = so.mode == TQ_PROD;
    if (so.rot != TQ_ROT_RHT || si.rot != TQ_ROT_RHT || so.mode != si.mode) return false;
    if (m % 32 != 0 || m < 32 || m > 96 || so.d != m || si.d != kD - m) return false;
    if (so.b_mse < 1 || so.b_mse > 2 || si.b_mse < 1 || si.b_mse > 2) return false;
    return !prod || (so.mat_dtype == TQ_BF16 && si.mat_dtype == TQ_BF16);
}

int launch_encode_split_tc(const DevState& so, const DevState& si, const uint16_t* pmat, const uint16_t* sbd,
                           const void* x, int64_t n, int64_t ld, uint8_t* const codes[2], uint8_t* const qjl[2],
                           float* const norms[2], float* const rnorms[2], void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    CUtensorMap tmap;
    if (!encode_tiled_fn()) return (int)cudaErrorNotSupported;
    if (!make_tmap(&tmap, x, n, ld)) return (int)cudaErrorInvalidValue;
    TcParams p = {};
    p.s = sbd;
    p.n = n;
    DuoGroups gp = {};
    gp.pmat = pmat;
    gp.m32 = so.d / 32;
    const DevState* st[2] = {&so, &si};
    for (int g = 0; g < 2; ++g) {
        gp.codes[g] = codes[g];
        gp.qjl[g] = qjl[g];
        gp.norms[g] = norms[g];
        gp.rnorms[g] = rnorms[g];
        gp.code_bytes[g] = st[g]->code_bytes;
        gp.qjl_bytes[g] = st[g]->qjl_bytes;
        duo_levels(*st[g], gp, g);
    }
    const bool prod = so.mode == TQ_PROD;
    if (so.b_mse == 1)
        return prod ? launch_split_b1<1, true>(si.b_mse, tmap, p, gp, s) : launch_split_b1<1, false>(si.b_mse, tmap, p, gp, s);
    return prod ? launch_split_b1<2, true>(si.b_mse, tmap, p, gp, s) : launch_split_b1<2, false>(si.b_mse, tmap, p, gp, s);
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
