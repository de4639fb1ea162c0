// Inner-product estimates straight from packed codes through per-query lookup tables.
//
// TurboQuant review (Jump2Paper): the estimate of <q, x> is <q, x~> (unbiased for prod,
// Theorem 2); with q' = Pi q and u = S q' it reads
//     <q, x~> = ||x|| ( sum_j q'_j c[idx_j] + ||r|| sqrt(pi/2)/d sum_j u_j (2 z_j - 1) ),
// i.e. the keys are never un-rotated: the query is rotated once (the rotated-query reading
// of the Hacker News digest's "un-rotation for future queries").
//
// For each query of the block the sums are tabulated over small groups of packed bits:
//   MSE part: a group of G bits (G = 4, or 6 for 3-bit codes) holds G/b codes; table
//             T_k[e] = sum over the codes i of group k of q'_{k*G/b + i} c[code_i(e)];
//   QJL part: a nibble holds 4 signs; U_k[e] = sum_i u_{4k+i} (2 bit_i(e) - 1).
// A key then costs one table read per group: with 16-entry tables every lane of a warp
// reading the same table hits a distinct bank or shares a word (no bank conflicts).
// One thread scores one key against up to QT queries; the query preparation
// (q' = Pi q, u = S q', the tables) is done by each block in shared memory.
#include "common.cuh"
#include "prep.cuh"

namespace tq {

namespace {

constexpr int kThreads = 256;

template <int B>
struct Groups {
    static constexpr int G = (B == 3) ? 6 : 4;          // bits per table index
    static constexpr int CPG = G / B;                    // codes per group
    static constexpr int E = 1 << G;                     // entries per table
};

template <int D, int B, bool PROD>
struct LutShape {
    using Gr = Groups<B>;
    static constexpr int NG = D * B / Gr::G;        // MSE tables per query
    static constexpr int NQ = D / 4;                // QJL tables per query
    static constexpr int MSE = NG * Gr::E;          // floats
    static constexpr int QJL = PROD ? NQ * 16 : 0;  // floats
    static constexpr int SIZE = MSE + QJL;          // floats per query (a multiple of 4)
};

// One block per query: q' = Pi q, u = S q', then the tables, written to `luts`.
template <int D, int B, bool PROD>
__global__ void __launch_bounds__(kThreads)
score_prep_kernel(const DevState st, const void* __restrict__ q, int qdtype, float* __restrict__ luts) {
    using Gr = Groups<B>;
    using LS = LutShape<D, B, PROD>;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float* ctab = reinterpret_cast<float*>(smem_raw);
    float* qs = ctab + kMaxLevels;
    float* qp = qs + D;
    float* u = qp + D;
    unsigned char* stage = reinterpret_cast<unsigned char*>(u + D);
    const int64_t qi = blockIdx.x;   // flat query index (group-major)
    for (int i = threadIdx.x; i < st.L; i += blockDim.x) ctab[i] = st.c[i];
    const size_t qelem = (qdtype == TQ_F32) ? 4 : 2;
    prep_queries_dev(st, reinterpret_cast<const unsigned char*>(q) + (size_t)qi * D * qelem, qdtype, 1, qs, qp, u,
                     stage);
    float* out = luts + qi * LS::SIZE;
    for (int i = threadIdx.x; i < LS::MSE; i += blockDim.x) {
        const int k = i / Gr::E, e = i % Gr::E;
        float a = 0.f;
#pragma unroll
        for (int c = 0; c < Gr::CPG; ++c)
            a = fmaf(qp[k * Gr::CPG + c], ctab[(e >> (B * c)) & ((1 << B) - 1)], a);
        out[i] = a;
    }
    if constexpr (PROD) {
        for (int i = threadIdx.x; i < LS::QJL; i += blockDim.x) {
            const int k = i / 16, e = i % 16;
            float a = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float v = u[4 * k + c];
                a += ((e >> c) & 1) ? v : -v;
            }
            out[LS::MSE + i] = a;
        }
    }
}

// d = 128: the same preparation split over several blocks per query, the RHT butterfly done
// by one warp with shuffles and the matrix-vector products split over all 256 threads.
constexpr int kD128 = 128;

// out[j] = sum_k MT[k][j] in[k] (MT row-major 128 x 128, shared or global); threads (j, half) each sum
// 64 rows, `part` holds the halves.
__device__ __forceinline__ void matvec128(const unsigned char* MT, int dtype, const float* in, float* part,
                                          float* out) {
    const int j = threadIdx.x & (kD128 - 1), h = threadIdx.x >> 7;
    float a0 = 0.f, a1 = 0.f;
    if (dtype == TQ_F32) {
        const float* m = reinterpret_cast<const float*>(MT) + h * 64 * kD128 + j;
#pragma unroll 16
        for (int k = 0; k < 64; k += 2) {
            a0 = fmaf(m[k * kD128], in[h * 64 + k], a0);
            a1 = fmaf(m[(k + 1) * kD128], in[h * 64 + k + 1], a1);
        }
    } else {
        const uint16_t* m = reinterpret_cast<const uint16_t*>(MT) + h * 64 * kD128 + j;
#pragma unroll 16
        for (int k = 0; k < 64; k += 2) {
            a0 = fmaf(bf16_bits_to_float(m[k * kD128]), in[h * 64 + k], a0);
            a1 = fmaf(bf16_bits_to_float(m[(k + 1) * kD128]), in[h * 64 + k + 1], a1);
        }
    }
    part[h * kD128 + j] = a0 + a1;
    __syncthreads();
    if (threadIdx.x < kD128) out[threadIdx.x] = part[threadIdx.x] + part[kD128 + threadIdx.x];
    __syncthreads();
}

// Sylvester Walsh-Hadamard transform of the 128 values in src (signs eps applied first), times
// 1/sqrt(d), into dst: one warp, lane l holding elements 4l .. 4l+3; stages h = 1, 2 in
// registers, h >= 4 across lanes.
__device__ __forceinline__ void warp_rht128(const DevState& st, const float* src, float* dst) {
    const int l = threadIdx.x & 31;
    float v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = rht_neg(st, 4 * l + i) ? -src[4 * l + i] : src[4 * l + i];
#pragma unroll
    for (int h = 1; h < 4; h <<= 1) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if ((i & h) == 0) {
                const float a = v[i], b = v[i + h];
                v[i] = a + b;
                v[i + h] = a - b;
            }
        }
    }
#pragma unroll
    for (int hl = 1; hl < 32; hl <<= 1) {
        const bool upper = (l & hl) != 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float o = __shfl_xor_sync(0xffffffffu, v[i], hl);
            v[i] = upper ? o - v[i] : v[i] + o;
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[4 * l + i] = v[i] * st.rsqrt_d;
}

// One vector x of d = 128 encoded by the whole block (TurboQuant review, Theorem 1 and
// Definition 1 / Theorem 2): ||x||; y = Pi x / ||x||; code_j = #{k : t_k <= y_j}; prod: the
// residual r = y - c[code], ||r|| and the signs [(S r)_j >= 0]; codes packed LSB-first.
// piT / sT are the state's transposed matrices (row-major 128 x 128, in shared or global
// memory). The state has at most 16 levels. buf: 5 x 128 + 8 floats, cb: 128 bytes, both in
// shared memory. Every thread of the block calls this.
__device__ void block_encode128(const DevState& st, const void* x, int dtype, const unsigned char* piT,
                                const unsigned char* sT, uint8_t* codes, uint8_t* qjl, float* norm, float* rnorm,
                                float* buf, uint8_t* cb) {
    float* xs = buf;
    float* ys = xs + kD128;
    float* part = ys + kD128;   // 2 x 128
    float* red = part + 2 * kD128;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float xv = 0.f;
    if (tid < kD128) {
        xv = (dtype == TQ_F32) ? __ldg(reinterpret_cast<const float*>(x) + tid)
                               : bf16_bits_to_float(__ldg(reinterpret_cast<const uint16_t*>(x) + tid));
        xs[tid] = xv;
    }
    const float ss = warp_sum(xv * xv);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    const float nu = sqrtf((red[0] + red[1]) + (red[2] + red[3]));
    if (st.rot == TQ_ROT_RHT) {
        if (warp == 0) warp_rht128(st, xs, ys);
        __syncthreads();
    } else {
        matvec128(piT, st.mat_dtype, xs, part, ys);
    }
    const float sc = (nu > 0.f) ? 1.f / nu : 0.f;
    float r = 0.f;
    if (tid < kD128) {
        const float y = ys[tid] * sc;
        const int c = (st.b_mse > 0) ? quantize_coord(st, nullptr, y) : 0;
        cb[tid] = (uint8_t)c;
        r = (nu > 0.f) ? (y - (st.b_mse > 0 ? st.c[c] : 0.f)) : 0.f;
        xs[tid] = r;
    }
    const float rr = warp_sum(r * r);
    if (lane == 0) red[4 + warp] = rr;   // the norm was read before the rotation's barriers
    __syncthreads();
    if (tid == 0) {
        *norm = nu;
        if (st.mode == TQ_PROD) *rnorm = sqrtf((red[4] + red[5]) + (red[6] + red[7]));
    }
    if (st.mode == TQ_PROD) {
        matvec128(sT, st.mat_dtype, xs, part, ys);   // ys = S r
        if (tid < kD128) {
            const uint32_t z = __ballot_sync(0xffffffffu, ys[tid] >= 0.f);
            if (lane == 0) reinterpret_cast<uint32_t*>(qjl)[warp] = z;
        }
    }
    // stream bit p = 32 w + lane holds bit p % b of code p / b
    const int b = st.b_mse;
    for (int w = warp; w < b * kD128 / 32; w += kThreads / 32) {
        const int p = 32 * w + lane;
        const int j = p / b;
        const uint32_t word = __ballot_sync(0xffffffffu, (cb[j] >> (p - j * b)) & 1u);
        if (lane == 0) reinterpret_cast<uint32_t*>(codes)[w] = word;
    }
    __syncthreads();
}

// Per query the lookup tables of q' = Pi q against the code groups and of u = S q' against the
// QJL nibbles, split over kParts blocks (grid count x kParts): block p writes the quarter p of
// the code-group tables and the QJL tables of nibbles 8p .. 8p + 7, so it needs all of q' but
// only u_j for j in [32p, 32p + 32). The matrices are read from L2 (no staging): q' = Pi q by
// the whole block (or the Hadamard transform by one warp), u_j = sum_k S^T[k][j] q'_k by 8
// threads per output. APPEND (a decode step that appends one token): one more block per query
// (blockIdx.y == kParts) in which the first query head of each group of G encodes the new K and
// V vectors of its KV head into row T of that head's planes, before the attention launch that
// reads them.
constexpr int kParts = 4;

template <int B, bool PROD, bool APPEND>
__global__ void __launch_bounds__(kThreads)
tables128_part_kernel(const DevState st, const void* __restrict__ q, int qdtype, float* __restrict__ luts,
                      const DevState vs, const AppendRow app) {
    using Gr = Groups<B>;
    using LS = LutShape<kD128, B, PROD>;
    static_assert(LS::NG % kParts == 0 && LS::NQ % kParts == 0, "whole tables per part");
    __shared__ float ctab[16];
    __shared__ float qs[kD128], qp[kD128], part[2 * kD128], uq[kD128 / kParts];
    __shared__ float upart[8][kD128 / kParts];
    const int64_t qi = blockIdx.x;
    const int pt = blockIdx.y;
    if constexpr (APPEND) {
        if (pt == kParts) {
            if (qi % app.G == 0) {
                __shared__ __align__(16) float ebuf[5 * kD128 + 8];
                __shared__ uint8_t ecb[kD128];
                const int64_t g = qi / app.G;   // KV head
                const size_t es = (app.dtype == TQ_F32) ? 4 : 2;
                const int64_t row = g * app.Tcap;
                block_encode128(st, reinterpret_cast<const unsigned char*>(app.k_new) + g * kD128 * es, app.dtype,
                                reinterpret_cast<const unsigned char*>(st.piT),
                                reinterpret_cast<const unsigned char*>(st.sT), app.kcodes + row * st.code_bytes,
                                PROD ? app.kqjl + row * st.qjl_bytes : nullptr, app.knorms + row,
                                PROD ? app.krnorms + row : nullptr, ebuf, ecb);
                block_encode128(vs, reinterpret_cast<const unsigned char*>(app.v_new) + g * kD128 * es, app.dtype,
                                reinterpret_cast<const unsigned char*>(vs.piT),
                                reinterpret_cast<const unsigned char*>(vs.sT), app.vcodes + row * vs.code_bytes,
                                vs.mode == TQ_PROD ? app.vqjl + row * vs.qjl_bytes : nullptr, app.vnorms + row,
                                vs.mode == TQ_PROD ? app.vrnorms + row : nullptr, ebuf, ecb);
            }
            return;
        }
    }
    if (threadIdx.x < 16) ctab[threadIdx.x] = (threadIdx.x < st.L) ? st.c[threadIdx.x] : 0.f;
    if (threadIdx.x < kD128) {
        const int i = threadIdx.x;
        qs[i] = (qdtype == TQ_F32) ? __ldg(reinterpret_cast<const float*>(q) + qi * kD128 + i)
                                   : bf16_bits_to_float(__ldg(reinterpret_cast<const uint16_t*>(q) + qi * kD128 + i));
    }
    __syncthreads();
    if (st.rot != TQ_ROT_RHT) {
        matvec128(reinterpret_cast<const unsigned char*>(st.piT), st.mat_dtype, qs, part, qp);
    } else {
        if (threadIdx.x < 32) warp_rht128(st, qs, qp);
        __syncthreads();
    }
    if constexpr (PROD) {
        // u_j, j = 32 pt + jl: thread (jl, h) sums k in [16 h, 16 h + 16)
        constexpr int kJ = kD128 / kParts;
        const int jl = threadIdx.x % kJ, h = threadIdx.x / kJ;
        const int j = pt * kJ + jl;
        float a = 0.f;
        if (st.mat_dtype == TQ_F32) {
            const float* m = reinterpret_cast<const float*>(st.sT) + (size_t)(16 * h) * kD128 + j;
#pragma unroll
            for (int k = 0; k < 16; ++k) a = fmaf(__ldg(m + k * kD128), qp[16 * h + k], a);
        } else {
            const uint16_t* m = reinterpret_cast<const uint16_t*>(st.sT) + (size_t)(16 * h) * kD128 + j;
#pragma unroll
            for (int k = 0; k < 16; ++k) a = fmaf(bf16_bits_to_float(__ldg(m + k * kD128)), qp[16 * h + k], a);
        }
        upart[h][jl] = a;
        __syncthreads();
        if (threadIdx.x < kJ) {
            float sum = 0.f;
#pragma unroll
            for (int hh = 0; hh < 8; ++hh) sum += upart[hh][threadIdx.x];
            uq[threadIdx.x] = sum;
        }
        __syncthreads();
    }
    float* out = luts + qi * LS::SIZE;
    constexpr int kMsePart = LS::MSE / kParts;
    for (int i = pt * kMsePart + threadIdx.x; i < (pt + 1) * kMsePart; i += kThreads) {
        const int k = i / Gr::E, e = i % Gr::E;
        float a = 0.f;
#pragma unroll
        for (int c = 0; c < Gr::CPG; ++c)
            a = fmaf(qp[k * Gr::CPG + c], ctab[(e >> (B * c)) & ((1 << B) - 1)], a);
        out[i] = a;
    }
    if constexpr (PROD) {
        constexpr int kQjlPart = LS::QJL / kParts;   // 8 nibble tables of 16
        for (int i = threadIdx.x; i < kQjlPart; i += kThreads) {
            const int kl = i / 16, e = i % 16;   // nibble 8 pt + kl: u_j for j = 4 (8 pt + kl) + c
            float a = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float v = uq[4 * kl + c];
                a += ((e >> c) & 1) ? v : -v;
            }
            out[LS::MSE + pt * kQjlPart + i] = a;
        }
    }
}

// Tables of `count` queries (rows of q) into luts[count][SIZE].
template <int D, int B, bool PROD>
int launch_tables(const DevState& st, const void* q, int qdtype, int64_t count, float* luts, cudaStream_t s) {
    if (count <= 0) return 0;
    if (count > (1ll << 31) - 1) return (int)cudaErrorInvalidConfiguration;
    if constexpr (D == kD128) {
        tables128_part_kernel<B, PROD, false><<<dim3((unsigned)count, kParts), kThreads, 0, s>>>(st, q, qdtype, luts,
                                                                                               st, AppendRow{});
    } else {
        auto k = score_prep_kernel<D, B, PROD>;
        const size_t smem = (size_t)(kMaxLevels + 3 * D) * sizeof(float) + kPrepStageBytes;
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return (int)e;
        }
        k<<<(unsigned)count, kThreads, smem, s>>>(st, q, qdtype, luts);
    }
    return (int)cudaGetLastError();
}

// N consecutive 32-bit words from a row whose stride is 4 N bytes (16-, 8- or 4-byte loads).
template <int N>
__device__ __forceinline__ void load_words(const uint32_t* __restrict__ src, uint32_t (&w)[N]) {
    if constexpr (N % 4 == 0) {
#pragma unroll
        for (int i = 0; i < N / 4; ++i) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    } else if constexpr (N % 2 == 0) {
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(src) + i);
            w[2 * i] = v.x; w[2 * i + 1] = v.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) w[i] = __ldg(src + i);
    }
}

template <int D, int B, bool PROD, int QT>
__global__ void __launch_bounds__(kThreads)
score_lut_kernel(const DevState st, const float* __restrict__ luts, int64_t nq,
                 const uint8_t* __restrict__ codes, const uint8_t* __restrict__ qjl,
                 const float* __restrict__ norms, const float* __restrict__ rnorms, int64_t n,
                 int keys_per_block, int accumulate, float* __restrict__ scores) {
    using Gr = Groups<B>;
    using LS = LutShape<D, B, PROD>;
    constexpr int NG = LS::NG;
    constexpr int NQ = LS::NQ;
    constexpr int CW = D * B / 32;         // code words per key
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float* tab = reinterpret_cast<float*>(smem_raw);   // QT x SIZE

    const int64_t grp = blockIdx.z;
    const int64_t q0 = (int64_t)blockIdx.y * QT;
    const int nqt = (int)((nq - q0) < QT ? (nq - q0) : QT);
    {
        const float4* src = reinterpret_cast<const float4*>(luts + (grp * nq + q0) * LS::SIZE);
        float4* dst = reinterpret_cast<float4*>(tab);
        for (int i = threadIdx.x; i < nqt * LS::SIZE / 4; i += kThreads) dst[i] = __ldg(src + i);
        for (int i = nqt * LS::SIZE / 4 + threadIdx.x; i < QT * LS::SIZE / 4; i += kThreads)
            dst[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();

    const int64_t k_begin = (int64_t)blockIdx.x * keys_per_block;
    const int64_t k_end = (n < k_begin + keys_per_block) ? n : k_begin + keys_per_block;
    // The next key's bytes are loaded before the current key's lookups (one key in flight
    // per thread while the tables are read).
    constexpr int ZW = PROD ? D / 32 : 1;
    auto load_key = [&](int64_t key, uint32_t (&w)[CW], uint32_t (&z)[ZW], float& rn, float& nu) {
        const int64_t gk = grp * n + key;
        load_words<CW>(reinterpret_cast<const uint32_t*>(codes + gk * (D * B / 8)), w);
        rn = 0.f;
        if constexpr (PROD) {
            load_words<ZW>(reinterpret_cast<const uint32_t*>(qjl + gk * (D / 8)), z);
            rn = __ldg(rnorms + gk);
        }
        nu = __ldg(norms + gk);
    };
    uint32_t wn[CW] = {}, zn[ZW] = {};
    float rnn = 0.f, nun = 0.f;
    if (k_begin + threadIdx.x < k_end) load_key(k_begin + threadIdx.x, wn, zn, rnn, nun);
    for (int64_t key = k_begin + threadIdx.x; key < k_end; key += kThreads) {
        uint32_t w[CW], z[ZW];
#pragma unroll
        for (int i = 0; i < CW; ++i) w[i] = wn[i];
#pragma unroll
        for (int i = 0; i < ZW; ++i) z[i] = zn[i];
        const float g2 = rnn * st.qjl_scale;
        const float nu = nun;
        if (key + kThreads < k_end) load_key(key + kThreads, wn, zn, rnn, nun);
        float a1[QT], a2[QT];
        float2 p1[QT], p2[QT];   // paired accumulators of the nibble lookups
#pragma unroll
        for (int qi = 0; qi < QT; ++qi) {
            a1[qi] = a2[qi] = 0.f;
            p1[qi] = p2[qi] = make_float2(0.f, 0.f);
        }
        if constexpr (Gr::G == 4) {
            // 16-entry tables: the 8 nibbles of a word, pre-scaled to byte offsets 4 e
#pragma unroll
            for (int wi = 0; wi < CW; ++wi) add_nibbles<QT, LS::SIZE>(w[wi], tab + 8 * wi * 16, p1);
        } else {
#pragma unroll
            for (int k = 0; k < NG; ++k) {
                const int bit = k * Gr::G;
                const int wi = bit >> 5, sh = bit & 31;
                uint32_t e;
                if (sh + Gr::G <= 32) {
                    e = (w[wi] >> sh) & (Gr::E - 1);
                } else {
                    e = ((w[wi] >> sh) | (w[wi + 1] << (32 - sh))) & (Gr::E - 1);
                }
#pragma unroll
                for (int qi = 0; qi < QT; ++qi) a1[qi] += tab[qi * LS::SIZE + k * Gr::E + e];
            }
        }
        if constexpr (PROD) {
#pragma unroll
            for (int wi = 0; wi < NQ / 8; ++wi) add_nibbles<QT, LS::SIZE>(z[wi], tab + LS::MSE + 8 * wi * 16, p2);
        }
#pragma unroll
        for (int qi = 0; qi < QT; ++qi) {
            a1[qi] += p1[qi].x + p1[qi].y;
            a2[qi] += p2[qi].x + p2[qi].y;
            if (qi < nqt) {
                float* dst = scores + (grp * nq + q0 + qi) * n + key;   // key of this group
                const float v = nu * fmaf(g2, a2[qi], a1[qi]);
                *dst = accumulate ? *dst + v : v;
            }
        }
    }
}


int sm_count_lut() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

template <int D, int B, bool PROD, int QT>
int launch_lut(const DevState& st, const void* q, int qdtype, int64_t groups, int64_t nq, const uint8_t* codes,
               const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, int accumulate,
               float* scores, float* luts, cudaStream_t s) {
    using LS = LutShape<D, B, PROD>;
    const int64_t qtiles = (nq + QT - 1) / QT;
    if (qtiles > 65535 || groups > 65535 || groups * nq > (1ll << 31) - 1) return (int)cudaErrorInvalidConfiguration;
    // Per-query tables in the caller's workspace, built once per query.
    cudaError_t ce = (cudaError_t)launch_tables<D, B, PROD>(st, q, qdtype, groups * nq, luts, s);
    if (ce == cudaSuccess) {
        auto kern = score_lut_kernel<D, B, PROD, QT>;
        const size_t smem = (size_t)QT * LS::SIZE * sizeof(float);
        if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        // A few waves of blocks; at least 1024 keys per block.
        const int64_t want_blocks = (int64_t)sm_count_lut() * 8;
        int64_t per = (n * qtiles * groups + want_blocks - 1) / want_blocks;
        per = std::max<int64_t>(per, 1024);
        per = (per + kThreads - 1) / kThreads * kThreads;
        const int64_t kb = (n + per - 1) / per;
        if (kb > (1ll << 31) - 1) {
            ce = cudaErrorInvalidConfiguration;
        } else {
            dim3 grid((unsigned)kb, (unsigned)qtiles, (unsigned)groups);
            kern<<<grid, kThreads, smem, s>>>(st, luts, nq, codes, qjl, norms, rnorms, n, (int)per, accumulate, scores);
            ce = cudaGetLastError();
        }
    }
    return (int)ce;
}

template <int D, int B, bool PROD>
int launch_lut_q(const DevState& st, const void* q, int qdtype, int64_t groups, int64_t nq, const uint8_t* codes,
                 const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, int accumulate, float* scores,
                 float* luts, cudaStream_t s) {
    if (nq == 1) return launch_lut<D, B, PROD, 1>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
    return launch_lut<D, B, PROD, 4>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
}

template <int D, int B>
int launch_lut_m(const DevState& st, const void* q, int qdtype, int64_t groups, int64_t nq, const uint8_t* codes,
                 const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, int accumulate, float* scores,
                 float* luts, cudaStream_t s) {
    if (qjl) return launch_lut_q<D, B, true>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
    return launch_lut_q<D, B, false>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
}

template <int D>
int launch_lut_b(const DevState& st, const void* q, int qdtype, int64_t groups, int64_t nq, const uint8_t* codes,
                 const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, int accumulate, float* scores,
                 float* luts, cudaStream_t s) {
    switch (st.b_mse) {
        case 1: return launch_lut_m<D, 1>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
        case 2: return launch_lut_m<D, 2>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
        case 3: return launch_lut_m<D, 3>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
        case 4: return launch_lut_m<D, 4>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
        default: return (int)cudaErrorInvalidValue;
    }
}

template <bool PROD>
int launch_tables128_b(const DevState& st, const void* q, int qdtype, int64_t count, float* luts, cudaStream_t s) {
    switch (st.b_mse) {
        case 1: return launch_tables<128, 1, PROD>(st, q, qdtype, count, luts, s);
        case 2: return launch_tables<128, 2, PROD>(st, q, qdtype, count, luts, s);
        case 3: return launch_tables<128, 3, PROD>(st, q, qdtype, count, luts, s);
        case 4: return launch_tables<128, 4, PROD>(st, q, qdtype, count, luts, s);
        default: return (int)cudaErrorInvalidValue;
    }
}

}  // namespace

size_t query_table_floats(const DevState& st) {
    const bool prod = st.mode == TQ_PROD;
    switch (st.b_mse) {
        case 1: return prod ? LutShape<128, 1, true>::SIZE : LutShape<128, 1, false>::SIZE;
        case 2: return prod ? LutShape<128, 2, true>::SIZE : LutShape<128, 2, false>::SIZE;
        case 3: return prod ? LutShape<128, 3, true>::SIZE : LutShape<128, 3, false>::SIZE;
        case 4: return prod ? LutShape<128, 4, true>::SIZE : LutShape<128, 4, false>::SIZE;
        default: return 0;
    }
}

int launch_query_tables128(const DevState& st, const void* q, int qdtype, int64_t count, float* luts, void* stream) {
    if (st.d != 128) return (int)cudaErrorInvalidValue;
    cudaStream_t s = (cudaStream_t)stream;
    if (st.mode == TQ_PROD) return launch_tables128_b<true>(st, q, qdtype, count, luts, s);
    return launch_tables128_b<false>(st, q, qdtype, count, luts, s);
}

namespace {
template <int B, bool PROD>
int launch_append_tables(const DevState& ks, const DevState& vs, const void* q, int qdtype, int64_t count,
                         float* luts, const AppendRow& app, cudaStream_t s) {
    tables128_part_kernel<B, PROD, true><<<dim3((unsigned)count, kParts + 1), kThreads, 0, s>>>(ks, q, qdtype, luts,
                                                                                              vs, app);
    return (int)cudaGetLastError();
}

template <bool PROD>
int launch_append_tables_b(const DevState& ks, const DevState& vs, const void* q, int qdtype, int64_t count,
                           float* luts, const AppendRow& app, cudaStream_t s) {
    switch (ks.b_mse) {
        case 2: return launch_append_tables<2, PROD>(ks, vs, q, qdtype, count, luts, app, s);
        case 3: return launch_append_tables<3, PROD>(ks, vs, q, qdtype, count, luts, app, s);
        case 4: return launch_append_tables<4, PROD>(ks, vs, q, qdtype, count, luts, app, s);
        default: return (int)cudaErrorInvalidValue;
    }
}
}  // namespace

// The query tables of `count` heads, the first head of each group of app.G also appending the
// new K and V token of its KV head (d = 128, key and value codes of 2 to 4 bits).
int launch_append_tables128(const DevState& ks, const DevState& vs, const void* q, int qdtype, int64_t count,
                            float* luts, const AppendRow& app, void* stream) {
    if (ks.d != 128 || vs.d != 128 || ks.L > 16 || vs.L > 16 || app.G <= 0) return (int)cudaErrorInvalidValue;
    cudaStream_t s = (cudaStream_t)stream;
    if (ks.mode == TQ_PROD) return launch_append_tables_b<true>(ks, vs, q, qdtype, count, luts, app, s);
    return launch_append_tables_b<false>(ks, vs, q, qdtype, count, luts, app, s);
}

namespace {
template <int D>
size_t lut_floats_d(int b, bool prod) {
    switch (b) {
        case 1: return prod ? LutShape<D, 1, true>::SIZE : LutShape<D, 1, false>::SIZE;
        case 2: return prod ? LutShape<D, 2, true>::SIZE : LutShape<D, 2, false>::SIZE;
        case 3: return prod ? LutShape<D, 3, true>::SIZE : LutShape<D, 3, false>::SIZE;
        case 4: return prod ? LutShape<D, 4, true>::SIZE : LutShape<D, 4, false>::SIZE;
        default: return 0;
    }
}
}  // namespace

// Floats of the lookup tables of one query of the table scorer.
size_t score_lut_floats(const DevState& st) {
    const bool prod = st.mode == TQ_PROD;
    switch (st.d) {
        case 32: return lut_floats_d<32>(st.b_mse, prod);
        case 64: return lut_floats_d<64>(st.b_mse, prod);
        case 96: return lut_floats_d<96>(st.b_mse, prod);
        case 128: return lut_floats_d<128>(st.b_mse, prod);
        case 256: return lut_floats_d<256>(st.b_mse, prod);
        default: return 0;
    }
}

bool score_lut_supported(const DevState& st) {
    const bool dim = st.d == 32 || st.d == 64 || st.d == 96 || st.d == 128 || st.d == 256;
    return dim && st.b_mse >= 1 && st.b_mse <= 4;
}

int launch_score_lut(const DevState& st, const void* q, int qdtype, int64_t groups, int64_t nq, const uint8_t* codes,
                     const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, int accumulate, float* scores,
                     void* ws, void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    float* luts = reinterpret_cast<float*>(ws);
    switch (st.d) {
        case 32: return launch_lut_b<32>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
        case 64: return launch_lut_b<64>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
        case 96: return launch_lut_b<96>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
        case 128: return launch_lut_b<128>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
        default: return launch_lut_b<256>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, luts, s);
    }
}

}  // namespace tq
