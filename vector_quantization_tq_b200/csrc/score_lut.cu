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

template <int D, int B, bool PROD, int QT>
__global__ void __launch_bounds__(kThreads)
score_lut_kernel(const DevState st, const void* __restrict__ q, int qdtype, int64_t nq,
                 const uint8_t* __restrict__ codes, const uint8_t* __restrict__ qjl,
                 const float* __restrict__ norms, const float* __restrict__ rnorms, int64_t n,
                 int keys_per_block, float* __restrict__ scores) {
    using Gr = Groups<B>;
    constexpr int NG = D * B / Gr::G;      // MSE tables per query
    constexpr int NQ = D / 4;              // QJL tables per query
    constexpr int CW = D * B / 32;         // code words per key
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float* ctab = reinterpret_cast<float*>(smem_raw);          // kMaxLevels
    float* qs = ctab + kMaxLevels;                              // QT*D
    float* qp = qs + QT * D;                                    // QT*D
    float* u = qp + QT * D;                                     // QT*D
    float* tm = u + QT * D;                                     // QT*NG*E
    float* tz = tm + QT * NG * Gr::E;                           // QT*NQ*16 (prod)
    unsigned char* stage = reinterpret_cast<unsigned char*>(tz + (PROD ? QT * NQ * 16 : 0));

    const int64_t grp = blockIdx.z;
    const int64_t q0 = (int64_t)blockIdx.y * QT;
    const int nqt = (int)((nq - q0) < QT ? (nq - q0) : QT);
    for (int i = threadIdx.x; i < st.L; i += blockDim.x) ctab[i] = st.c[i];
    const size_t qelem = (qdtype == TQ_F32) ? 4 : 2;
    prep_queries_dev(st, reinterpret_cast<const unsigned char*>(q) + (size_t)((grp * nq + q0) * D) * qelem, qdtype,
                     nqt, qs, qp, u, stage);
    // tables (queries beyond nqt get zero tables; their scores are not stored)
    for (int i = threadIdx.x; i < QT * NG * Gr::E; i += blockDim.x) {
        const int qi = i / (NG * Gr::E);
        const int k = (i / Gr::E) % NG;
        const int e = i % Gr::E;
        float a = 0.f;
        if (qi < nqt) {
#pragma unroll
            for (int c = 0; c < Gr::CPG; ++c) {
                const int j = k * Gr::CPG + c;
                a = fmaf(qp[qi * D + j], ctab[(e >> (B * c)) & ((1 << B) - 1)], a);
            }
        }
        tm[i] = a;
    }
    if constexpr (PROD) {
        for (int i = threadIdx.x; i < QT * NQ * 16; i += blockDim.x) {
            const int qi = i / (NQ * 16);
            const int k = (i / 16) % NQ;
            const int e = i % 16;
            float a = 0.f;
            if (qi < nqt) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float v = u[qi * D + 4 * k + c];
                    a += ((e >> c) & 1) ? v : -v;
                }
            }
            tz[i] = a;
        }
    }
    __syncthreads();

    const int64_t k_begin = (int64_t)blockIdx.x * keys_per_block;
    const int64_t k_end = (n < k_begin + keys_per_block) ? n : k_begin + keys_per_block;
    for (int64_t key = k_begin + threadIdx.x; key < k_end; key += kThreads) {
        const int64_t gk = grp * n + key;
        uint32_t w[CW];
        {
            const uint4* src = reinterpret_cast<const uint4*>(codes + gk * (D * B / 8));
#pragma unroll
            for (int i = 0; i < CW / 4; ++i) {
                const uint4 v = __ldg(src + i);
                w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
            }
        }
        float a1[QT];
#pragma unroll
        for (int qi = 0; qi < QT; ++qi) a1[qi] = 0.f;
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
            for (int qi = 0; qi < QT; ++qi) a1[qi] += tm[(qi * NG + k) * Gr::E + e];
        }
        float a2[QT];
#pragma unroll
        for (int qi = 0; qi < QT; ++qi) a2[qi] = 0.f;
        float g2 = 0.f;
        if constexpr (PROD) {
            uint32_t z[D / 32];
            const uint4* zs = reinterpret_cast<const uint4*>(qjl + gk * (D / 8));
#pragma unroll
            for (int i = 0; i < D / 128; ++i) {
                const uint4 v = __ldg(zs + i);
                z[4 * i] = v.x; z[4 * i + 1] = v.y; z[4 * i + 2] = v.z; z[4 * i + 3] = v.w;
            }
#pragma unroll
            for (int k = 0; k < NQ; ++k) {
                const uint32_t e = (z[k >> 3] >> ((k & 7) * 4)) & 15u;
#pragma unroll
                for (int qi = 0; qi < QT; ++qi) a2[qi] += tz[(qi * NQ + k) * 16 + e];
            }
            g2 = __ldg(rnorms + gk) * st.qjl_scale;
        }
        const float nu = __ldg(norms + gk);
#pragma unroll
        for (int qi = 0; qi < QT; ++qi)
            if (qi < nqt) scores[(grp * nq + q0 + qi) * n + key] = nu * fmaf(g2, a2[qi], a1[qi]);
    }
}

template <int D, int B, bool PROD, int QT>
size_t lut_smem() {
    using Gr = Groups<B>;
    return (size_t)(kMaxLevels + 3 * QT * D + QT * (D * B / Gr::G) * Gr::E + (PROD ? QT * (D / 4) * 16 : 0)) *
               sizeof(float) + kPrepStageBytes;
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
               const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, float* scores,
               cudaStream_t s) {
    auto kern = score_lut_kernel<D, B, PROD, QT>;
    const size_t smem = lut_smem<D, B, PROD, QT>();
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return (int)e;
    }
    const int64_t qtiles = (nq + QT - 1) / QT;
    if (qtiles > 65535 || groups > 65535) return (int)cudaErrorInvalidConfiguration;
    // Enough blocks for a few waves, at least 1024 keys per block so the table set-up
    // stays small next to the scoring.
    const int64_t want_blocks = (int64_t)sm_count_lut() * 8;
    int64_t per = (n * qtiles * groups + want_blocks - 1) / want_blocks;
    per = std::max<int64_t>(per, 1024);
    per = (per + kThreads - 1) / kThreads * kThreads;
    const int64_t kb = (n + per - 1) / per;
    if (kb > (1ll << 31) - 1) return (int)cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)kb, (unsigned)qtiles, (unsigned)groups);
    kern<<<grid, kThreads, smem, s>>>(st, q, qdtype, nq, codes, qjl, norms, rnorms, n, (int)per, scores);
    return (int)cudaGetLastError();
}

template <int D, int B, bool PROD>
int launch_lut_q(const DevState& st, const void* q, int qdtype, int64_t groups, int64_t nq, const uint8_t* codes,
                 const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, float* scores,
                 cudaStream_t s) {
    if (nq == 1) return launch_lut<D, B, PROD, 1>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, scores, s);
    return launch_lut<D, B, PROD, 4>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, scores, s);
}

template <int D, int B>
int launch_lut_m(const DevState& st, const void* q, int qdtype, int64_t groups, int64_t nq, const uint8_t* codes,
                 const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, float* scores,
                 cudaStream_t s) {
    if (qjl) return launch_lut_q<D, B, true>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, scores, s);
    return launch_lut_q<D, B, false>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, scores, s);
}

template <int D>
int launch_lut_b(const DevState& st, const void* q, int qdtype, int64_t groups, int64_t nq, const uint8_t* codes,
                 const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, float* scores,
                 cudaStream_t s) {
    switch (st.b_mse) {
        case 1: return launch_lut_m<D, 1>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, scores, s);
        case 2: return launch_lut_m<D, 2>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, scores, s);
        case 3: return launch_lut_m<D, 3>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, scores, s);
        case 4: return launch_lut_m<D, 4>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, scores, s);
        default: return (int)cudaErrorInvalidValue;
    }
}

}  // namespace

bool score_lut_supported(const DevState& st) {
    return (st.d == 128 || st.d == 256) && st.b_mse >= 1 && st.b_mse <= 4;
}

int launch_score_lut(const DevState& st, const void* q, int qdtype, int64_t groups, int64_t nq, const uint8_t* codes,
                     const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, float* scores,
                     void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    if (st.d == 128) return launch_lut_b<128>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, scores, s);
    return launch_lut_b<256>(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, scores, s);
}

}  // namespace tq
