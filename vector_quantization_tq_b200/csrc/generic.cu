// General-purpose libtq kernels: encode (TurboQuant_mse / _prod), dequant, score,
// decode attention and top-k search, for every supported d, fp32 or bf16 state.
//
// Thread layout: a group of NT threads owns one vector at a time, each thread E
// consecutive coordinates (j = tid*E + e, d = NT*E). For d <= 256 a group is one warp
// and a block holds 8 independent groups; for d >= 512 a group is the whole block.
//
// The rotation and QJL products are CUDA-core FMA loops over the stored matrices
// (fp32 accumulate), the RHT is an in-register / shuffle / shared-memory butterfly.
// The specialised tensor-core encoder for d = 128 lives in encode_tc.cu.
#include <mutex>

#include "common.cuh"
#include "prep.cuh"

namespace tq {
namespace {

template <int NT>
__device__ __forceinline__ void group_sync() {
    if constexpr (NT == 32) __syncwarp(); else __syncthreads();
}

// Sum over the NT threads of a group; `red` holds NT/32 floats (used when NT > 32).
template <int NT>
__device__ __forceinline__ float group_sum(float v, float* red) {
    v = warp_sum(v);
    if constexpr (NT == 32) {
        return v;
    } else {
        const int w = threadIdx.x >> 5;
        if ((threadIdx.x & 31) == 0) red[w] = v;
        __syncthreads();
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < NT / 32; ++i) s += red[i];
        __syncthreads();
        return s;
    }
}

// In-place unnormalised Sylvester Walsh-Hadamard transform of the group's vector:
// stages with stride < E in registers, then across threads (shuffle or shared memory).
// For element j with bit h clear: y_j = x_j + x_{j+h}; with it set: y_j = x_{j-h} - x_j.
template <int E, int NT>
__device__ __forceinline__ void fwht(float (&v)[E], int tid, float* xch) {
#pragma unroll
    for (int h = 1; h < E; h <<= 1) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            if ((e & h) == 0 && e + h < E) {   // always true for the power-of-two E the RHT uses
                const float a = v[e], b = v[e + h];
                v[e] = a + b;
                v[e + h] = a - b;
            }
        }
    }
#pragma unroll
    for (int m = 1; m < NT; m <<= 1) {
        if (m < 32) {
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float o = __shfl_xor_sync(0xffffffffu, v[e], m);
                v[e] = (tid & m) ? (o - v[e]) : (v[e] + o);
            }
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) xch[tid * E + e] = v[e];
            __syncthreads();
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float o = xch[(tid ^ m) * E + e];
                v[e] = (tid & m) ? (o - v[e]) : (v[e] + o);
            }
            __syncthreads();
        }
    }
}

template <int NT>
__device__ __forceinline__ int groups_per_block() { return NT == 32 ? 8 : 1; }

// ------------------------------------------------------------------------------------
// Encode: norm, rotate, normalise, quantize, (prod) residual + QJL signs, pack.
// Per group shared memory: d floats (broadcast buffer) + d bytes codes + d bytes signs.
// ------------------------------------------------------------------------------------
template <int E, int NT>
__global__ void __launch_bounds__(NT == 32 ? 256 : NT)
encode_kernel(const DevState st, const void* __restrict__ x, int dtype, int64_t n, int64_t ld,
              const int32_t* __restrict__ chan, int64_t ostride, uint8_t* __restrict__ codes,
              uint8_t* __restrict__ qjl, float* __restrict__ norms, float* __restrict__ rnorms,
              uint16_t* __restrict__ r2out, float* __restrict__ rho_out, int rho_stride) {
    constexpr int D = NT * E;
    constexpr int GPB = (NT == 32) ? 8 : 1;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float* ctab = reinterpret_cast<float*>(smem_raw);                 // kMaxLevels
    float* ttab = ctab + kMaxLevels;                                   // kMaxLevels
    float* red = ttab + kMaxLevels;                                    // 8
    const int g = threadIdx.x / NT;
    const int tid = threadIdx.x % NT;
    float* vbuf = red + 8 + g * D;                                     // D floats per group
    uint8_t* cbuf = reinterpret_cast<uint8_t*>(red + 8 + GPB * D) + g * 2 * D;
    uint8_t* zbuf = cbuf + D;
    for (int i = threadIdx.x; i < st.L; i += blockDim.x) {
        ctab[i] = st.c[i];
        ttab[i] = st.t[i];
    }
    __syncthreads();
    const bool prod = (st.mode == TQ_PROD);
    const int lane = threadIdx.x & 31;
    const int warp_in_group = tid >> 5;
    constexpr int WPG = NT / 32;

    for (int64_t vec = (int64_t)blockIdx.x * GPB + g; vec < n; vec += (int64_t)gridDim.x * GPB) {
        float xv[E];
        if (chan == nullptr) {
            load_elems<E>(x, dtype, vec * ld + (int64_t)tid * E, xv);
        } else {   // element j of this vector is channel chan[j] of the input row
#pragma unroll
            for (int e = 0; e < E; ++e) xv[e] = mat_elem(x, dtype, vec * ld + __ldg(chan + tid * E + e));
        }
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) ss = fmaf(xv[e], xv[e], ss);
        const float nu = sqrtf(group_sum<NT>(ss, red));
        float y[E];
        if (st.rot == TQ_ROT_RHT) {
#pragma unroll
            for (int e = 0; e < E; ++e) y[e] = rht_neg(st, tid * E + e) ? -xv[e] : xv[e];
            if constexpr ((D & (D - 1)) == 0) {
                fwht<E, NT>(y, tid, vbuf);
            } else {   // d = 12 * 2^k
#pragma unroll
                for (int e = 0; e < E; ++e) vbuf[tid * E + e] = y[e];
                group_sync<NT>();
                kron_hadamard(vbuf, D, st.h12, false, tid, NT, [] { group_sync<NT>(); });
#pragma unroll
                for (int e = 0; e < E; ++e) y[e] = vbuf[tid * E + e];
                group_sync<NT>();
            }
            const float sc = (nu > 0.f) ? st.rsqrt_d / nu : 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) y[e] *= sc;
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) vbuf[tid * E + e] = xv[e];
            group_sync<NT>();
            matvec_cols<E>(st.piT, st.mat_dtype, D, tid * E, vbuf, y);
            group_sync<NT>();
            const float sc = (nu > 0.f) ? 1.f / nu : 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) y[e] *= sc;
        }
        // quantize (+ residual)
        float r[E];
        float rr = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            int c = 0;
            if (st.b_mse > 0) c = quantize_coord(st, ttab, y[e]);
            cbuf[tid * E + e] = (uint8_t)c;
            r[e] = (nu > 0.f) ? (y[e] - (st.b_mse > 0 ? ctab[c] : 0.f)) : 0.f;
            rr = fmaf(r[e], r[e], rr);
        }
        if (r2out != nullptr) {
            // prod with S r on the tensor core: the residual as [r_hi | r_lo] bf16 rows
            // (r_lo = bf16(r - r_hi)) and ||r||^2 for the signs pass
            if constexpr (E == 8) {   // 16-byte stores of the thread's 8 hi and 8 lo halves
                uint32_t hw[4], lw[4];
#pragma unroll
                for (int e = 0; e < E; e += 2) {
                    uint32_t hb[2], lb[2];
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        hb[k] = __bfloat16_as_ushort(__float2bfloat16_rn(r[e + k]));
                        const float lo = r[e + k] - __uint_as_float(hb[k] << 16);
                        lb[k] = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
                    }
                    hw[e / 2] = hb[0] | (hb[1] << 16);
                    lw[e / 2] = lb[0] | (lb[1] << 16);
                }
                *reinterpret_cast<uint4*>(r2out + vec * 2 * D + tid * E) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                *reinterpret_cast<uint4*>(r2out + vec * 2 * D + D + tid * E) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            } else {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int j = tid * E + e;
                    const uint16_t hb = __bfloat16_as_ushort(__float2bfloat16_rn(r[e]));
                    const float lo = r[e] - __uint_as_float((uint32_t)hb << 16);
                    r2out[vec * 2 * D + j] = hb;
                    r2out[vec * 2 * D + D + j] = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
                }
            }
            const float rsum = group_sum<NT>(rr, red);
            if (tid == 0) {
                norms[vec * ostride] = nu;
                rho_out[vec * rho_stride] = rsum;
                for (int t = 1; t < rho_stride; ++t) rho_out[vec * rho_stride + t] = 0.f;
            }
        } else if (prod) {
            const float rho = sqrtf(group_sum<NT>(rr, red));
#pragma unroll
            for (int e = 0; e < E; ++e) vbuf[tid * E + e] = r[e];
            group_sync<NT>();
            float s[E];
            matvec_cols<E>(st.sT, st.mat_dtype, D, tid * E, vbuf, s);
#pragma unroll
            for (int e = 0; e < E; ++e) zbuf[tid * E + e] = (s[e] >= 0.f) ? 1 : 0;
            if (tid == 0) {
                norms[vec * ostride] = nu;
                rnorms[vec * ostride] = rho;
            }
        } else if (tid == 0) {
            norms[vec * ostride] = nu;
        }
        group_sync<NT>();
        // pack codes: stream bit p = 32w + lane -> code p / b, bit p % b
        if (st.b_mse > 0) {
            const int b = st.b_mse;
            const int W = b * D / 32;
            uint32_t* out = reinterpret_cast<uint32_t*>(codes + vec * ostride * st.code_bytes);
            for (int w = warp_in_group; w < W; w += WPG) {
                const int p = 32 * w + lane;
                const int j = p / b;
                const uint32_t bit = (cbuf[j] >> (p - j * b)) & 1u;
                const uint32_t word = __ballot_sync(0xffffffffu, bit);
                if (lane == 0) out[w] = word;
            }
        }
        if (prod && r2out == nullptr) {
            uint32_t* out = reinterpret_cast<uint32_t*>(qjl + vec * ostride * st.qjl_bytes);
            for (int w = warp_in_group; w < D / 32; w += WPG) {
                const uint32_t word = __ballot_sync(0xffffffffu, zbuf[32 * w + lane]);
                if (lane == 0) out[w] = word;
            }
        }
        group_sync<NT>();
    }
}

// ------------------------------------------------------------------------------------
// Dequant: x~ = ||x|| Pi^T (c[idx] + ||r|| sqrt(pi/2)/d S^T (2z-1)).
// ------------------------------------------------------------------------------------
template <int E, int NT>
__global__ void __launch_bounds__(NT == 32 ? 256 : NT)
dequant_kernel(const DevState st, const uint8_t* __restrict__ codes, const uint8_t* __restrict__ qjl,
               const float* __restrict__ norms, const float* __restrict__ rnorms, int64_t n,
               const int32_t* __restrict__ chan, int64_t ldo, float* __restrict__ out) {
    constexpr int D = NT * E;
    constexpr int GPB = (NT == 32) ? 8 : 1;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    float* ctab = reinterpret_cast<float*>(smem_raw);
    const int g = threadIdx.x / NT;
    const int tid = threadIdx.x % NT;
    float* vbuf = ctab + kMaxLevels + g * D;
    for (int i = threadIdx.x; i < st.L; i += blockDim.x) ctab[i] = st.c[i];
    __syncthreads();
    const bool prod = (qjl != nullptr);
    const int nwords = st.code_bytes / 4;
    for (int64_t vec = (int64_t)blockIdx.x * GPB + g; vec < n; vec += (int64_t)gridDim.x * GPB) {
        float yt[E];
        const uint32_t* row = reinterpret_cast<const uint32_t*>(codes + vec * st.code_bytes);
#pragma unroll
        for (int e = 0; e < E; ++e)
            yt[e] = (st.b_mse > 0) ? ctab[extract_code(row, nwords, tid * E + e, st.b_mse)] : 0.f;
        if (prod) {
            const uint8_t* zr = qjl + vec * st.qjl_bytes;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const int j = tid * E + e;
                vbuf[j] = ((__ldg(zr + (j >> 3)) >> (j & 7)) & 1u) ? 1.f : -1.f;
            }
            group_sync<NT>();
            float t[E];
            matvec_cols<E>(st.s, st.mat_dtype, D, tid * E, vbuf, t);   // (S^T z)_k = sum_j S[j][k] z_j
            group_sync<NT>();
            const float a = __ldg(rnorms + vec) * st.qjl_scale;
#pragma unroll
            for (int e = 0; e < E; ++e) yt[e] = fmaf(a, t[e], yt[e]);
        }
        float xo[E];
        if (st.rot == TQ_ROT_RHT) {
            if constexpr ((D & (D - 1)) == 0) {
                fwht<E, NT>(yt, tid, vbuf);
            } else {   // d = 12 * 2^k: the transposed transform
#pragma unroll
                for (int e = 0; e < E; ++e) vbuf[tid * E + e] = yt[e];
                group_sync<NT>();
                kron_hadamard(vbuf, D, st.h12, true, tid, NT, [] { group_sync<NT>(); });
#pragma unroll
                for (int e = 0; e < E; ++e) yt[e] = vbuf[tid * E + e];
                group_sync<NT>();
            }
#pragma unroll
            for (int e = 0; e < E; ++e) xo[e] = (rht_neg(st, tid * E + e) ? -yt[e] : yt[e]) * st.rsqrt_d;
        } else {
#pragma unroll
            for (int e = 0; e < E; ++e) vbuf[tid * E + e] = yt[e];
            group_sync<NT>();
            matvec_cols<E>(st.pi, st.mat_dtype, D, tid * E, vbuf, xo);   // x_k = sum_j Pi[j][k] y_j
            group_sync<NT>();
        }
        const float nu = __ldg(norms + vec);
        if (chan == nullptr) {
            float* o = out + vec * ldo + tid * E;
#pragma unroll
            for (int e = 0; e < E; ++e) o[e] = xo[e] * nu;
        } else {   // element j goes to channel chan[j] of the output row
#pragma unroll
            for (int e = 0; e < E; ++e) out[vec * ldo + __ldg(chan + tid * E + e)] = xo[e] * nu;
        }
    }
}

// The two sums of an estimate for up to QT queries against one key:
//   a1 = sum_j qp_j c[idx_j],  a2 = sum_j u_j (2 z_j - 1).
template <int QT>
__device__ __forceinline__ void score_sums(const DevState& st, const float* ctab, const float* qp,
                                           const float* u, int nqt, const uint8_t* codes,
                                           const uint8_t* qjl, int64_t key, float (&a1)[QT],
                                           float (&a2)[QT]) {
    const int d = st.d;
#pragma unroll
    for (int i = 0; i < QT; ++i) a1[i] = a2[i] = 0.f;
    if (st.b_mse > 0) {
        const uint32_t* row = reinterpret_cast<const uint32_t*>(codes + key * st.code_bytes);
        const int b = st.b_mse;
        const uint32_t mask = (1u << b) - 1u;
        uint64_t buf = 0;
        int have = 0, wi = 0;
        for (int j = 0; j < d; ++j) {
            if (have < b) {
                buf |= (uint64_t)__ldg(row + wi++) << have;
                have += 32;
            }
            const float cv = ctab[buf & mask];
            buf >>= b;
            have -= b;
#pragma unroll
            for (int i = 0; i < QT; ++i)
                if (i < nqt) a1[i] = fmaf(qp[i * d + j], cv, a1[i]);
        }
    }
    if (qjl != nullptr) {
        const uint32_t* zr = reinterpret_cast<const uint32_t*>(qjl + key * st.qjl_bytes);
        for (int w = 0; w < d / 32; ++w) {
            const uint32_t word = __ldg(zr + w);
            for (int bt = 0; bt < 32; ++bt) {
                const float sg = ((word >> bt) & 1u) ? 1.f : -1.f;
                const int j = w * 32 + bt;
#pragma unroll
                for (int i = 0; i < QT; ++i)
                    if (i < nqt) a2[i] = fmaf(u[i * d + j], sg, a2[i]);
            }
        }
    }
}

constexpr int kScoreQT = 8;
constexpr int kScoreThreads = 256;

size_t score_smem_bytes(int d) { return (size_t)(kMaxLevels + 3 * kScoreQT * d) * sizeof(float) + kPrepStageBytes; }

__global__ void __launch_bounds__(kScoreThreads)
score_kernel(const DevState st, const void* __restrict__ q, int qdtype, int64_t nq,
             const uint8_t* __restrict__ codes, const uint8_t* __restrict__ qjl,
             const float* __restrict__ norms, const float* __restrict__ rnorms, int64_t n,
             int accumulate, float* __restrict__ scores) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int d = st.d;
    float* ctab = reinterpret_cast<float*>(smem_raw);
    float* qs = ctab + kMaxLevels;
    float* qp = qs + kScoreQT * d;
    float* u = qp + kScoreQT * d;
    unsigned char* stage = reinterpret_cast<unsigned char*>(u + kScoreQT * d);
    const int64_t grp = blockIdx.z;
    const int64_t q0 = (int64_t)blockIdx.y * kScoreQT;
    const int nqt = (int)(nq - q0 < kScoreQT ? nq - q0 : kScoreQT);
    for (int i = threadIdx.x; i < st.L; i += blockDim.x) ctab[i] = st.c[i];
    const size_t qelem = (qdtype == TQ_F32) ? 4 : 2;
    prep_queries_dev(st, reinterpret_cast<const unsigned char*>(q) + (size_t)((grp * nq + q0) * d) * qelem,
                 qdtype, nqt, qs, qp, u, stage);
    for (int64_t key = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; key < n;
         key += (int64_t)gridDim.x * blockDim.x) {
        const int64_t gk = grp * n + key;
        float a1[kScoreQT], a2[kScoreQT];
        score_sums<kScoreQT>(st, ctab, qp, u, nqt, codes, qjl, gk, a1, a2);
        const float nu = __ldg(norms + gk);
        const float g2 = (qjl != nullptr) ? __ldg(rnorms + gk) * st.qjl_scale : 0.f;
        for (int i = 0; i < nqt; ++i) {
            float* dst = scores + (grp * nq + q0 + i) * n + key;
            const float v = nu * fmaf(g2, a2[i], a1[i]);
            *dst = accumulate ? *dst + v : v;
        }
    }
}

// ------------------------------------------------------------------------------------
// Decode attention, split over tokens (flash-decoding style), then a combine launch.
// Partial record per (head, split): m, l, acc[d] (value sum in the rotated domain).
// ------------------------------------------------------------------------------------
constexpr int kAttThreads = 256;
constexpr int kAttMaxJ = kMaxDim / kAttThreads;   // coordinates per thread when d > 256

size_t attend_smem_bytes(int d) {
    const int accs = (d > kAttThreads) ? d : kAttThreads;
    return (size_t)(2 * kMaxLevels + 3 * d + kAttThreads + 32 + accs) * sizeof(float) + kPrepStageBytes;
}

__global__ void __launch_bounds__(kAttThreads)
attend_split_kernel(const DevState ks, const DevState vs, const void* __restrict__ q, int qdtype,
                    int64_t T, int G, int64_t Tcap, int64_t chunk, const uint8_t* __restrict__ kcodes,
                    const uint8_t* __restrict__ kqjl, const float* __restrict__ knorms,
                    const float* __restrict__ krnorms, const uint8_t* __restrict__ vcodes,
                    const float* __restrict__ vnorms, float scale, float* __restrict__ part) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int d = ks.d;
    const int h = blockIdx.y;
    const int split = blockIdx.x;
    const int nsplit = gridDim.x;
    float* kc = reinterpret_cast<float*>(smem_raw);      // K centroids
    float* vc = kc + kMaxLevels;                          // V centroids
    float* qs = vc + kMaxLevels;                          // d
    float* qp = qs + d;                                   // d
    float* u = qp + d;                                    // d
    float* wt = u + d;                                    // kAttThreads weights p_t * ||v_t||
    float* red = wt + kAttThreads;                        // 32
    float* accs = red + 32;                               // max(d, kAttThreads)
    unsigned char* stage = reinterpret_cast<unsigned char*>(accs + (d > kAttThreads ? d : kAttThreads));
    for (int i = threadIdx.x; i < ks.L; i += blockDim.x) kc[i] = ks.c[i];
    for (int i = threadIdx.x; i < vs.L; i += blockDim.x) vc[i] = vs.c[i];
    const size_t qelem = (qdtype == TQ_F32) ? 4 : 2;
    prep_queries_dev(ks, reinterpret_cast<const unsigned char*>(q) + (size_t)h * d * qelem, qdtype, 1, qs, qp, u,
                     stage);

    const int64_t kvb = (int64_t)(h / G) * Tcap;   // planes of this query head's KV head
    const int64_t t_begin = (int64_t)split * chunk;
    const int64_t t_end = (T < t_begin + chunk) ? T : t_begin + chunk;
    // Value accumulation layout: d <= 256: `per` threads per coordinate split the tokens;
    // d > 256: each thread owns coordinates threadIdx.x + m*256 for all tokens.
    const int per = (d <= kAttThreads) ? kAttThreads / d : 1;
    const int jpt = (d <= kAttThreads) ? 1 : d / kAttThreads;
    const int j0 = (d <= kAttThreads) ? (threadIdx.x % d) : threadIdx.x;
    const int half = (d <= kAttThreads) ? (threadIdx.x / d) : 0;
    const bool vact = half < per;   // d not dividing 256: the last threads take no coordinate
    float acc[kAttMaxJ];
#pragma unroll
    for (int m = 0; m < kAttMaxJ; ++m) acc[m] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    const int vnw = vs.code_bytes / 4;
    for (int64_t t0 = t_begin; t0 < t_end; t0 += kAttThreads) {
        const int cnt = (int)(t_end - t0 < kAttThreads ? t_end - t0 : kAttThreads);
        float s = -INFINITY;
        if (threadIdx.x < cnt) {
            const int64_t gk = kvb + t0 + threadIdx.x;
            float a1[1], a2[1];
            score_sums<1>(ks, kc, qp, u, 1, kcodes, kqjl, gk, a1, a2);
            const float g2 = (kqjl != nullptr) ? __ldg(krnorms + gk) * ks.qjl_scale : 0.f;
            s = scale * __ldg(knorms + gk) * fmaf(g2, a2[0], a1[0]);
        }
        float mx = warp_max(s);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
        __syncthreads();
        float tmax = red[0];
        for (int i = 1; i < kAttThreads / 32; ++i) tmax = fmaxf(tmax, red[i]);
        __syncthreads();
        const float m_new = fmaxf(m_run, tmax);
        const float alpha = (m_run == -INFINITY) ? 0.f : __expf(m_run - m_new);
        const float p = (threadIdx.x < cnt) ? __expf(s - m_new) : 0.f;
        const float psum = warp_sum(p);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = psum;
        if (threadIdx.x < cnt) wt[threadIdx.x] = p * __ldg(vnorms + kvb + t0 + threadIdx.x);
        __syncthreads();
        float tsum = 0.f;
        for (int i = 0; i < kAttThreads / 32; ++i) tsum += red[i];
        l_run = l_run * alpha + tsum;
        m_run = m_new;
#pragma unroll
        for (int m = 0; m < kAttMaxJ; ++m) acc[m] *= alpha;
        for (int t = half; vact && t < cnt; t += per) {
            const uint32_t* row =
                reinterpret_cast<const uint32_t*>(vcodes + (kvb + t0 + t) * vs.code_bytes);
            const float w = wt[t];
#pragma unroll
            for (int m = 0; m < kAttMaxJ; ++m)
                if (m < jpt) acc[m] = fmaf(w, vc[extract_code(row, vnw, j0 + m * kAttThreads, vs.b_mse)], acc[m]);
        }
        __syncthreads();
    }
    float* rec = part + ((int64_t)h * nsplit + split) * (d + 2);
    if (d <= kAttThreads) {
        if (vact) accs[half * d + j0] = acc[0];
        __syncthreads();
        for (int jj = threadIdx.x; jj < d; jj += blockDim.x) {
            float a = 0.f;
            for (int hh = 0; hh < per; ++hh) a += accs[hh * d + jj];
            rec[2 + jj] = a;
        }
    } else {
        for (int m = 0; m < jpt; ++m) rec[2 + j0 + m * kAttThreads] = acc[m];
    }
    if (threadIdx.x == 0) {
        rec[0] = m_run;
        rec[1] = l_run;
    }
}

// Value sums of a decode step whose scores are given: per head h, s_t = scale * scores[h][t];
// block (split, h) writes the record (m, l, acc[dv]) of its tokens, acc in the rotated domain
// of the value state (the layout attend_combine_kernel merges). Used for channel-split caches,
// where each channel group of V has its own state and gets its own records.
__global__ void __launch_bounds__(kAttThreads)
attend_values_kernel(const DevState vs, const float* __restrict__ scores, float scale, int64_t T, int64_t chunk,
                     const uint8_t* __restrict__ vcodes, const float* __restrict__ vnorms, float* __restrict__ part) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int d = vs.d;
    const int h = blockIdx.y;
    const int split = blockIdx.x;
    const int nsplit = gridDim.x;
    float* vc = reinterpret_cast<float*>(smem_raw);       // V centroids
    float* wt = vc + kMaxLevels;                          // kAttThreads weights p_t * ||v_t||
    float* red = wt + kAttThreads;                        // 32
    float* accs = red + 32;                               // max(d, kAttThreads)
    for (int i = threadIdx.x; i < vs.L; i += blockDim.x) vc[i] = vs.c[i];
    __syncthreads();
    const int64_t t_begin = (int64_t)split * chunk;
    const int64_t t_end = (T < t_begin + chunk) ? T : t_begin + chunk;
    const int per = (d <= kAttThreads) ? kAttThreads / d : 1;
    const int jpt = (d <= kAttThreads) ? 1 : d / kAttThreads;
    const int j0 = (d <= kAttThreads) ? (threadIdx.x % d) : threadIdx.x;
    const int half = (d <= kAttThreads) ? (threadIdx.x / d) : 0;
    const bool vact = half < per;
    float acc[kAttMaxJ];
#pragma unroll
    for (int m = 0; m < kAttMaxJ; ++m) acc[m] = 0.f;
    float m_run = -INFINITY, l_run = 0.f;
    const int vnw = vs.code_bytes / 4;
    for (int64_t t0 = t_begin; t0 < t_end; t0 += kAttThreads) {
        const int cnt = (int)(t_end - t0 < kAttThreads ? t_end - t0 : kAttThreads);
        const float s = (threadIdx.x < cnt) ? scale * __ldg(scores + (int64_t)h * T + t0 + threadIdx.x) : -INFINITY;
        float mx = warp_max(s);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
        __syncthreads();
        float tmax = red[0];
        for (int i = 1; i < kAttThreads / 32; ++i) tmax = fmaxf(tmax, red[i]);
        __syncthreads();
        const float m_new = fmaxf(m_run, tmax);
        const float alpha = (m_run == -INFINITY) ? 0.f : __expf(m_run - m_new);
        const float p = (threadIdx.x < cnt) ? __expf(s - m_new) : 0.f;
        const float psum = warp_sum(p);
        if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = psum;
        if (threadIdx.x < cnt) wt[threadIdx.x] = p * __ldg(vnorms + (int64_t)h * T + t0 + threadIdx.x);
        __syncthreads();
        float tsum = 0.f;
        for (int i = 0; i < kAttThreads / 32; ++i) tsum += red[i];
        l_run = l_run * alpha + tsum;
        m_run = m_new;
#pragma unroll
        for (int m = 0; m < kAttMaxJ; ++m) acc[m] *= alpha;
        for (int t = half; vact && t < cnt; t += per) {
            const uint32_t* row =
                reinterpret_cast<const uint32_t*>(vcodes + ((int64_t)h * T + t0 + t) * vs.code_bytes);
            const float w = wt[t];
#pragma unroll
            for (int m = 0; m < kAttMaxJ; ++m)
                if (m < jpt) acc[m] = fmaf(w, vc[extract_code(row, vnw, j0 + m * kAttThreads, vs.b_mse)], acc[m]);
        }
        __syncthreads();
    }
    float* rec = part + ((int64_t)h * nsplit + split) * (d + 2);
    if (d <= kAttThreads) {
        if (vact) accs[half * d + j0] = acc[0];
        __syncthreads();
        for (int jj = threadIdx.x; jj < d; jj += blockDim.x) {
            float a = 0.f;
            for (int hh = 0; hh < per; ++hh) a += accs[hh * d + jj];
            rec[2 + jj] = a;
        }
    } else {
        for (int m = 0; m < jpt; ++m) rec[2 + j0 + m * kAttThreads] = acc[m];
    }
    if (threadIdx.x == 0) {
        rec[0] = m_run;
        rec[1] = l_run;
    }
}

// Shared memory of attend_combine_kernel: o[d], partial sums [max(256, d)], the splits'
// weights [nsplit], a reduction scratch [32].
size_t combine_smem_bytes(int d, int nsplit) { return (size_t)(d + std::max(256, d) + nsplit + 32) * sizeof(float); }

// Merge of the splits' (m, l, acc[d]) records per head, then out = Pi_V^T o. The splits are
// reduced in parallel: their maxima and weights exp(m_s - M) by a block reduction, the value
// sums by P = 256 / d groups of threads over interleaved splits (independent loads in flight).
__global__ void __launch_bounds__(256)
attend_combine_kernel(const DevState vs, int nsplit, const float* __restrict__ part, const int32_t* __restrict__ chan,
                      int64_t ldo, float* __restrict__ out) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int d = vs.d;
    const int h = blockIdx.x;
    const int tid = threadIdx.x, nt = blockDim.x;
    float* o = reinterpret_cast<float*>(smem_raw);   // d
    float* acc = o + d;                               // max(nt, d)
    float* w = acc + (nt > d ? nt : d);               // nsplit
    float* red = w + nsplit;                          // 32
    const int64_t rs = d + 2;
    const float* base = part + (int64_t)h * nsplit * rs;
    float mloc = -INFINITY;
    for (int s = tid; s < nsplit; s += nt) mloc = fmaxf(mloc, base[s * rs]);
    mloc = warp_max(mloc);
    if ((tid & 31) == 0) red[tid >> 5] = mloc;
    __syncthreads();
    float M = red[0];
    for (int i = 1; i < nt / 32; ++i) M = fmaxf(M, red[i]);
    __syncthreads();   // red is reused for the sum
    float lloc = 0.f;
    for (int s = tid; s < nsplit; s += nt) {
        const float m = base[s * rs];
        const float wt = (m == -INFINITY) ? 0.f : __expf(m - M);
        w[s] = wt;
        lloc = fmaf(base[s * rs + 1], wt, lloc);
    }
    lloc = warp_sum(lloc);
    if ((tid & 31) == 0) red[tid >> 5] = lloc;
    __syncthreads();   // also publishes w
    float Lsum = 0.f;
    for (int i = 0; i < nt / 32; ++i) Lsum += red[i];
    const int P = (d < nt) ? nt / d : 1;
    for (int idx = tid; idx < P * d; idx += nt) {
        const int j = idx % d, p = idx / d;
        float a0 = 0.f, a1 = 0.f;
        int s = p;
#pragma unroll 4
        for (; s + P < nsplit; s += 2 * P) {
            a0 = fmaf(w[s], base[s * rs + 2 + j], a0);
            a1 = fmaf(w[s + P], base[(s + P) * rs + 2 + j], a1);
        }
        if (s < nsplit) a0 = fmaf(w[s], base[s * rs + 2 + j], a0);
        acc[idx] = a0 + a1;
    }
    __syncthreads();
    for (int j = tid; j < d; j += nt) {
        float a = 0.f;
        for (int p = 0; p < P; ++p) a += acc[p * d + j];
        o[j] = a / Lsum;
    }
    __syncthreads();
    // out = Pi_V^T o
    if (vs.rot == TQ_ROT_RHT) {
        if ((d & (d - 1)) == 0) {
            for (int hh = 1; hh < d; hh <<= 1) {
                for (int p = threadIdx.x; p < d / 2; p += blockDim.x) {
                    const int j = (p / hh) * 2 * hh + (p % hh);
                    const float a = o[j], b = o[j + hh];
                    o[j] = a + b;
                    o[j + hh] = a - b;
                }
                __syncthreads();
            }
        } else {   // d = 12 * 2^k: the transposed transform
            kron_hadamard(o, d, vs.h12, true, threadIdx.x, blockDim.x, [] { __syncthreads(); });
        }
        for (int k = threadIdx.x; k < d; k += blockDim.x)
            out[(int64_t)h * ldo + (chan ? __ldg(chan + k) : k)] = (rht_neg(vs, k) ? -o[k] : o[k]) * vs.rsqrt_d;
    } else {
        for (int k = threadIdx.x; k < d; k += blockDim.x) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
            for (int j = 0; j < d; j += 2) {   // d is even
                a0 = fmaf(mat_elem(vs.pi, vs.mat_dtype, (int64_t)j * d + k), o[j], a0);
                a1 = fmaf(mat_elem(vs.pi, vs.mat_dtype, (int64_t)(j + 1) * d + k), o[j + 1], a1);
            }
            out[(int64_t)h * ldo + (chan ? __ldg(chan + k) : k)] = a0 + a1;
        }
    }
}

// ------------------------------------------------------------------------------------
// Top-k search: per (query tile, key block) candidates, then a per-query merge.
// Order: larger value first; equal values -> lower index first.
// ------------------------------------------------------------------------------------
constexpr int kSearchThreads = 256;

__device__ __forceinline__ bool better(float v1, int64_t i1, float v2, int64_t i2) {
    return (v1 > v2) || (v1 == v2 && i1 < i2);
}

// Block-wide selection of the best (v, i) among the threads' current candidates.
__device__ __forceinline__ void block_best(float v, int64_t i, float* rv, int64_t* ri, float& bv, int64_t& bi) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int64_t oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (better(ov, oi, v, i)) {
            v = ov;
            i = oi;
        }
    }
    const int w = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
        rv[w] = v;
        ri[w] = i;
    }
    __syncthreads();
    bv = rv[0];
    bi = ri[0];
    for (int k = 1; k < (int)(blockDim.x >> 5); ++k)
        if (better(rv[k], ri[k], bv, bi)) {
            bv = rv[k];
            bi = ri[k];
        }
    __syncthreads();
}

// Scores of a block of keys for up to kScoreQT queries, then the block's k best per query.
// Taken slots are overwritten with NaN, which never compares better.
__global__ void __launch_bounds__(kSearchThreads)
search_block_kernel(const DevState st, const void* __restrict__ q, int qdtype, int64_t nq,
                    const uint8_t* __restrict__ codes, const uint8_t* __restrict__ qjl,
                    const float* __restrict__ norms, const float* __restrict__ rnorms, int64_t n, int k,
                    int block_keys, float* __restrict__ cand_v, int64_t* __restrict__ cand_i) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int d = st.d;
    float* ctab = reinterpret_cast<float*>(smem_raw);
    float* qs = ctab + kMaxLevels;
    float* qp = qs + kScoreQT * d;
    float* u = qp + kScoreQT * d;
    float* rv = u + kScoreQT * d;                                   // 8
    int64_t* ri = reinterpret_cast<int64_t*>(rv + 8);               // 8
    unsigned char* stage = reinterpret_cast<unsigned char*>(ri + 8);  // kPrepStageBytes
    float* sv = reinterpret_cast<float*>(stage + kPrepStageBytes);  // kScoreQT * block_keys
    const int64_t q0 = (int64_t)blockIdx.y * kScoreQT;
    const int nqt = (int)(nq - q0 < kScoreQT ? nq - q0 : kScoreQT);
    for (int i = threadIdx.x; i < st.L; i += blockDim.x) ctab[i] = st.c[i];
    const size_t qelem = (qdtype == TQ_F32) ? 4 : 2;
    prep_queries_dev(st, reinterpret_cast<const unsigned char*>(q) + (size_t)(q0 * d) * qelem, qdtype, nqt, qs, qp, u,
                     stage);
    const int64_t k0 = (int64_t)blockIdx.x * block_keys;
    for (int local = threadIdx.x; local < block_keys; local += blockDim.x) {
        const int64_t key = k0 + local;
        if (key < n) {
            float a1[kScoreQT], a2[kScoreQT];
            score_sums<kScoreQT>(st, ctab, qp, u, nqt, codes, qjl, key, a1, a2);
            const float nu = __ldg(norms + key);
            const float g2 = (qjl != nullptr) ? __ldg(rnorms + key) * st.qjl_scale : 0.f;
            for (int i = 0; i < nqt; ++i) sv[i * block_keys + local] = nu * fmaf(g2, a2[i], a1[i]);
        } else {
            for (int i = 0; i < nqt; ++i) sv[i * block_keys + local] = __int_as_float(0x7fc00000);
        }
    }
    __syncthreads();
    const int64_t nblk = gridDim.x;
    for (int i = 0; i < nqt; ++i) {
        float* row = sv + i * block_keys;
        for (int sel = 0; sel < k; ++sel) {
            float bv = -INFINITY;
            int64_t bi = INT64_MAX;
            for (int t = threadIdx.x; t < block_keys; t += blockDim.x)
                if (better(row[t], k0 + t, bv, bi)) {
                    bv = row[t];
                    bi = k0 + t;
                }
            float wv;
            int64_t wi;
            block_best(bv, bi, rv, ri, wv, wi);
            if (threadIdx.x == 0) {
                const int64_t o = ((q0 + i) * nblk + blockIdx.x) * k + sel;
                cand_v[o] = wv;
                cand_i[o] = wi;
                if (wi != INT64_MAX) row[wi - k0] = __int_as_float(0x7fc00000);
            }
            __syncthreads();
        }
    }
}

__global__ void __launch_bounds__(kSearchThreads)
search_merge_kernel(int64_t ncand, int k, const float* __restrict__ cand_v, const int64_t* __restrict__ cand_i,
                    int64_t* __restrict__ idx, float* __restrict__ vals) {
    __shared__ float rv[8];
    __shared__ int64_t ri[8];
    __shared__ int64_t taken[64];
    const int64_t qi = blockIdx.x;
    const float* cv = cand_v + qi * ncand;
    const int64_t* ci = cand_i + qi * ncand;
    for (int sel = 0; sel < k; ++sel) {
        float bv = -INFINITY;
        int64_t bi = INT64_MAX;
        for (int64_t t = threadIdx.x; t < ncand; t += blockDim.x) {
            const int64_t id = ci[t];
            if (id == INT64_MAX) continue;
            bool used = false;
            for (int s = 0; s < sel; ++s) used |= (taken[s] == id);
            if (!used && better(cv[t], id, bv, bi)) {
                bv = cv[t];
                bi = id;
            }
        }
        float wv;
        int64_t wi;
        block_best(bv, bi, rv, ri, wv, wi);
        if (threadIdx.x == 0) {
            taken[sel] = wi;
            idx[qi * k + sel] = wi;
            vals[qi * k + sel] = wv;
        }
        __syncthreads();
    }
}

}  // namespace

int launch_search_merge(int64_t nq, int64_t ncand, int k, const float* cand_v, const int64_t* cand_i, int64_t* idx,
                        float* vals, void* stream) {
    search_merge_kernel<<<(unsigned)nq, kSearchThreads, 0, (cudaStream_t)stream>>>(ncand, k, cand_v, cand_i, idx,
                                                                                   vals);
    return (int)cudaGetLastError();
}

namespace {

// ------------------------------------------------------------------------------------
// launch helpers
// ------------------------------------------------------------------------------------
int num_sms() {
    static int sms = 0;
    if (sms == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

template <int E, int NT>
int launch_encode_t(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, const int32_t* chan,
                    int64_t ostride, uint8_t* codes, uint8_t* qjl, float* norms, float* rnorms, uint16_t* r2out,
                    float* rho_out, int rho_stride, cudaStream_t s) {
    constexpr int GPB = (NT == 32) ? 8 : 1;
    const int threads = NT * GPB;
    const size_t smem = (2 * kMaxLevels + 8) * sizeof(float) + GPB * (NT * E) * (sizeof(float) + 2);
    auto kern = encode_kernel<E, NT>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int64_t blocks_needed = (n + GPB - 1) / GPB;
    const int blocks = (int)std::min<int64_t>(blocks_needed, (int64_t)num_sms() * 16);
    kern<<<blocks, threads, smem, s>>>(st, x, dtype, n, ld, chan, ostride, codes, qjl, norms, rnorms, r2out,
                                       rho_out, rho_stride);
    return (int)cudaGetLastError();
}

template <int E, int NT>
int launch_dequant_t(const DevState& st, const uint8_t* codes, const uint8_t* qjl, const float* norms,
                     const float* rnorms, int64_t n, const int32_t* chan, int64_t ldo, float* out, cudaStream_t s) {
    constexpr int GPB = (NT == 32) ? 8 : 1;
    const int threads = NT * GPB;
    const size_t smem = kMaxLevels * sizeof(float) + GPB * (NT * E) * sizeof(float);
    auto kern = dequant_kernel<E, NT>;
    if (smem > 48 * 1024) cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int64_t blocks_needed = (n + GPB - 1) / GPB;
    const int blocks = (int)std::min<int64_t>(blocks_needed, (int64_t)num_sms() * 16);
    kern<<<blocks, threads, smem, s>>>(st, codes, qjl, norms, rnorms, n, chan, ldo, out);
    return (int)cudaGetLastError();
}

// Calls f(E, NT) (as integral constants) for the thread layout of dimension d: a warp per
// vector with E = d / 32 coordinates per lane up to d = 256, a block of NT = d / 8 above.
template <typename F>
int with_layout(int d, F&& f) {
    using std::integral_constant;
    switch (d) {
        case 32: return f(integral_constant<int, 1>{}, integral_constant<int, 32>{});
        case 64: return f(integral_constant<int, 2>{}, integral_constant<int, 32>{});
        case 96: return f(integral_constant<int, 3>{}, integral_constant<int, 32>{});
        case 128: return f(integral_constant<int, 4>{}, integral_constant<int, 32>{});
        case 160: return f(integral_constant<int, 5>{}, integral_constant<int, 32>{});
        case 192: return f(integral_constant<int, 6>{}, integral_constant<int, 32>{});
        case 224: return f(integral_constant<int, 7>{}, integral_constant<int, 32>{});
        case 256: return f(integral_constant<int, 8>{}, integral_constant<int, 32>{});
        case 512: return f(integral_constant<int, 8>{}, integral_constant<int, 64>{});
        case 1024: return f(integral_constant<int, 8>{}, integral_constant<int, 128>{});
        case 1536: return f(integral_constant<int, 8>{}, integral_constant<int, 192>{});
        case 2048: return f(integral_constant<int, 8>{}, integral_constant<int, 256>{});
        default: return (int)cudaErrorInvalidValue;
    }
}

}  // namespace

int launch_encode_generic(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, const int32_t* chan,
                          int64_t ostride, uint8_t* codes, uint8_t* qjl, float* norms, float* rnorms, void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    return with_layout(st.d, [&](auto e, auto nt) {
        return launch_encode_t<decltype(e)::value, decltype(nt)::value>(st, x, dtype, n, ld, chan, ostride, codes,
                                                                         qjl, norms, rnorms, nullptr, nullptr, 0, s);
    });
}

// Codes, norms, the residual operand [r_hi | r_lo] and ||r||^2 (first of rho_stride slots) of
// a prod encode whose S r runs on the tensor core.
bool residual_rht_supported(const DevState& st);
int launch_residual_rht(const DevState& st, const void* x, int64_t n, int64_t ld, uint8_t* codes, float* norms,
                        uint16_t* r2out, float* rho_out, int rho_stride, void* stream);

int launch_encode_residual(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, uint8_t* codes,
                           float* norms, uint16_t* r2out, float* rho_out, int rho_stride, void* stream) {
    if (dtype == TQ_BF16 && residual_rht_supported(st))   // warp per vector, Hadamard in registers
        return launch_residual_rht(st, x, n, ld, codes, norms, r2out, rho_out, rho_stride, stream);
    cudaStream_t s = (cudaStream_t)stream;
    return with_layout(st.d, [&](auto e, auto nt) {
        return launch_encode_t<decltype(e)::value, decltype(nt)::value>(st, x, dtype, n, ld, nullptr, 1, codes,
                                                                         nullptr, norms, nullptr, r2out, rho_out,
                                                                         rho_stride, s);
    });
}

bool dequant_dense_supported(const DevState& st, int64_t n, const int32_t* chan, int64_t ldo);
int launch_dequant_dense(const DevState& st, const uint8_t* codes, const uint8_t* qjl, const float* norms,
                         const float* rnorms, int64_t n, int64_t ldo, float* out, void* stream);

int launch_dequant(const DevState& st, const uint8_t* codes, const uint8_t* qjl, const float* norms,
                   const float* rnorms, int64_t n, const int32_t* chan, int64_t ldo, float* out, void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    // d = 128 / 256 with dense fp32 matrices: the tiled dequantizer (both products as
    // register-tiled GEMMs over a tile of vectors)
    if (dequant_dense_supported(st, n, chan, ldo))
        return launch_dequant_dense(st, codes, qjl, norms, rnorms, n, ldo, out, stream);
    return with_layout(st.d, [&](auto e, auto nt) {
        return launch_dequant_t<decltype(e)::value, decltype(nt)::value>(st, codes, qjl, norms, rnorms, n, chan,
                                                                          ldo, out, s);
    });
}

namespace {
// out[r][j] = q[r][chan[j]] (elements of 2 or 4 bytes).
template <typename T>
__global__ void gather_rows_kernel(const T* __restrict__ q, int64_t count, int64_t ldq,
                                   const int32_t* __restrict__ chan, int m, T* __restrict__ out) {
    const int64_t total = count * m;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / m;
        out[i] = q[r * ldq + __ldg(chan + (i - r * m))];
    }
}
}  // namespace

int launch_gather_rows(const void* q, int dtype, int64_t count, int64_t ldq, const int32_t* chan, int m, void* out,
                       void* stream) {
    if (count <= 0 || m <= 0) return 0;
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t total = count * m;
    const int blocks = (int)std::min<int64_t>((total + 255) / 256, (int64_t)num_sms() * 8);
    if (dtype == TQ_F32)
        gather_rows_kernel<float><<<blocks, 256, 0, s>>>(reinterpret_cast<const float*>(q), count, ldq, chan, m,
                                                         reinterpret_cast<float*>(out));
    else
        gather_rows_kernel<uint16_t><<<blocks, 256, 0, s>>>(reinterpret_cast<const uint16_t*>(q), count, ldq, chan,
                                                            m, reinterpret_cast<uint16_t*>(out));
    return (int)cudaGetLastError();
}

bool score_lut_supported(const DevState& st);
size_t score_lut_floats(const DevState& st);
int launch_score_lut(const DevState& st, const void* q, int qdtype, int64_t groups, int64_t nq, const uint8_t* codes,
                     const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, int accumulate,
                     float* scores, void* ws, void* stream);

size_t score_ws_bytes(const DevState& st, int64_t groups, int64_t nq) {
    if (!score_lut_supported(st) || groups <= 0 || nq <= 0) return 0;
    return ((size_t)groups * nq * score_lut_floats(st) * sizeof(float) + 255) & ~(size_t)255;
}

int launch_score(const DevState& st, const void* q, int qdtype, int64_t groups, int64_t nq, const uint8_t* codes,
                 const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, int accumulate,
                 float* scores, void* ws, void* stream) {
    if (score_lut_supported(st))
        return launch_score_lut(st, q, qdtype, groups, nq, codes, qjl, norms, rnorms, n, accumulate, scores, ws,
                                stream);
    cudaStream_t s = (cudaStream_t)stream;
    const size_t smem = score_smem_bytes(st.d);
    if (smem > 48 * 1024) cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int64_t qtiles = (nq + kScoreQT - 1) / kScoreQT;
    if (qtiles > 65535) return (int)cudaErrorInvalidConfiguration;
    int64_t kb = (n + kScoreThreads - 1) / kScoreThreads;
    const int64_t want = std::max<int64_t>(1, (int64_t)num_sms() * 8 / std::max<int64_t>(1, qtiles * groups));
    kb = std::min<int64_t>(kb, std::max<int64_t>(want, 1));
    kb = std::min<int64_t>(kb, 1 << 20);
    dim3 grid((unsigned)kb, (unsigned)qtiles, (unsigned)groups);
    score_kernel<<<grid, kScoreThreads, smem, s>>>(st, q, qdtype, nq, codes, qjl, norms, rnorms, n, accumulate,
                                                     scores);
    return (int)cudaGetLastError();
}

namespace {
// Token splits of a decode step over `blocks_per_split` blocks (heads, or head groups).
int attend_splits(int blocks_per_split, int64_t T) {
    int64_t target = (int64_t)num_sms() * 4;
    int64_t sp = std::max<int64_t>(1, target / std::max(1, blocks_per_split));
    sp = std::min<int64_t>(sp, (T + kAttThreads - 1) / kAttThreads);
    return (int)std::max<int64_t>(1, sp);
}

// Splits the workspace provides for: enough for the largest head group (4 query heads of one
// KV head per block), so that grouped decode can use as many splits per head group.
int attend_max_splits(int H, int64_t T) { return attend_splits(std::max(1, H / 4), T); }
}  // namespace

// Query heads of one KV group that the table-based decode kernel takes per block.
int attend_heads_per_block(int G) { return (G % 4 == 0) ? 4 : ((G % 2 == 0) ? 2 : 1); }

bool attend_lut_supported(const DevState& ks, const DevState& vs, const void* kcodes, const void* kqjl,
                          const void* vcodes);
int launch_attend_lut_split(const DevState& ks, const DevState& vs, const float* luts, int H, int64_t T, int G,
                            int64_t Tcap, int nsplit, int64_t chunk, const uint8_t* kcodes, const uint8_t* kqjl,
                            const float* knorms, const float* krnorms, const uint8_t* vcodes, const float* vnorms,
                            float scale, float* part, void* stream);

size_t attend_part_bytes(const DevState& ks, int H, int64_t T) {
    const int sp = attend_max_splits(H, T);
    return ((size_t)H * sp * (ks.d + 2) * sizeof(float) + 255) & ~(size_t)255;
}

// Split partials, then (d = 128, 2- to 4-bit key codes) the per-head query tables.
size_t attend_workspace_bytes(const DevState& ks, int H, int64_t T) {
    if (H <= 0 || T <= 0) return 0;
    size_t b = attend_part_bytes(ks, H, T);
    if (ks.d == 128 && ks.b_mse >= 2 && ks.b_mse <= 4) b += (size_t)H * query_table_floats(ks) * sizeof(float);
    return b;
}

int launch_attend(const DevState& ks, const DevState& vs, const void* q, int qdtype, int H, int64_t T, int G,
                  int64_t Tcap, const uint8_t* kcodes, const uint8_t* kqjl, const float* knorms, const float* krnorms,
                  const uint8_t* vcodes, const float* vnorms, float scale, float* out, void* ws, size_t ws_bytes,
                  void* stream, const AppendRow* app) {
    cudaStream_t s = (cudaStream_t)stream;
    const bool lut = attend_lut_supported(ks, vs, kcodes, kqjl, vcodes);
    // the table kernel takes a group's query heads per block: as many splits per head group
    const int sp = lut ? attend_splits(H / attend_heads_per_block(G), T) : attend_splits(H, T);
    const int64_t chunk = (T + sp - 1) / sp;
    const int nsplit = (int)((T + chunk - 1) / chunk);
    float* part = reinterpret_cast<float*>(ws);
    cudaError_t e;
    if (app && !lut) {
        // the general path appends with the general encoder, one launch per plane set
        const int Hkv = H / G;
        e = (cudaError_t)launch_encode_strided(ks, app->k_new, app->dtype, Hkv, ks.d, Tcap, app->kcodes, app->kqjl,
                                               app->knorms, app->krnorms, stream);
        if (e == cudaSuccess)
            e = (cudaError_t)launch_encode_strided(vs, app->v_new, app->dtype, Hkv, vs.d, Tcap, app->vcodes,
                                                   app->vqjl, app->vnorms, app->vrnorms, stream);
        if (e != cudaSuccess) return (int)e;
    }
    if (lut) {
        float* luts = reinterpret_cast<float*>(reinterpret_cast<unsigned char*>(ws) + attend_part_bytes(ks, H, T));
        e = app ? (cudaError_t)launch_append_tables128(ks, vs, q, qdtype, H, luts, *app, stream)
                : (cudaError_t)launch_query_tables128(ks, q, qdtype, H, luts, stream);
        if (e == cudaSuccess)
            e = (cudaError_t)launch_attend_lut_split(ks, vs, luts, H, T, G, Tcap, nsplit, chunk, kcodes, kqjl, knorms,
                                                     krnorms, vcodes, vnorms, scale, part, stream);
    } else {
        const size_t smem = attend_smem_bytes(ks.d);
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(attend_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        dim3 grid((unsigned)nsplit, (unsigned)H);
        attend_split_kernel<<<grid, kAttThreads, smem, s>>>(ks, vs, q, qdtype, T, G, Tcap, chunk, kcodes, kqjl,
                                                             knorms, krnorms, vcodes, vnorms, scale, part);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return (int)e;
    attend_combine_kernel<<<H, 256, combine_smem_bytes(vs.d, nsplit), s>>>(vs, nsplit, part, nullptr, vs.d, out);
    return (int)cudaGetLastError();
}

// ------------------------------------------------------------------------------------
// Decode attention over channel-split K and V caches: scores summed over the two K groups
// into the workspace, then per V group the value records and their combine (Pi_V^T of the
// group, scattered to the group's channels of out).
// ------------------------------------------------------------------------------------
namespace {
size_t al256(size_t b) { return (b + 255) & ~(size_t)255; }
}  // namespace

// Layout: scores [H][T] | the queries' channel groups | V partials of each group | the K
// groups' score tables (one region, used by the two score launches in turn).
size_t split_attend_ws_bytes(const DevState& ko, const DevState& ki, int dv_outer, int dv, int H, int64_t T) {
    if (H <= 0 || T <= 0) return 0;
    const int sp = attend_splits(H, T);
    const int dk = ko.d + ki.d;
    return al256((size_t)H * T * sizeof(float)) + al256((size_t)H * dk * sizeof(float)) +
           al256((size_t)H * sp * (dv_outer + 2) * sizeof(float)) +
           al256((size_t)H * sp * (dv - dv_outer + 2) * sizeof(float)) +
           std::max(score_ws_bytes(ko, H, 1), score_ws_bytes(ki, H, 1));
}

int launch_split_attend(const DevState& ko, const DevState& ki, const int32_t* kchan, const DevState& vo,
                        const DevState& vi, const int32_t* vchan, const void* q, int qdtype, int H, int64_t T,
                        const SplitPlanes& kp, const SplitPlanes& vp, float scale, float* out, void* ws,
                        void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    const int dk = ko.d + ki.d, dv = vo.d + vi.d;
    const size_t es = (qdtype == TQ_F32) ? 4 : 2;
    unsigned char* w = reinterpret_cast<unsigned char*>(ws);
    float* scores = reinterpret_cast<float*>(w);
    w += al256((size_t)H * T * sizeof(float));
    unsigned char* qo = w;
    unsigned char* qi = w + (size_t)H * ko.d * es;   // ko.d * es is a multiple of 16
    w += al256((size_t)H * dk * sizeof(float));
    const int sp = attend_splits(H, T);
    const int64_t chunk = (T + sp - 1) / sp;
    const int nsplit = (int)((T + chunk - 1) / chunk);
    float* part_o = reinterpret_cast<float*>(w);
    float* part_i = reinterpret_cast<float*>(w + al256((size_t)H * sp * (vo.d + 2) * sizeof(float)));
    void* tables = w + al256((size_t)H * sp * (vo.d + 2) * sizeof(float)) +
                   al256((size_t)H * sp * (vi.d + 2) * sizeof(float));
    int e = launch_gather_rows(q, qdtype, H, dk, kchan, ko.d, qo, stream);
    if (e == 0) e = launch_gather_rows(q, qdtype, H, dk, kchan + ko.d, ki.d, qi, stream);
    if (e == 0)
        e = launch_score(ko, qo, qdtype, H, 1, kp.codes[0], kp.qjl[0], kp.norms[0], kp.rnorms[0], T, 0, scores,
                         tables, stream);
    if (e == 0)
        e = launch_score(ki, qi, qdtype, H, 1, kp.codes[1], kp.qjl[1], kp.norms[1], kp.rnorms[1], T, 1, scores,
                         tables, stream);
    if (e != 0) return e;
    for (int g = 0; g < 2; ++g) {
        const DevState& v = g ? vi : vo;
        float* part = g ? part_i : part_o;
        const size_t smem = (size_t)(kMaxLevels + kAttThreads + 32 + (v.d > kAttThreads ? v.d : kAttThreads)) *
                            sizeof(float);
        dim3 grid((unsigned)nsplit, (unsigned)H);
        attend_values_kernel<<<grid, kAttThreads, smem, s>>>(v, scores, scale, T, chunk, vp.codes[g], vp.norms[g],
                                                             part);
        attend_combine_kernel<<<H, 256, combine_smem_bytes(v.d, nsplit), s>>>(v, nsplit, part,
                                                                             g ? vchan + vo.d : vchan, dv, out);
    }
    return (int)cudaGetLastError();
}

// ------------------------------------------------------------------------------------
// Decode attention without a caller-supplied workspace.
//
// For callers that cannot allocate device memory (runtimes that hand all device memory to
// their own pool allocator, or latency-critical decode loops where an allocation's cost or
// possible failure is not acceptable): the split partials live
// in a fixed, file-scope device array instead of a workspace. Every GPU that loads the
// library holds this array until the process exits. All calls share it and it keeps the
// last call's contents; nothing in it needs to start at zero (each partial record is
// written before the combine step reads it). Calls whose work overlaps on the GPU (other
// streams, other threads) race on it and must be serialised by the caller.
// ------------------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_attend_scratch[kAttendStaticScratchBytes];

namespace {
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};
}  // namespace

int attend_static_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return (int)e;
    if (dev < 0 || dev >= kMaxDevices) return (int)cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
        // The array's name is a host-side stand-in: its device address must be looked up,
        // once per device, with that device current.
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attend_scratch);
        if (e != cudaSuccess) return (int)e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return 0;
}

namespace {
int search_block_keys(int d) {
    const size_t base = score_smem_bytes(d) + 8 * 4 + 8 * 8;
    const size_t budget = 200 * 1024;
    int keys = (int)((budget - base) / (kScoreQT * sizeof(float)));
    keys = std::min(keys, 4096);
    return std::max(kSearchThreads, keys / kSearchThreads * kSearchThreads);
}
int64_t search_blocks(int64_t n, int d) {
    const int bk = search_block_keys(d);
    return (n + bk - 1) / bk;
}
}  // namespace

bool search_tc_supported(const DevState& st, int qdtype, int k);
size_t search_tc_ws_bytes(const DevState& st, int64_t nq, int64_t n, int k);
int launch_search_tc(const DevState& st, const void* q, int qdtype, int64_t nq, const uint8_t* codes,
                     const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, int k, int64_t* idx,
                     float* vals, void* ws, void* stream);

size_t search_workspace_bytes(const DevState& st, int64_t nq, int64_t n, int k) {
    if (nq <= 0 || n <= 0) return 0;
    const size_t nc = (size_t)nq * search_blocks(n, st.d) * k;
    size_t b = nc * sizeof(float);
    b = (b + 255) & ~(size_t)255;
    b += nc * sizeof(int64_t);
    if (search_tc_supported(st, TQ_BF16, k)) {
        const size_t t = search_tc_ws_bytes(st, nq, n, k);
        if (t > b) b = t;
    }
    return b;
}

int launch_search(const DevState& st, const void* q, int qdtype, int64_t nq, const uint8_t* codes,
                  const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, int k, int64_t* idx,
                  float* vals, void* ws, size_t ws_bytes, void* stream) {
    (void)ws_bytes;
    if (search_tc_supported(st, qdtype, k) && nq <= (1 << 20))
        return launch_search_tc(st, q, qdtype, nq, codes, qjl, norms, rnorms, n, k, idx, vals, ws, stream);
    cudaStream_t s = (cudaStream_t)stream;
    const int bk = search_block_keys(st.d);
    const int64_t nblk = search_blocks(n, st.d);
    const size_t nc = (size_t)nq * nblk * k;
    float* cand_v = reinterpret_cast<float*>(ws);
    const size_t off = (nc * sizeof(float) + 255) & ~(size_t)255;
    int64_t* cand_i = reinterpret_cast<int64_t*>(reinterpret_cast<unsigned char*>(ws) + off);
    const size_t smem = score_smem_bytes(st.d) + 8 * 4 + 8 * 8 + (size_t)kScoreQT * bk * sizeof(float);
    cudaFuncSetAttribute(search_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    const int64_t qtiles = (nq + kScoreQT - 1) / kScoreQT;
    if (qtiles > 65535 || nblk > (1ll << 31) - 1 || nq > (1ll << 31) - 1) return (int)cudaErrorInvalidConfiguration;
    dim3 grid((unsigned)nblk, (unsigned)qtiles);
    search_block_kernel<<<grid, kSearchThreads, smem, s>>>(st, q, qdtype, nq, codes, qjl, norms, rnorms, n, k, bk,
                                                            cand_v, cand_i);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return (int)e;
    search_merge_kernel<<<(unsigned)nq, kSearchThreads, 0, s>>>((int64_t)nblk * k, k, cand_v, cand_i, idx, vals);
    return (int)cudaGetLastError();
}

}  // namespace tq
