// Fused decode attention over a compressed KV cache, d = 128 (one query per head).
//
// Per head h: s_t = scale * <q_h, k~_t>, p = softmax(s), out_h = sum_t p_t v~_t, with
// v~_t = ||v_t|| Pi_V^T c_V[idx_t]. The standard attention form is the PolarQuant review's
// (attention over a quantized cache); the score is TurboQuant's inner-product estimate
// (Jump2Paper review, Theorem 2): <q, k~> = ||k|| (sum_j q'_j c[idx_j] + ||r|| sqrt(pi/2)/d
// sum_j u_j (2 z_j - 1)), q' = Pi_K q, u = S q'.
//
// A table launch first builds, once per head, the lookup tables of q' = Pi_K q against the
// key code groups and of u = S q' against the QJL nibbles (the scorer's tables).
// Flash-decoding split over tokens: block (split, h) copies its head's tables, walks tiles
// of 256 tokens (staged with cp.async, double-buffered) with an online softmax and writes
// (m, l, acc[d]) for the combine launch, which merges the splits and applies Pi_V^T once
// per head. Inside a tile:
//   A. one thread per token scores it through per-query tables over packed code groups
//      (16- or 64-entry tables in shared memory, as in the LUT scorer);
//   B. the block updates the running max and sum and forms w_t = p_t ||v_t||;
//   C. one warp per token accumulates w_t c_V[idx_tj] into the rotated-domain value sum,
//      each lane owning 4 coordinates (a 2-byte slice of the token's 4-bit code row).
// Only the compressed bytes are read: 72 B (keys, prod b=4) + 68 B (values, mse b=4) per
// token and head.
#include "common.cuh"

namespace tq {

int attend_heads_per_block(int G);

namespace {

constexpr int kD = 128;
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <int B>
struct KGroups {
    static constexpr int G = (B == 3) ? 6 : 4;   // bits per table index (as in the scorer's tables)
    static constexpr int E = 1 << G;
    static constexpr int NG = kD * B / G;
};

// Asynchronous global -> shared copies (16 bytes, L2 only; 4 bytes through L1).
__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(void* dst, const void* src) {
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait0() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// One tile of a head's compressed cache in shared memory.
template <int BK, bool KPROD, int BV>
struct TileBuf {
    static constexpr int KROW = kD * BK / 8;   // bytes of key codes per token
    static constexpr int VROW = kD * BV / 8;   // bytes of value codes per token
    uint8_t kc[kThreads * KROW];
    uint8_t kz[KPROD ? kThreads * 16 : 16];
    uint8_t vc[kThreads * VROW];
    float kn[kThreads];
    float kr[kThreads];
    float vn[kThreads];
};

// QH query heads of one KV group per block (GQA): the tile of the group's compressed cache is
// staged once, every token is scored against the QH heads' tables, and the value codes of a
// token are decoded once for all QH weighted sums.
template <int BK, bool KPROD, int BV, int QH>
__global__ void __launch_bounds__(kThreads)
attend_lut_kernel(const DevState ks, const DevState vs, const float* __restrict__ luts, int64_t T, int G, int64_t Tcap,
                  int64_t chunk, const uint8_t* __restrict__ kcodes, const uint8_t* __restrict__ kqjl,
                  const float* __restrict__ knorms, const float* __restrict__ krnorms,
                  const uint8_t* __restrict__ vcodes, const float* __restrict__ vnorms, float scale,
                  float* __restrict__ part) {
    using KG = KGroups<BK>;
    using TB = TileBuf<BK, KPROD, BV>;
    constexpr int NQ = kD / 4;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    constexpr int LSIZE = KG::NG * KG::E + (KPROD ? NQ * 16 : 0);   // floats of one query's tables
    // Four query heads per block: one tile buffer, and the warps' value sums laid over it at
    // the end, so that two blocks fit on an SM (16 warps to hide the table lookups' latency);
    // otherwise two tile buffers, the next tile staged while this one is processed.
    constexpr int kBufs = (QH == 4) ? 1 : 2;
    TB* tb = reinterpret_cast<TB*>(smem_raw);
    float* vc = reinterpret_cast<float*>(tb + kBufs);           // 32 (V centroids)
    float* tm = vc + 32;                                         // QH x LSIZE: head qh's tables at qh * LSIZE
    float* wt = tm + QH * LSIZE;                                 // QH x kThreads
    float* red = wt + QH * kThreads;                             // QH x 32
    float* accw = (kBufs == 1) ? reinterpret_cast<float*>(tb) : red + QH * 32;   // kWarps x QH x kD

    const int h0 = blockIdx.y * QH;   // the block's first query head
    const int split = blockIdx.x;
    const int nsplit = gridDim.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t t_begin = (int64_t)split * chunk;
    const int64_t t_end = (T < t_begin + chunk) ? T : t_begin + chunk;
    const int64_t hT = (int64_t)(h0 / G) * Tcap;   // planes of the heads' KV head

    // Stage a tile (tokens t0 .. t0+255 of this KV head) into buffer `sb`; rows past the end
    // of this split are not copied and not read.
    auto stage_tile = [&](int sb, int64_t t0) {
        TB& B = tb[sb];
        const int cnt = (int)((t_end - t0) < kThreads ? (t_end - t0) : kThreads);
        const uint8_t* kc = kcodes + (hT + t0) * TB::KROW;
        for (int i = threadIdx.x; i < cnt * (TB::KROW / 16); i += kThreads) cp_async16(B.kc + i * 16, kc + i * 16);
        const uint8_t* vcp = vcodes + (hT + t0) * TB::VROW;
        for (int i = threadIdx.x; i < cnt * (TB::VROW / 16); i += kThreads) cp_async16(B.vc + i * 16, vcp + i * 16);
        if ((int)threadIdx.x < cnt) {
            const int64_t g = hT + t0 + threadIdx.x;
            if constexpr (KPROD) {
                cp_async16(B.kz + threadIdx.x * 16, kqjl + g * 16);
                cp_async4(B.kr + threadIdx.x, krnorms + g);
            }
            cp_async4(B.kn + threadIdx.x, knorms + g);
            cp_async4(B.vn + threadIdx.x, vnorms + g);
        }
    };

    // the heads' tables (q' against the K code groups, u against the QJL nibbles), built once
    // per head by the table launch and consecutive in `luts`, arrive with the first tile
    for (int i = threadIdx.x; i < QH * LSIZE / 4; i += kThreads)
        cp_async16(tm + 4 * i, luts + (int64_t)h0 * LSIZE + 4 * i);
    if (kBufs == 2 && t_begin < t_end) stage_tile(0, t_begin);
    cp_async_commit();
    if (threadIdx.x < 32) vc[threadIdx.x] = (threadIdx.x < vs.L) ? vs.c[threadIdx.x] : 0.f;

    // per head: this warp's value sums, coordinates 4 lane .. +3 (8 (lane % 16) .. +7 for 4-bit
    // values, the two half-warps taking different tokens)
    constexpr int VC = (BV == 4) ? 8 : 4;
    float acc[QH][VC];
    float m_run[QH], l_run[QH];
#pragma unroll
    for (int q = 0; q < QH; ++q) {
        m_run[q] = -INFINITY;
        l_run[q] = 0.f;
#pragma unroll
        for (int c = 0; c < VC; ++c) acc[q][c] = 0.f;
    }
    int it = 0;
    for (int64_t t0 = t_begin; t0 < t_end; t0 += kThreads, ++it) {
        const int cnt = (int)((t_end - t0) < kThreads ? (t_end - t0) : kThreads);
        const int sb = (kBufs == 2) ? (it & 1) : 0;
        if constexpr (kBufs == 2) {
            if (t0 + kThreads < t_end) stage_tile(sb ^ 1, t0 + kThreads);   // prefetch the next tile
            cp_async_commit();
            cp_async_wait1();
        } else {
            stage_tile(0, t0);
            cp_async_commit();
            cp_async_wait0();
        }
        __syncthreads();
        const TB& B = tb[sb];
        // ---- A: scores of token t0 + threadIdx.x against the QH heads ----
        float s[QH];
#pragma unroll
        for (int q = 0; q < QH; ++q) s[q] = -INFINITY;
        if ((int)threadIdx.x < cnt) {
            constexpr int CW = kD * BK / 32;
            uint32_t w[CW];
            const uint4* src = reinterpret_cast<const uint4*>(B.kc + threadIdx.x * TB::KROW);
#pragma unroll
            for (int i = 0; i < CW / 4; ++i) {
                const uint4 v = src[i];
                w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
            }
            // table lookups into paired accumulators (two independent chains, f32x2 adds)
            float2 p1[QH];
#pragma unroll
            for (int q = 0; q < QH; ++q) p1[q] = make_float2(0.f, 0.f);
            if constexpr (KG::G == 4) {
#pragma unroll
                for (int wi = 0; wi < CW; ++wi) add_nibbles<QH, LSIZE>(w[wi], tm + 8 * wi * 16, p1);
            } else {
                static_assert(KG::NG % 2 == 0, "groups in pairs");
#pragma unroll
                for (int k = 0; k < KG::NG; ++k) {
                    const int bit = k * KG::G;
                    const int wi = bit >> 5, sh = bit & 31;
                    uint32_t e;
                    if (sh + KG::G <= 32) e = (w[wi] >> sh) & (KG::E - 1);
                    else e = ((w[wi] >> sh) | (w[wi + 1] << (32 - sh))) & (KG::E - 1);
#pragma unroll
                    for (int q = 0; q < QH; ++q) {
                        if (k & 1) p1[q].y += tm[q * LSIZE + k * KG::E + e];
                        else p1[q].x += tm[q * LSIZE + k * KG::E + e];
                    }
                }
            }
            float2 p2[QH];
#pragma unroll
            for (int q = 0; q < QH; ++q) p2[q] = make_float2(0.f, 0.f);
            float g2 = 0.f;
            if constexpr (KPROD) {
                const uint4 zv = *reinterpret_cast<const uint4*>(B.kz + threadIdx.x * 16);
                const uint32_t z[4] = {zv.x, zv.y, zv.z, zv.w};
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) add_nibbles<QH, LSIZE>(z[wi], tm + KG::NG * KG::E + 8 * wi * 16, p2);
                g2 = B.kr[threadIdx.x] * ks.qjl_scale;
            }
            const float kn = scale * B.kn[threadIdx.x];
#pragma unroll
            for (int q = 0; q < QH; ++q) s[q] = kn * fmaf(g2, p2[q].x + p2[q].y, p1[q].x + p1[q].y);
        }
        // ---- B: online softmax bookkeeping, per head ----
#pragma unroll
        for (int q = 0; q < QH; ++q) {
            const float wm = warp_max(s[q]);
            if (lane == 0) red[q * 32 + warp] = wm;
        }
        __syncthreads();
        float alpha[QH], p[QH];
#pragma unroll
        for (int q = 0; q < QH; ++q) {
            float tmax = red[q * 32];
#pragma unroll
            for (int i = 1; i < kWarps; ++i) tmax = fmaxf(tmax, red[q * 32 + i]);
            const float m_new = fmaxf(m_run[q], tmax);
            alpha[q] = (m_run[q] == -INFINITY) ? 0.f : __expf(m_run[q] - m_new);
            p[q] = ((int)threadIdx.x < cnt) ? __expf(s[q] - m_new) : 0.f;
            m_run[q] = m_new;
        }
        __syncthreads();   // everyone has read red[] (max) before it is reused
        const float vnt = ((int)threadIdx.x < cnt) ? B.vn[threadIdx.x] : 0.f;
#pragma unroll
        for (int q = 0; q < QH; ++q) {
            const float ps = warp_sum(p[q]);
            if (lane == 0) red[q * 32 + warp] = ps;
            wt[q * kThreads + threadIdx.x] = p[q] * vnt;
        }
        __syncthreads();
#pragma unroll
        for (int q = 0; q < QH; ++q) {
            float tsum = 0.f;
#pragma unroll
            for (int i = 0; i < kWarps; ++i) tsum += red[q * 32 + i];
            l_run[q] = l_run[q] * alpha[q] + tsum;
#pragma unroll
            for (int c = 0; c < VC; ++c) acc[q][c] *= alpha[q];
        }
        if constexpr (BV == 4) {
            // ---- C: value sums, two tokens per warp step (at step i half-warp h takes token
            // 16 i + 2 warp + h, so the two rows lie in different banks), 8 coordinates per lane: a 4-byte slice of the token's code row,
            // one lookup per coordinate in the 16-entry table (one entry per bank: no conflicts)
            // and paired FMAs ----
            const int hsel = lane >> 4, hl = lane & 15;
            const char* cbase = reinterpret_cast<const char*>(vc);
#pragma unroll
            for (int i0 = 0; i0 < kThreads / kWarps / 2; i0 += 8) {
                uint32_t bits[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int t = 16 * (i0 + j) + 2 * warp + hsel;
                    bits[j] = (t < cnt) ? reinterpret_cast<const uint32_t*>(B.vc + t * TB::VROW)[hl] : 0u;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int tt = 16 * (i0 + j) + 2 * warp + hsel;
                    const bool live = tt < cnt;
                    const int t = live ? tt : 0;   // weights of absent tokens are 0
                    // byte offsets 4 e of the eight nibbles: even coordinates in `lo`, odd in `hi`
                    const uint32_t lo = (bits[j] << 2) & 0x3C3C3C3Cu, hi = (bits[j] >> 2) & 0x3C3C3C3Cu;
                    float2 cv[4];
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        cv[c] = make_float2(*reinterpret_cast<const float*>(cbase + __byte_perm(lo, 0u, 0x4440u | c)),
                                            *reinterpret_cast<const float*>(cbase + __byte_perm(hi, 0u, 0x4440u | c)));
#pragma unroll
                    for (int q = 0; q < QH; ++q) {
                        const float wv = live ? wt[q * kThreads + t] : 0.f;
                        const float2 w2 = make_float2(wv, wv);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const float2 a = __ffma2_rn(w2, cv[c], make_float2(acc[q][2 * c], acc[q][2 * c + 1]));
                            acc[q][2 * c] = a.x;
                            acc[q][2 * c + 1] = a.y;
                        }
                    }
                }
            }
        } else {
            // ---- C: value sums, one warp per token, 4 coordinates per lane; 32 tokens per warp ----
            const int ntok = (cnt - warp + kWarps - 1) / kWarps;   // tokens t = warp + 8 * i < cnt
            // batches of 8 tokens: the 8 code slices are loaded before their FMAs
#pragma unroll
            for (int i0 = 0; i0 < kThreads / kWarps; i0 += 8) {
                uint32_t bits[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int i = i0 + j;
                    const int t = warp + i * kWarps;
                    uint32_t b = 0;
                    if (i < ntok) {
                        const uint8_t* row = B.vc + t * TB::VROW;
                        if constexpr (BV == 2) {
                            b = row[lane];
                        } else {
                            const int b0 = lane * 4 * BV;
                            const int wi = b0 >> 5, sh = b0 & 31;
                            const uint32_t* r32 = reinterpret_cast<const uint32_t*>(row);
                            uint64_t win = r32[wi];
                            if ((sh + 4 * BV > 32) && (wi + 1) * 32 < kD * BV) win |= (uint64_t)r32[wi + 1] << 32;
                            b = (uint32_t)(win >> sh);
                        }
                    }
                    bits[j] = b;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int i = i0 + j;
                    const int t = (i < ntok) ? warp + i * kWarps : 0;   // weights of absent tokens are 0
                    float cv[4];
                    if constexpr (BV == 2) {
                        const char* cbase = reinterpret_cast<const char*>(vc);
                        const uint32_t b8 = bits[j];
                        cv[0] = *reinterpret_cast<const float*>(cbase + ((b8 << 2) & 0xCu));
                        cv[1] = *reinterpret_cast<const float*>(cbase + (b8 & 0xCu));
                        cv[2] = *reinterpret_cast<const float*>(cbase + ((b8 >> 2) & 0xCu));
                        cv[3] = *reinterpret_cast<const float*>(cbase + ((b8 >> 4) & 0xCu));
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c) cv[c] = vc[(bits[j] >> (BV * c)) & ((1u << BV) - 1u)];
                    }
#pragma unroll
                    for (int q = 0; q < QH; ++q) {
                        const float wv = (i < ntok) ? wt[q * kThreads + t] : 0.f;
#pragma unroll
                        for (int c = 0; c < 4; ++c) acc[q][c] = fmaf(wv, cv[c], acc[q][c]);
                    }
                }
            }
        }
        __syncthreads();   // wt / red and the tile buffer are reused
    }
    cp_async_wait0();
    // ---- reduce the warps' value sums and write the split records ----
    if constexpr (BV == 4) {
        // the two half-warps hold the same coordinates for different tokens
#pragma unroll
        for (int q = 0; q < QH; ++q)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[q][c] += __shfl_xor_sync(0xffffffffu, acc[q][c], 16);
        if (lane < 16) {
#pragma unroll
            for (int q = 0; q < QH; ++q)
#pragma unroll
                for (int c = 0; c < 8; c += 4)
                    *reinterpret_cast<float4*>(&accw[(warp * QH + q) * kD + 8 * lane + c]) =
                        make_float4(acc[q][c], acc[q][c + 1], acc[q][c + 2], acc[q][c + 3]);
        }
    } else {
#pragma unroll
        for (int q = 0; q < QH; ++q)
#pragma unroll
            for (int c = 0; c < 4; ++c) accw[(warp * QH + q) * kD + 4 * lane + c] = acc[q][c];
    }
    __syncthreads();
    for (int j = threadIdx.x; j < QH * kD; j += kThreads) {
        const int q = j / kD, jj = j % kD;
        float a = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < kWarps; ++w2) a += accw[(w2 * QH + q) * kD + jj];
        part[((int64_t)(h0 + q) * nsplit + split) * (kD + 2) + 2 + jj] = a;
    }
#pragma unroll
    for (int q = 0; q < QH; ++q) {
        if ((int)threadIdx.x == q) {
            float* rec = part + ((int64_t)(h0 + q) * nsplit + split) * (kD + 2);
            rec[0] = m_run[q];
            rec[1] = l_run[q];
        }
    }
}

template <int BK, bool KPROD, int BV, int QH>
size_t smem_bytes() {
    using KG = KGroups<BK>;
    constexpr int kBufs = (QH == 4) ? 1 : 2;   // as in the kernel
    static_assert(kBufs == 2 || sizeof(TileBuf<BK, KPROD, BV>) >= sizeof(float) * kWarps * QH * kD,
                  "the value sums fit over the tile buffer");
    return kBufs * sizeof(TileBuf<BK, KPROD, BV>) +
           (size_t)(32 + QH * (KG::NG * KG::E + (KPROD ? (kD / 4) * 16 : 0)) + QH * kThreads + QH * 32 +
                    (kBufs == 2 ? kWarps * QH * kD : 0)) *
               sizeof(float);
}

template <int BK, bool KPROD, int BV, int QH>
int launch_q(const DevState& ks, const DevState& vs, const float* luts, int H, int64_t T, int G, int64_t Tcap,
             int nsplit, int64_t chunk, const uint8_t* kcodes, const uint8_t* kqjl, const float* knorms,
             const float* krnorms, const uint8_t* vcodes, const float* vnorms, float scale, float* part,
             cudaStream_t s) {
    auto kern = attend_lut_kernel<BK, KPROD, BV, QH>;
    const size_t smem = smem_bytes<BK, KPROD, BV, QH>();
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return (int)e;
    }
    dim3 grid((unsigned)nsplit, (unsigned)(H / QH));
    kern<<<grid, kThreads, smem, s>>>(ks, vs, luts, T, G, Tcap, chunk, kcodes, kqjl, knorms, krnorms, vcodes, vnorms, scale,
                                      part);
    return (int)cudaGetLastError();
}

// Query heads per block: 4 (or 2) when every group of G query heads splits evenly.
template <int BK, bool KPROD, int BV>
int launch_t(const DevState& ks, const DevState& vs, const float* luts, int H, int64_t T, int G, int64_t Tcap, int nsplit,
             int64_t chunk, const uint8_t* kcodes, const uint8_t* kqjl, const float* knorms, const float* krnorms,
             const uint8_t* vcodes, const float* vnorms, float scale, float* part, cudaStream_t s) {
    const int qh = attend_heads_per_block(G);
    if (qh == 4)
        return launch_q<BK, KPROD, BV, 4>(ks, vs, luts, H, T, G, Tcap, nsplit, chunk, kcodes, kqjl, knorms, krnorms,
                                          vcodes, vnorms, scale, part, s);
    if (qh == 2)
        return launch_q<BK, KPROD, BV, 2>(ks, vs, luts, H, T, G, Tcap, nsplit, chunk, kcodes, kqjl, knorms, krnorms,
                                          vcodes, vnorms, scale, part, s);
    return launch_q<BK, KPROD, BV, 1>(ks, vs, luts, H, T, G, Tcap, nsplit, chunk, kcodes, kqjl, knorms, krnorms,
                                      vcodes, vnorms, scale, part, s);
}

template <int BK, bool KPROD>
int launch_v(const DevState& ks, const DevState& vs, const float* luts, int H, int64_t T, int G, int64_t Tcap, int nsplit,
             int64_t chunk, const uint8_t* kcodes, const uint8_t* kqjl, const float* knorms, const float* krnorms,
             const uint8_t* vcodes, const float* vnorms, float scale, float* part, cudaStream_t s) {
    switch (vs.b_mse) {
        case 2: return launch_t<BK, KPROD, 2>(ks, vs, luts, H, T, G, Tcap, nsplit, chunk, kcodes, kqjl, knorms, krnorms,
                                              vcodes, vnorms, scale, part, s);
        case 3: return launch_t<BK, KPROD, 3>(ks, vs, luts, H, T, G, Tcap, nsplit, chunk, kcodes, kqjl, knorms, krnorms,
                                              vcodes, vnorms, scale, part, s);
        case 4: return launch_t<BK, KPROD, 4>(ks, vs, luts, H, T, G, Tcap, nsplit, chunk, kcodes, kqjl, knorms, krnorms,
                                              vcodes, vnorms, scale, part, s);
        default: return (int)cudaErrorInvalidValue;
    }
}

template <bool KPROD>
int launch_k(const DevState& ks, const DevState& vs, const float* luts, int H, int64_t T, int G, int64_t Tcap, int nsplit,
             int64_t chunk, const uint8_t* kcodes, const uint8_t* kqjl, const float* knorms, const float* krnorms,
             const uint8_t* vcodes, const float* vnorms, float scale, float* part, cudaStream_t s) {
    switch (ks.b_mse) {
        case 2: return launch_v<2, KPROD>(ks, vs, luts, H, T, G, Tcap, nsplit, chunk, kcodes, kqjl, knorms, krnorms,
                                          vcodes, vnorms, scale, part, s);
        case 3: return launch_v<3, KPROD>(ks, vs, luts, H, T, G, Tcap, nsplit, chunk, kcodes, kqjl, knorms, krnorms,
                                          vcodes, vnorms, scale, part, s);
        case 4: return launch_v<4, KPROD>(ks, vs, luts, H, T, G, Tcap, nsplit, chunk, kcodes, kqjl, knorms, krnorms,
                                          vcodes, vnorms, scale, part, s);
        default: return (int)cudaErrorInvalidValue;
    }
}

}  // namespace

bool attend_lut_supported(const DevState& ks, const DevState& vs, const void* kcodes, const void* kqjl,
                          const void* vcodes) {
    const auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    return a16(kcodes) && a16(vcodes) && (kqjl == nullptr || a16(kqjl)) && ks.d == kD && vs.d == kD && ks.b_mse >= 2 && ks.b_mse <= 4 && vs.b_mse >= 2 && vs.b_mse <= 4;
}

int launch_attend_lut_split(const DevState& ks, const DevState& vs, const float* luts, int H, int64_t T, int G,
                            int64_t Tcap, int nsplit, int64_t chunk, const uint8_t* kcodes, const uint8_t* kqjl,
                            const float* knorms, const float* krnorms, const uint8_t* vcodes, const float* vnorms,
                            float scale, float* part, void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    if (kqjl) return launch_k<true>(ks, vs, luts, H, T, G, Tcap, nsplit, chunk, kcodes, kqjl, knorms, krnorms, vcodes,
                                    vnorms, scale, part, s);
    return launch_k<false>(ks, vs, luts, H, T, G, Tcap, nsplit, chunk, kcodes, kqjl, knorms, krnorms, vcodes, vnorms,
                           scale, part, s);
}

}  // namespace tq
