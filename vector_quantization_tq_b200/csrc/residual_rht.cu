// Residual pass of TurboQuant_prod with the randomized Hadamard rotation at large d, bf16
// input (the pass before S r on the tensor core).
//
// TurboQuant review (Jump2Paper): Theorem 1 (rotate, per-coordinate Lloyd-Max code) and the
// prod variant's residual r = y - c[idx] with ||r|| kept; Pi = H_d diag(eps) / sqrt(d).
// For d = R * 128 the Hadamard matrix factors as H_R (x) H_128 (Sylvester's H_R for R a power
// of two, Paley's H_12 for R = 12, the order the rest of the library uses): coordinate
// a * 128 + c is row a, column c of an R x 128 array; H_128 acts along the rows and H_R across
// them.
//
// One warp per vector, lane l owning columns 4l .. 4l + 3 of every row, so that:
//   loads and stores of a row are 8 bytes per lane, 256 contiguous bytes per warp;
//   H_128 is two butterfly stages inside the lane and five across lanes (shuffles);
//   H_R is lane-local (all R rows of a column are in the lane's registers);
//   ||x|| and ||r||^2 are warp sums, and the codes of a row are assembled with shuffles.
// Outputs are those of the general encoder's residual pass: codes, ||x||, the residual as
// bf16 rows [hi | lo] (lo = bf16(r - hi)), and ||r||^2 for the signs pass.
#include "common.cuh"

namespace tq {

namespace {

constexpr int kWarpsPerBlock = 8;

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int R, int BM>
__global__ void __launch_bounds__(kWarpsPerBlock * 32, 2)   // two blocks (16 warps) per SM
residual_rht_kernel(const DevState st, const uint16_t* __restrict__ x, int64_t n, int64_t ld,
                    uint8_t* __restrict__ codes, float* __restrict__ norms, uint16_t* __restrict__ r2out,
                    float* __restrict__ rho_out, int rho_stride) {
    constexpr int D = R * 128;
    constexpr int L = 1 << BM;
    constexpr int LPW = 8 / BM;   // lanes whose codes share a 32-bit word
    const int lane = threadIdx.x & 31;
    const int64_t w0 = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
    const int64_t nw = (int64_t)gridDim.x * kWarpsPerBlock;

    // (signs, H_12 rows, levels and boundaries are read from the kernel parameters, which
    // sit in the constant bank: no registers held for them)

    for (int64_t v = w0; v < n; v += nw) {
        float y[R][4];
        float ss = 0.f;
        const uint16_t* xr = x + v * ld + 4 * lane;
#pragma unroll
        for (int a = 0; a < R; ++a) {
            const uint2 w = __ldg(reinterpret_cast<const uint2*>(xr + a * 128));
            const float e[4] = {__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                                __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u)};
            // signs of coordinates a * 128 + 4 lane + k: bits 4 (lane % 8) + k of word 4 a + lane / 8
            const uint32_t sg = st.signs[4 * a + (lane >> 3)] >> (4 * (lane & 7));
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                ss = fmaf(e[k], e[k], ss);
                y[a][k] = ((sg >> k) & 1u) ? -e[k] : e[k];
            }
        }
        // H_128 along each row: column bits 0, 1 inside the lane, bits 2..6 across lanes
#pragma unroll
        for (int a = 0; a < R; ++a) {
            const float u0 = y[a][0] + y[a][1], u1 = y[a][0] - y[a][1];
            const float u2 = y[a][2] + y[a][3], u3 = y[a][2] - y[a][3];
            y[a][0] = u0 + u2;
            y[a][1] = u1 + u3;
            y[a][2] = u0 - u2;
            y[a][3] = u1 - u3;
        }
#pragma unroll
        for (int s = 1; s < 32; s <<= 1) {
            const bool upper = (lane & s) != 0;
#pragma unroll
            for (int a = 0; a < R; ++a) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float o = __shfl_xor_sync(0xffffffffu, y[a][k], s);
                    y[a][k] = upper ? o - y[a][k] : y[a][k] + o;
                }
            }
        }
        // H_R across the rows
        if constexpr (R == 12) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float t[12];
#pragma unroll
                for (int c = 0; c < 12; ++c) t[c] = y[c][k];
#pragma unroll
                for (int a = 0; a < 12; ++a) {
                    float acc = 0.f;
#pragma unroll
                    for (int c = 0; c < 12; ++c) acc += ((st.h12[a] >> c) & 1u) ? -t[c] : t[c];
                    y[a][k] = acc;
                }
            }
        } else {
#pragma unroll
            for (int h = 1; h < R; h <<= 1) {
#pragma unroll
                for (int a = 0; a < R; ++a) {
                    if ((a & h) == 0) {
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float p = y[a][k], q = y[a + h][k];
                            y[a][k] = p + q;
                            y[a + h][k] = p - q;
                        }
                    }
                }
            }
        }
        const float nu = sqrtf(warp_sum_f(ss));
        const float sc = (nu > 0.f) ? st.rsqrt_d / nu : 0.f;
        // quantize, residual (bf16 hi + lo rows), codes
        float rr = 0.f;
        uint32_t* cw = reinterpret_cast<uint32_t*>(codes + v * st.code_bytes);
        uint16_t* rh = r2out + v * 2 * D + 4 * lane;
#pragma unroll
        for (int a = 0; a < R; ++a) {
            uint32_t cb = 0u;
            float r[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float ys = y[a][k] * sc;
                int idx = 0;
#pragma unroll
                for (int i = 0; i < L - 1; ++i) idx += (ys >= st.t[i]) ? 1 : 0;   // #{t_i <= y}
                float cv = st.c[0];
#pragma unroll
                for (int i = 1; i < L; ++i) cv = (idx == i) ? st.c[i] : cv;
                r[k] = (nu > 0.f) ? ys - cv : 0.f;
                rr = fmaf(r[k], r[k], rr);
                cb |= (uint32_t)idx << (BM * k);
            }
            uint32_t hw[2], lw[2];
#pragma unroll
            for (int k = 0; k < 4; k += 2) {
                uint32_t hb[2], lb[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    hb[e] = __bfloat16_as_ushort(__float2bfloat16_rn(r[k + e]));
                    lb[e] = __bfloat16_as_ushort(__float2bfloat16_rn(r[k + e] - __uint_as_float(hb[e] << 16)));
                }
                hw[k / 2] = hb[0] | (hb[1] << 16);
                lw[k / 2] = lb[0] | (lb[1] << 16);
            }
            *reinterpret_cast<uint2*>(rh + a * 128) = make_uint2(hw[0], hw[1]);
            *reinterpret_cast<uint2*>(rh + D + a * 128) = make_uint2(lw[0], lw[1]);
            // the lane's 4 codes sit at bit 4 BM (lane % LPW) of word lane / LPW of the row
            uint32_t word = cb << (4 * BM * (lane % LPW));
#pragma unroll
            for (int s = 1; s < LPW; s <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, s);
            if (lane % LPW == 0) cw[a * 4 * BM + lane / LPW] = word;
        }
        rr = warp_sum_f(rr);
        if (lane == 0) {
            norms[v] = nu;
            rho_out[v * rho_stride] = rr;
            for (int t = 1; t < rho_stride; ++t) rho_out[v * rho_stride + t] = 0.f;
        }
    }
}

template <int R>
int launch_r(const DevState& st, const uint16_t* x, int64_t n, int64_t ld, uint8_t* codes, float* norms,
             uint16_t* r2out, float* rho_out, int rho_stride, cudaStream_t s) {
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t need = (n + kWarpsPerBlock - 1) / kWarpsPerBlock;
    const int64_t cap = (int64_t)sms * 16;
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    switch (st.b_mse) {
        case 1: residual_rht_kernel<R, 1><<<grid, kWarpsPerBlock * 32, 0, s>>>(st, x, n, ld, codes, norms, r2out, rho_out, rho_stride); break;
        case 2: residual_rht_kernel<R, 2><<<grid, kWarpsPerBlock * 32, 0, s>>>(st, x, n, ld, codes, norms, r2out, rho_out, rho_stride); break;
        default: residual_rht_kernel<R, 4><<<grid, kWarpsPerBlock * 32, 0, s>>>(st, x, n, ld, codes, norms, r2out, rho_out, rho_stride); break;
    }
    return (int)cudaGetLastError();
}

}  // namespace

// True for d = 512, 1024, 1536, 2048 with b_mse 1, 2 or 4 (the randomized Hadamard rotation).
bool residual_rht_supported(const DevState& st) {
    const bool dim = st.d == 512 || st.d == 1024 || st.d == 1536 || st.d == 2048;
    return st.rot == TQ_ROT_RHT && dim && (st.b_mse == 1 || st.b_mse == 2 || st.b_mse == 4);
}

int launch_residual_rht(const DevState& st, const void* x, int64_t n, int64_t ld, uint8_t* codes, float* norms,
                        uint16_t* r2out, float* rho_out, int rho_stride, void* stream) {
    cudaStream_t s = (cudaStream_t)stream;
    const uint16_t* xb = reinterpret_cast<const uint16_t*>(x);
    switch (st.d) {
        case 512: return launch_r<4>(st, xb, n, ld, codes, norms, r2out, rho_out, rho_stride, s);
        case 1024: return launch_r<8>(st, xb, n, ld, codes, norms, r2out, rho_out, rho_stride, s);
        case 1536: return launch_r<12>(st, xb, n, ld, codes, norms, r2out, rho_out, rho_stride, s);
        case 2048: return launch_r<16>(st, xb, n, ld, codes, norms, r2out, rho_out, rho_stride, s);
        default: return (int)cudaErrorInvalidValue;
    }
}

}  // namespace tq
