// Query preparation shared by the scoring kernels: q' = Pi q and u = S q' per query,
// computed by the whole block into shared memory.
#pragma once

#include "common.cuh"

namespace tq {

constexpr int kPrepStageBytes = 16 * 1024;   // shared-memory staging buffer for matrix rows
constexpr int kPrepMaxSlots = 8;             // outputs per thread: count * d <= 8 * blockDim.x

// out[qi][j] = sum_k MT[k][j] * in[qi][k] for qi < count (MT row-major d x d, fp32 or bf16).
// Rows of MT are staged through `stage` in chunks with 16-byte loads, so the global reads
// are coalesced and all in flight at once; the products then come from shared memory.
__device__ __forceinline__ void block_matvec_t(const void* MT, int dtype, int d, const float* in, float* out,
                                               int count, unsigned char* stage) {
    const int es = (dtype == TQ_F32) ? 4 : 2;
    const int kc = kPrepStageBytes / (d * es);   // rows per chunk (d * es divides 16 KiB for d <= 2048)
    const int nout = count * d;
    const unsigned char* src = reinterpret_cast<const unsigned char*>(MT);
    // Outputs in rounds of kPrepMaxSlots * blockDim.x; each round streams the matrix once.
    for (int o0 = 0; o0 < nout; o0 += kPrepMaxSlots * (int)blockDim.x) {
        float acc[kPrepMaxSlots];
#pragma unroll
        for (int s = 0; s < kPrepMaxSlots; ++s) acc[s] = 0.f;
        for (int k0 = 0; k0 < d; k0 += kc) {
            const int rows = (d - k0 < kc) ? d - k0 : kc;
            const int nvec = rows * d * es / 16;
            for (int i = threadIdx.x; i < nvec; i += blockDim.x)
                reinterpret_cast<uint4*>(stage)[i] =
                    __ldg(reinterpret_cast<const uint4*>(src + (size_t)k0 * d * es) + i);
            __syncthreads();
#pragma unroll
            for (int s = 0; s < kPrepMaxSlots; ++s) {
                const int o = o0 + threadIdx.x + s * blockDim.x;
                if (o < nout) {
                    const int qi = o / d, j = o - qi * d;
                    const float* x = in + qi * d + k0;
                    float a = acc[s];
                    if (dtype == TQ_F32) {
                        const float* m = reinterpret_cast<const float*>(stage) + j;
                        for (int kk = 0; kk < rows; ++kk) a = fmaf(m[kk * d], x[kk], a);
                    } else {
                        const uint16_t* m = reinterpret_cast<const uint16_t*>(stage) + j;
                        for (int kk = 0; kk < rows; ++kk) a = fmaf(bf16_bits_to_float(m[kk * d]), x[kk], a);
                    }
                    acc[s] = a;
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int s = 0; s < kPrepMaxSlots; ++s) {
            const int o = o0 + threadIdx.x + s * blockDim.x;
            if (o < nout) out[o] = acc[s];
        }
    }
}

// qp = Pi q and u = S qp for `count` queries (rows of q with stride d, fp32 or bf16) into
// shared memory [count][d], using a kPrepStageBytes staging buffer.
__device__ __forceinline__ void prep_queries_dev(const DevState& st, const void* q, int qdtype, int count,
                                                 float* qs, float* qp, float* u, unsigned char* stage) {
    const int d = st.d;
    for (int i = threadIdx.x; i < count * d; i += blockDim.x)
        qs[i] = (qdtype == TQ_F32) ? __ldg(reinterpret_cast<const float*>(q) + i)
                                   : bf16_bits_to_float(__ldg(reinterpret_cast<const uint16_t*>(q) + i));
    __syncthreads();
    if (st.rot == TQ_ROT_RHT) {
        for (int i = threadIdx.x; i < count * d; i += blockDim.x) {
            const int j = i % d;
            qp[i] = rht_neg(st, j) ? -qs[i] : qs[i];
        }
        __syncthreads();
        if ((d & (d - 1)) == 0) {
            for (int h = 1; h < d; h <<= 1) {
                for (int p = threadIdx.x; p < count * d / 2; p += blockDim.x) {
                    const int qi = p / (d / 2), pr = p % (d / 2);
                    const int j = (pr / h) * 2 * h + (pr % h);
                    float* v = qp + qi * d;
                    const float a = v[j], b = v[j + h];
                    v[j] = a + b;
                    v[j + h] = a - b;
                }
                __syncthreads();
            }
        } else {   // d = 12 * 2^k
            for (int qi = 0; qi < count; ++qi)
                kron_hadamard(qp + qi * d, d, st.h12, false, threadIdx.x, blockDim.x, [] { __syncthreads(); });
        }
        for (int i = threadIdx.x; i < count * d; i += blockDim.x) qp[i] *= st.rsqrt_d;
    } else {
        block_matvec_t(st.piT, st.mat_dtype, d, qs, qp, count, stage);
    }
    __syncthreads();
    if (st.mode == TQ_PROD) block_matvec_t(st.sT, st.mat_dtype, d, qp, u, count, stage);
    __syncthreads();
}

}  // namespace tq
