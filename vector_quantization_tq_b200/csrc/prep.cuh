// Query preparation shared by the scoring kernels.
#pragma once

#include "common.cuh"

namespace tq {

// ------------------------------------------------------------------------------------
// Query preparation inside a block: qp = Pi q and u = S qp for `count` queries
// (rows of q with stride d, fp32 or bf16) into shared memory [count][d].
// ------------------------------------------------------------------------------------
__device__ __forceinline__ void prep_queries_dev(const DevState& st, const void* q, int qdtype, int count,
                             float* qs, float* qp, float* u) {
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
        for (int i = threadIdx.x; i < count * d; i += blockDim.x) qp[i] *= st.rsqrt_d;
    } else {
        for (int i = threadIdx.x; i < count * d; i += blockDim.x) {
            const int qi = i / d, j = i % d;
            float a = 0.f;
            for (int k = 0; k < d; ++k) a = fmaf(mat_elem(st.piT, st.mat_dtype, (int64_t)k * d + j), qs[qi * d + k], a);
            qp[i] = a;
        }
    }
    __syncthreads();
    if (st.mode == TQ_PROD) {
        for (int i = threadIdx.x; i < count * d; i += blockDim.x) {
            const int qi = i / d, j = i % d;
            float a = 0.f;
            for (int k = 0; k < d; ++k) a = fmaf(mat_elem(st.sT, st.mat_dtype, (int64_t)k * d + j), qp[qi * d + k], a);
            u[i] = a;
        }
    }
    __syncthreads();
}


}  // namespace tq
