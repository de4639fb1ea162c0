// Chooses the encoder for a state: the tensor-core encoders where one exists for the
// configuration, the tiled CUDA-core encoders for d = 128 and d = 256 with a dense rotation,
// else the general kernel.
#include "common.cuh"

namespace tq {

int launch_encode_generic(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, const int32_t* chan,
                          int64_t ostride, uint8_t* codes, uint8_t* qjl, float* norms, float* rnorms, void* stream);

bool encode_tc_supported(const DevState& st, int dtype, int64_t n, int64_t ld);
int launch_encode_tc(const DevState& st, const void* x, int64_t n, int64_t ld, uint8_t* codes, uint8_t* qjl,
                     float* norms, float* rnorms, void* stream);

bool encode_dense128_supported(const DevState& st, int dtype, int64_t n, int64_t ld);
int launch_encode_dense128(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, uint8_t* codes,
                           uint8_t* qjl, float* norms, float* rnorms, void* stream);

bool encode_dense256_supported(const DevState& st, int dtype, int64_t n, int64_t ld);
int launch_encode_dense256(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, uint8_t* codes,
                           uint8_t* qjl, float* norms, float* rnorms, void* stream);

bool encode_gemm_supported(const DevState& st, int dtype, int64_t n, int64_t ld);
bool encode_rht_gemm_supported(const DevState& st, int dtype, int64_t n, int64_t ld);
int launch_signs_gemm(const DevState& st, int64_t n, uint8_t* qjl, float* rnorms, void* ws, void* stream);
int launch_encode_residual(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, uint8_t* codes,
                           float* norms, uint16_t* r2out, float* rho_out, int rho_stride, void* stream);
size_t encode_gemm_ws_bytes(int d, int64_t n);
int launch_encode_gemm(const DevState& st, const void* x, int64_t n, int64_t ld, uint8_t* codes, uint8_t* qjl,
                       float* norms, float* rnorms, void* ws, void* stream);

// Vectors per pass of the d >= 512 tensor-core encoders (dense Pi, or the Hadamard residual
// pass then the S r GEMM): each vector keeps a bf16 residual pair per coordinate in the
// caller's workspace between the two passes (65536 x 1536 x 4 B = 384 MiB at d = 1536).
constexpr int64_t kGemmChunk = 65536;

namespace {
bool uses_gemm_ws(const DevState& st, int dtype, int64_t n, int64_t ld) {
    return encode_gemm_supported(st, dtype, n, ld) || encode_rht_gemm_supported(st, dtype, n, ld);
}

// Largest pass that fits ws_bytes (a multiple of the 128-vector tile when it is that large).
int64_t chunk_for(const DevState& st, int64_t n, size_t ws_bytes) {
    int64_t c = std::min<int64_t>(n, kGemmChunk);
    while (c > 0 && encode_gemm_ws_bytes(st.d, c) > ws_bytes) c = (c > 128) ? (c - 1) / 128 * 128 : c - 1;
    return c;
}
}  // namespace

size_t encode_ws_bytes(const DevState& st, int dtype, int64_t n, int64_t ld) {
    if (n <= 0 || !uses_gemm_ws(st, dtype, n, ld)) return 0;
    return encode_gemm_ws_bytes(st.d, std::min<int64_t>(n, kGemmChunk));
}

size_t encode_ws_min_bytes(const DevState& st, int dtype, int64_t n, int64_t ld) {
    if (n <= 0 || !uses_gemm_ws(st, dtype, n, ld)) return 0;
    return encode_gemm_ws_bytes(st.d, std::min<int64_t>(n, 128));
}

int launch_encode(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, uint8_t* codes,
                  uint8_t* qjl, float* norms, float* rnorms, void* ws, size_t ws_bytes, void* stream) {
    const bool dense = encode_gemm_supported(st, dtype, n, ld);
    if (dense || encode_rht_gemm_supported(st, dtype, n, ld)) {
        const int64_t chunk = chunk_for(st, n, ws_bytes);
        if (chunk <= 0 || !ws) return (int)cudaErrorInvalidValue;
        int rc = 0;
        for (int64_t c0 = 0; c0 < n && rc == 0; c0 += chunk) {
            const int64_t cn = (n - c0 < chunk) ? n - c0 : chunk;
            const uint16_t* xc = reinterpret_cast<const uint16_t*>(x) + c0 * ld;
            if (dense) {
                rc = launch_encode_gemm(st, xc, cn, ld, codes + c0 * st.code_bytes,
                                        qjl ? qjl + c0 * st.qjl_bytes : nullptr, norms + c0,
                                        rnorms ? rnorms + c0 : nullptr, ws, stream);
            } else {
                uint16_t* r2 = reinterpret_cast<uint16_t*>(ws);
                float* rho = reinterpret_cast<float*>(r2 + (size_t)cn * 2 * st.d);
                rc = launch_encode_residual(st, xc, TQ_BF16, cn, ld, codes + c0 * st.code_bytes, norms + c0, r2, rho,
                                            st.d / 256, stream);
                if (rc == 0) rc = launch_signs_gemm(st, cn, qjl + c0 * st.qjl_bytes, rnorms + c0, ws, stream);
            }
        }
        return rc;
    }
    if (encode_tc_supported(st, dtype, n, ld))
        return launch_encode_tc(st, x, n, ld, codes, qjl, norms, rnorms, stream);
    if (encode_dense128_supported(st, dtype, n, ld))
        return launch_encode_dense128(st, x, dtype, n, ld, codes, qjl, norms, rnorms, stream);
    if (encode_dense256_supported(st, dtype, n, ld))
        return launch_encode_dense256(st, x, dtype, n, ld, codes, qjl, norms, rnorms, stream);
    return launch_encode_generic(st, x, dtype, n, ld, nullptr, 1, codes, qjl, norms, rnorms, stream);
}

// Encode the channels chan[0..d) of each input row (a channel group of a split).
int launch_encode_channels(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, const int32_t* chan,
                           uint8_t* codes, uint8_t* qjl, float* norms, float* rnorms, void* stream) {
    return launch_encode_generic(st, x, dtype, n, ld, chan, 1, codes, qjl, norms, rnorms, stream);
}

// Encode n rows into plane rows 0, ostride, 2 ostride, ... (one new token per head of a
// cache whose heads are ostride rows apart).
int launch_encode_strided(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, int64_t ostride,
                          uint8_t* codes, uint8_t* qjl, float* norms, float* rnorms, void* stream) {
    return launch_encode_generic(st, x, dtype, n, ld, nullptr, ostride, codes, qjl, norms, rnorms, stream);
}

}  // namespace tq
