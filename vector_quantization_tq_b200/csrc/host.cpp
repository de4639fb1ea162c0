// C ABI of libtq: argument validation, state management, dispatch to the kernels.
// The operations are defined in include/tq.h (with the passages they follow).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <vector>

#include "internal.h"

namespace tq {

static thread_local int g_last_cuda_error = 0;

void set_cuda_error(int err) { g_last_cuda_error = err; }

namespace {

// Restores the caller's current device on scope exit.
struct DeviceGuard {
    int prev = -1;
    bool ok = false;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) return;
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) return;
        ok = true;
    }
    ~DeviceGuard() {
        int cur;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

bool kernel_dim_supported(int d) {
    switch (d) {
        case 32: case 64: case 96: case 128: case 160: case 192: case 224: case 256:
        case 512: case 1024: case 1536: case 2048:
            return true;
        default:
            return false;
    }
}

bool is_pow2(int d) { return d > 0 && (d & (d - 1)) == 0; }

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return TQ_OK;
    set_cuda_error((int)e);
    (void)cudaGetLastError();   // clear a non-sticky error
    return (e == cudaErrorMemoryAllocation) ? TQ_ENOMEM : TQ_ECUDA;
}

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

int check_vectors(const tq_state* st, const void* x, int dtype, int64_t n, int64_t ld) {
    if (dtype != TQ_F32 && dtype != TQ_BF16) return TQ_EINVAL;
    if (n < 0) return TQ_EINVAL;
    if (n == 0) return TQ_OK;
    if (!x || ld < st->p.d) return TQ_EINVAL;
    const int64_t es = (dtype == TQ_F32) ? 4 : 2;
    if (!aligned16(x) || ((ld * es) & 15)) return TQ_EINVAL;
    return TQ_OK;
}

uint16_t to_bf16_bits(float v) {
    float r = bf16_round_host(v);
    uint32_t u;
    std::memcpy(&u, &r, 4);
    return (uint16_t)(u >> 16);
}

// Upload Pi, Pi^T, S, S^T at the stored dtype and fill the kernel view.
int finish_state(tq_state* st) {
    const tq_params& p = st->p;
    const int d = p.d;
    tq::DevState& ds = st->dev;
    std::memset(&ds, 0, sizeof(ds));
    ds.d = d;
    ds.b_mse = st->b_mse;
    ds.L = 1 << st->b_mse;
    ds.mode = p.mode;
    ds.rot = p.rot;
    ds.mat_dtype = p.mat_dtype;
    ds.code_bytes = (st->b_mse * d + 7) / 8;
    ds.qjl_bytes = (p.mode == TQ_PROD) ? d / 8 : 0;
    ds.qjl_scale = (float)(std::sqrt(M_PI / 2.0) / d);
    ds.rsqrt_d = (float)(1.0 / std::sqrt((double)d));
    for (int i = 0; i < ds.L; ++i) ds.c[i] = (float)st->centroids[i];
    for (int i = 0; i + 1 < ds.L; ++i) ds.t[i] = (float)st->bounds[i];
    if (p.rot == TQ_ROT_RHT) {
        for (int j = 0; j < d; ++j)
            if (st->signs[j] < 0) ds.signs[j / 32] |= 1u << (j % 32);
        if (!is_pow2(d)) paley_hadamard12_rows(ds.h12);   // d = 12 * 2^k: H_12 (x) Sylvester
    }

    const size_t es = (p.mat_dtype == TQ_F32) ? 4 : 2;
    const size_t mat = (size_t)d * d * es;
    const bool dense = (p.rot == TQ_ROT_DENSE);
    const bool prod = (p.mode == TQ_PROD);
    const size_t nmat = (dense ? 2 : 0) + (prod ? 2 : 0);
    if (nmat == 0) return TQ_OK;

    std::vector<unsigned char> host(nmat * mat);
    auto put = [&](size_t slot, const std::vector<double>& m, bool transpose) {
        unsigned char* dst = host.data() + slot * mat;
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) {
                double v = transpose ? m[(size_t)j * d + i] : m[(size_t)i * d + j];
                size_t o = (size_t)i * d + j;
                if (p.mat_dtype == TQ_F32) {
                    float f = (float)v;
                    std::memcpy(dst + o * 4, &f, 4);
                } else {
                    uint16_t h = to_bf16_bits((float)v);
                    std::memcpy(dst + o * 2, &h, 2);
                }
            }
    };
    size_t slot = 0;
    size_t pi_slot = 0, s_slot = 0;
    if (dense) {
        pi_slot = slot;
        put(slot++, st->pi, false);
        put(slot++, st->pi, true);
    }
    if (prod) {
        s_slot = slot;
        put(slot++, st->s, false);
        put(slot++, st->s, true);
    }
    DeviceGuard g(p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    cudaError_t e = cudaMalloc(&st->d_mem, host.size());
    if (e != cudaSuccess) {
        st->d_mem = nullptr;
        return cuda_status(e);
    }
    e = cudaMemcpy(st->d_mem, host.data(), host.size(), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_status(e);
    unsigned char* base = (unsigned char*)st->d_mem;
    if (dense) {
        ds.pi = base + pi_slot * mat;
        ds.piT = base + (pi_slot + 1) * mat;
    }
    if (prod) {
        ds.s = base + s_slot * mat;
        ds.sT = base + (s_slot + 1) * mat;
    }
    return TQ_OK;
}

double stored_value(double v, int dtype) {
    return (dtype == TQ_F32) ? (double)(float)v : (double)bf16_round_host((float)v);
}

int validate_params(const tq_params* p) {
    if (!p) return TQ_EINVAL;
    if (p->mode != TQ_MSE && p->mode != TQ_PROD) return TQ_EINVAL;
    if (p->rot != TQ_ROT_DENSE && p->rot != TQ_ROT_RHT) return TQ_EINVAL;
    if (p->mat_dtype != TQ_F32 && p->mat_dtype != TQ_BF16) return TQ_EINVAL;
    if (p->d < 2 || p->d > kMaxDim) return p->d < 2 ? TQ_EINVAL : TQ_EUNSUPPORTED;
    if (p->mode == TQ_MSE && (p->b < 1 || p->b > 8)) return TQ_EINVAL;
    if (p->mode == TQ_PROD && (p->b < 1 || p->b > 9)) return TQ_EINVAL;
    if (p->device < 0) return TQ_EINVAL;
    // Hadamard orders: 2^k (Sylvester), or 12 * 2^k (Paley's order 12 Kronecker Sylvester)
    if (p->rot == TQ_ROT_RHT && !is_pow2(p->d) && !(p->d % 12 == 0 && is_pow2(p->d / 12)))
        return TQ_EUNSUPPORTED;
    if (!kernel_dim_supported(p->d)) return TQ_EUNSUPPORTED;
    return TQ_OK;
}

}  // namespace
}  // namespace tq

using namespace tq;

extern "C" {

const char* tq_status_string(int status) {
    switch (status) {
        case TQ_OK: return "ok";
        case TQ_EINVAL: return "invalid argument";
        case TQ_EUNSUPPORTED: return "unsupported configuration";
        case TQ_ENOMEM: return "out of memory or workspace too small";
        case TQ_ECUDA: return "CUDA runtime error";
        case TQ_EDEVICE: return "device-side error";
        default: return "unknown status";
    }
}

int tq_last_cuda_error(void) { return g_last_cuda_error; }

int tq_version(void) { return 100; }

int tq_device_status(int device) {
    if (device < 0) return TQ_EINVAL;
    DeviceGuard g(device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_status(e);
    int flag = 0;
    int rc = read_device_error(&flag);
    if (rc != 0) return cuda_status((cudaError_t)rc);
    return flag ? TQ_EDEVICE : TQ_OK;
}

int tq_check_error_path(int device, uint32_t limit_us) {
    if (device < 0 || limit_us == 0 || limit_us > 1000000) return TQ_EINVAL;
    DeviceGuard g(device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    return cuda_status((cudaError_t)launch_expired_wait((uint64_t)limit_us * 1000ull, nullptr));
}

int tq_build_codebook(int d, int b, double* h_c, double* h_t, double* h_dmse) {
    if (d < 2 || b < 1 || b > 8) return TQ_EINVAL;
    return build_codebook(d, b, h_c, h_t, h_dmse);
}

int tq_draw_gaussian(uint64_t seed, size_t count, double* h_out) {
    if (!h_out && count) return TQ_EINVAL;
    philox_gaussian(seed, count, h_out);
    return TQ_OK;
}

int tq_draw_signs(uint64_t seed, size_t count, int8_t* h_out) {
    if (!h_out && count) return TQ_EINVAL;
    philox_signs(seed, count, h_out);
    return TQ_OK;
}

int tq_haar_rotation(int d, const double* h_g, double* h_pi) {
    if (d < 2 || !h_g || !h_pi) return TQ_EINVAL;
    return haar_from_gaussian(d, h_g, h_pi);
}

int tq_state_create(const tq_params* p, const double* h_gauss_pi, const int8_t* h_signs,
                    const double* h_s, tq_state** out) {
    if (!out) return TQ_EINVAL;
    *out = nullptr;
    int rc = validate_params(p);
    if (rc != TQ_OK) return rc;
    tq_state* st = new (std::nothrow) tq_state();
    if (!st) return TQ_ENOMEM;
    st->p = *p;
    const int d = p->d;
    st->b_mse = (p->mode == TQ_MSE) ? p->b : p->b - 1;
    const int L = 1 << st->b_mse;
    st->centroids.assign(L, 0.0);
    st->bounds.assign(L > 1 ? L - 1 : 0, 0.0);
    if (st->b_mse > 0) {
        rc = build_codebook(d, st->b_mse, st->centroids.data(), st->bounds.data(), &st->dmse);
    } else {
        st->dmse = 1.0;   // 0-bit MSE: x~_mse = 0, D = E||y||^2 = 1
    }
    if (rc != TQ_OK) {
        delete st;
        return rc;
    }
    if (p->rot == TQ_ROT_DENSE) {
        std::vector<double> g;
        const double* gp = h_gauss_pi;
        if (!gp) {
            g.resize((size_t)d * d);
            philox_gaussian(p->seed_pi, g.size(), g.data());
            gp = g.data();
        }
        st->pi.resize((size_t)d * d);
        rc = haar_from_gaussian(d, gp, st->pi.data());
        if (rc != TQ_OK) {
            delete st;
            return rc;
        }
        for (double& v : st->pi) v = stored_value(v, p->mat_dtype);
    } else {
        st->signs.resize(d);
        if (h_signs) {
            for (int j = 0; j < d; ++j) {
                if (h_signs[j] != 1 && h_signs[j] != -1) {
                    delete st;
                    return TQ_EINVAL;
                }
                st->signs[j] = h_signs[j];
            }
        } else {
            philox_signs(p->seed_pi, d, st->signs.data());
        }
    }
    if (p->mode == TQ_PROD) {
        st->s.resize((size_t)d * d);
        if (h_s) {
            for (size_t i = 0; i < st->s.size(); ++i) {
                if (!std::isfinite(h_s[i])) {
                    delete st;
                    return TQ_EINVAL;
                }
                st->s[i] = h_s[i];
            }
        } else {
            philox_gaussian(p->seed_s, st->s.size(), st->s.data());
        }
        for (double& v : st->s) v = stored_value(v, p->mat_dtype);
    }
    rc = finish_state(st);
    if (rc != TQ_OK) {
        tq_state_destroy(st);
        return rc;
    }
    *out = st;
    return TQ_OK;
}

int tq_state_destroy(tq_state* st) {
    if (!st) return TQ_OK;
    int rc = TQ_OK;
    if (st->d_mem) {
        DeviceGuard g(st->p.device);
        cudaError_t e = cudaFree(st->d_mem);
        if (e != cudaSuccess) rc = cuda_status(e);
    }
    delete st;
    return rc;
}

int tq_state_params(const tq_state* st, tq_params* out) {
    if (!st || !out) return TQ_EINVAL;
    *out = st->p;
    return TQ_OK;
}

int tq_state_codebook_info(const tq_state* st, int* b_mse, double* dmse) {
    if (!st) return TQ_EINVAL;
    if (b_mse) *b_mse = st->b_mse;
    if (dmse) *dmse = st->dmse;
    return TQ_OK;
}

int tq_state_copy(const tq_state* st, int field, double* h_out, size_t count) {
    if (!st || !h_out) return TQ_EINVAL;
    switch (field) {
        case TQ_FIELD_CENTROIDS:
            if (count < st->centroids.size()) return TQ_EINVAL;
            std::copy(st->centroids.begin(), st->centroids.end(), h_out);
            return TQ_OK;
        case TQ_FIELD_BOUNDS:
            if (count < st->bounds.size()) return TQ_EINVAL;
            std::copy(st->bounds.begin(), st->bounds.end(), h_out);
            return TQ_OK;
        case TQ_FIELD_PI:
            if (st->pi.empty() || count < st->pi.size()) return TQ_EINVAL;
            std::copy(st->pi.begin(), st->pi.end(), h_out);
            return TQ_OK;
        case TQ_FIELD_SIGNS:
            if (st->signs.empty() || count < st->signs.size()) return TQ_EINVAL;
            for (size_t i = 0; i < st->signs.size(); ++i) h_out[i] = st->signs[i];
            return TQ_OK;
        case TQ_FIELD_S:
            if (st->s.empty() || count < st->s.size()) return TQ_EINVAL;
            std::copy(st->s.begin(), st->s.end(), h_out);
            return TQ_OK;
        default:
            return TQ_EINVAL;
    }
}

// Export format (little-endian host layout): magic "TQS1", tq_params, b_mse, dmse,
// then the sizes and contents of centroids, bounds, pi, signs, s.
int tq_state_export(const tq_state* st, void* h_buf, size_t* bytes) {
    if (!st || !bytes) return TQ_EINVAL;
    const size_t need = 4 + sizeof(tq_params) + sizeof(int32_t) + sizeof(double) + 5 * sizeof(uint64_t) +
                        8 * (st->centroids.size() + st->bounds.size() + st->pi.size() + st->s.size()) +
                        st->signs.size();
    if (!h_buf) {
        *bytes = need;
        return TQ_OK;
    }
    if (*bytes < need) {
        *bytes = need;
        return TQ_ENOMEM;
    }
    unsigned char* o = (unsigned char*)h_buf;
    auto put = [&](const void* src, size_t n) {
        std::memcpy(o, src, n);
        o += n;
    };
    put("TQS1", 4);
    put(&st->p, sizeof(tq_params));
    int32_t bm = st->b_mse;
    put(&bm, sizeof(bm));
    put(&st->dmse, sizeof(double));
    uint64_t sz[5] = {st->centroids.size(), st->bounds.size(), st->pi.size(), st->signs.size(), st->s.size()};
    put(sz, sizeof(sz));
    put(st->centroids.data(), 8 * sz[0]);
    put(st->bounds.data(), 8 * sz[1]);
    put(st->pi.data(), 8 * sz[2]);
    put(st->signs.data(), sz[3]);
    put(st->s.data(), 8 * sz[4]);
    *bytes = need;
    return TQ_OK;
}

int tq_state_import(const void* h_buf, size_t bytes, int device, tq_state** out) {
    if (!h_buf || !out) return TQ_EINVAL;
    *out = nullptr;
    const unsigned char* in = (const unsigned char*)h_buf;
    const unsigned char* end = in + bytes;
    auto get = [&](void* dst, size_t n) -> bool {
        if ((size_t)(end - in) < n) return false;
        std::memcpy(dst, in, n);
        in += n;
        return true;
    };
    char magic[4];
    tq_params p;
    int32_t bm;
    double dmse;
    uint64_t sz[5];
    if (!get(magic, 4) || std::memcmp(magic, "TQS1", 4) != 0) return TQ_EINVAL;
    if (!get(&p, sizeof(p)) || !get(&bm, sizeof(bm)) || !get(&dmse, sizeof(dmse)) || !get(sz, sizeof(sz)))
        return TQ_EINVAL;
    if (device >= 0) p.device = device;
    int rc = validate_params(&p);
    if (rc != TQ_OK) return rc;
    const size_t d2 = (size_t)p.d * p.d;
    const int want_bm = (p.mode == TQ_MSE) ? p.b : p.b - 1;
    if (bm != want_bm || sz[0] != (1ull << bm) || sz[1] != (sz[0] - 1) ||
        sz[2] != (p.rot == TQ_ROT_DENSE ? d2 : 0) || sz[3] != (p.rot == TQ_ROT_RHT ? (size_t)p.d : 0) ||
        sz[4] != (p.mode == TQ_PROD ? d2 : 0))
        return TQ_EINVAL;
    tq_state* st = new (std::nothrow) tq_state();
    if (!st) return TQ_ENOMEM;
    st->p = p;
    st->b_mse = bm;
    st->dmse = dmse;
    st->centroids.resize(sz[0]);
    st->bounds.resize(sz[1]);
    st->pi.resize(sz[2]);
    st->signs.resize(sz[3]);
    st->s.resize(sz[4]);
    bool ok = get(st->centroids.data(), 8 * sz[0]) && get(st->bounds.data(), 8 * sz[1]) &&
              get(st->pi.data(), 8 * sz[2]) && get(st->signs.data(), sz[3]) && get(st->s.data(), 8 * sz[4]);
    if (!ok) {
        delete st;
        return TQ_EINVAL;
    }
    rc = finish_state(st);
    if (rc != TQ_OK) {
        tq_state_destroy(st);
        return rc;
    }
    *out = st;
    return TQ_OK;
}

int tq_code_layout(const tq_state* st, size_t* code_bytes, size_t* qjl_bytes) {
    if (!st) return TQ_EINVAL;
    if (code_bytes) *code_bytes = (size_t)st->dev.code_bytes;
    if (qjl_bytes) *qjl_bytes = (size_t)st->dev.qjl_bytes;
    return TQ_OK;
}

int tq_quantize_workspace(const tq_state* st, int dtype, int64_t n, int64_t ld, size_t* bytes) {
    if (!st || !bytes || n < 0 || (dtype != TQ_F32 && dtype != TQ_BF16)) return TQ_EINVAL;
    *bytes = encode_ws_bytes(st->dev, dtype, n, ld);
    return TQ_OK;
}

namespace {
int check_encode_ws(const tq_state* st, int dtype, int64_t n, int64_t ld, const void* ws, size_t ws_bytes) {
    const size_t need = encode_ws_min_bytes(st->dev, dtype, n, ld);
    if (need == 0) return TQ_OK;
    if (!ws || ((uintptr_t)ws & 255u)) return TQ_EINVAL;
    return ws_bytes < need ? TQ_ENOMEM : TQ_OK;
}
}  // namespace

int tq_quantize_mse(const tq_state* st, const void* x, int dtype, int64_t n, int64_t ld,
                    uint8_t* codes, float* norms, void* workspace, size_t ws_bytes, void* stream) {
    if (!st || st->p.mode != TQ_MSE) return TQ_EINVAL;
    int rc = check_vectors(st, x, dtype, n, ld);
    if (rc != TQ_OK || n == 0) return rc;
    if (!codes || !norms || !aligned16(codes) || !aligned16(norms)) return TQ_EINVAL;
    rc = check_encode_ws(st, dtype, n, ld, workspace, ws_bytes);
    if (rc != TQ_OK) return rc;
    DeviceGuard g(st->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    return cuda_status((cudaError_t)launch_encode(st->dev, x, dtype, n, ld, codes, nullptr, norms, nullptr,
                                                  workspace, ws_bytes, stream));
}

int tq_quantize_prod(const tq_state* st, const void* x, int dtype, int64_t n, int64_t ld,
                     uint8_t* codes, uint8_t* qjl, float* norms, float* rnorms, void* workspace, size_t ws_bytes,
                     void* stream) {
    if (!st || st->p.mode != TQ_PROD) return TQ_EINVAL;
    int rc = check_vectors(st, x, dtype, n, ld);
    if (rc != TQ_OK || n == 0) return rc;
    if ((st->b_mse > 0 && (!codes || !aligned16(codes))) || !qjl || !norms || !rnorms ||
        !aligned16(qjl) || !aligned16(norms) || !aligned16(rnorms))
        return TQ_EINVAL;
    rc = check_encode_ws(st, dtype, n, ld, workspace, ws_bytes);
    if (rc != TQ_OK) return rc;
    DeviceGuard g(st->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    return cuda_status((cudaError_t)launch_encode(st->dev, x, dtype, n, ld, codes, qjl, norms, rnorms, workspace,
                                                  ws_bytes, stream));
}

int tq_dequant(const tq_state* st, const uint8_t* codes, const uint8_t* qjl, const float* norms,
               const float* rnorms, int64_t n, float* out, void* stream) {
    if (!st || n < 0) return TQ_EINVAL;
    if (n == 0) return TQ_OK;
    const bool prod = st->p.mode == TQ_PROD;
    if ((st->b_mse > 0 && !codes) || !norms || !out || (prod && (!qjl || !rnorms))) return TQ_EINVAL;
    if (!aligned16(out)) return TQ_EINVAL;
    DeviceGuard g(st->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    return cuda_status((cudaError_t)launch_dequant(st->dev, codes, prod ? qjl : nullptr, norms,
                                                   prod ? rnorms : nullptr, n, nullptr, st->p.d, out, stream));
}

int tq_score_workspace(const tq_state* st, int64_t groups, int64_t nq, size_t* bytes) {
    if (!st || !bytes || groups < 0 || nq < 0) return TQ_EINVAL;
    *bytes = score_ws_bytes(st->dev, groups, nq);
    return TQ_OK;
}

int tq_score(const tq_state* st, const void* q, int qdtype, int64_t groups, int64_t nq,
             const uint8_t* codes, const uint8_t* qjl, const float* norms, const float* rnorms,
             int64_t n, float* scores, void* workspace, size_t ws_bytes, void* stream) {
    if (!st || groups < 0 || nq < 0 || n < 0) return TQ_EINVAL;
    if (qdtype != TQ_F32 && qdtype != TQ_BF16) return TQ_EINVAL;
    if (groups == 0 || nq == 0 || n == 0) return TQ_OK;
    if (groups > 65535) return TQ_EUNSUPPORTED;
    const bool prod = st->p.mode == TQ_PROD;
    if (!q || !scores || !norms || (st->b_mse > 0 && !codes) || (prod && (!qjl || !rnorms)))
        return TQ_EINVAL;
    if (!aligned16(q) || (codes && !aligned16(codes)) || (prod && !aligned16(qjl))) return TQ_EINVAL;
    const size_t need = score_ws_bytes(st->dev, groups, nq);
    if (need > 0) {
        if (!workspace || ((uintptr_t)workspace & 255u)) return TQ_EINVAL;
        if (ws_bytes < need) return TQ_ENOMEM;
    }
    DeviceGuard g(st->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    return cuda_status((cudaError_t)launch_score(st->dev, q, qdtype, groups, nq, codes, prod ? qjl : nullptr,
                                                 norms, prod ? rnorms : nullptr, n, 0, scores, workspace, stream));
}

// ---- prefix coding of the indices -------------------------------------------------------

int tq_entropy_table(const tq_state* st, int* h_lengths, uint32_t* h_words, double* h_mean_bits) {
    if (!st || st->b_mse < 1) return TQ_EINVAL;
    EntropyTable tab;
    int rc = build_prefix_code(st, &tab);
    if (rc != TQ_OK) return rc;
    for (int i = 0; i < tab.L; ++i) {
        if (h_lengths) h_lengths[i] = tab.len[i];
        if (h_words) h_words[i] = tab.word[i];
    }
    if (h_mean_bits) *h_mean_bits = tab.mean_bits;
    return TQ_OK;
}

int tq_entropy_max_bytes(const tq_state* st, int64_t n, size_t* bytes) {
    if (!st || st->b_mse < 1 || n < 0 || !bytes) return TQ_EINVAL;
    EntropyTable tab;
    int rc = build_prefix_code(st, &tab);
    if (rc != TQ_OK) return rc;
    const uint64_t bits = (uint64_t)n * st->p.d * tab.maxlen;
    *bytes = (size_t)((bits + 31) / 32) * 4 + 16;
    return TQ_OK;
}

int tq_entropy_workspace(const tq_state* st, int64_t n, size_t* bytes) {
    if (!st || n < 0 || !bytes) return TQ_EINVAL;
    *bytes = entropy_ws_bytes(n);
    return TQ_OK;
}

int tq_entropy_encode(const tq_state* st, const uint8_t* codes, int64_t n, uint64_t* offsets, uint8_t* stream,
                      size_t capacity, void* workspace, size_t ws_bytes, void* cuda_stream) {
    if (!st || st->b_mse < 1 || n < 0) return TQ_EINVAL;
    if (n == 0) return TQ_OK;
    if (!codes || !offsets || !stream || !workspace || !aligned16(codes) || ((uintptr_t)offsets & 7u) ||
        ((uintptr_t)stream & 3u) || ((uintptr_t)workspace & 255u))
        return TQ_EINVAL;
    EntropyTable tab;
    int rc = build_prefix_code(st, &tab);
    if (rc != TQ_OK) return rc;
    const uint64_t bits = (uint64_t)n * st->p.d * tab.maxlen;
    if (capacity < (size_t)((bits + 31) / 32) * 4 + 16 || ws_bytes < entropy_ws_bytes(n)) return TQ_ENOMEM;
    DeviceGuard g(st->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    return cuda_status((cudaError_t)launch_entropy_encode(st->dev, tab, codes, n, offsets, stream, capacity,
                                                          workspace, cuda_stream));
}

int tq_entropy_decode(const tq_state* st, const uint8_t* stream, const uint64_t* offsets, int64_t n, uint8_t* codes,
                      void* cuda_stream) {
    if (!st || st->b_mse < 1 || n < 0) return TQ_EINVAL;
    if (n == 0) return TQ_OK;
    if (!codes || !offsets || !stream || !aligned16(codes) || ((uintptr_t)offsets & 7u) || ((uintptr_t)stream & 3u))
        return TQ_EINVAL;
    EntropyTable tab;
    int rc = build_prefix_code(st, &tab);
    if (rc != TQ_OK) return rc;
    DeviceGuard g(st->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    return cuda_status((cudaError_t)launch_entropy_decode(st->dev, tab, stream, offsets, n, codes, cuda_stream));
}

// ---- outlier-channel split -----------------------------------------------------------

namespace {
bool planes_ok(const tq_state* st, const tq_planes* p) {
    if (!p || !p->norms || !aligned16(p->norms)) return false;
    if (st->b_mse > 0 && (!p->codes || !aligned16(p->codes))) return false;
    if (st->p.mode == TQ_PROD && (!p->qjl || !p->rnorms || !aligned16(p->qjl) || !aligned16(p->rnorms)))
        return false;
    return true;
}
}  // namespace

namespace {
// Entry (n, k) of the Hadamard matrix of a state's order d: Sylvester's (-1)^popcount(n & k) for
// d a power of two, else H_12 (x) H_{d/12} (Paley's H_12 from the state).
bool hadamard_negative(const tq_state* st, int n, int k) {
    const int d = st->p.d;
    if ((d & (d - 1)) == 0) return __builtin_popcount((unsigned)(n & k)) & 1;
    const int q = d / 12;
    const bool neg12 = (st->dev.h12[n / q] >> (k / q)) & 1u;
    return neg12 ^ (bool)(__builtin_popcount((unsigned)((n % q) & (k % q))) & 1);
}

uint16_t bf16_bits_exact(double v) {   // v is a stored bf16 value
    const float f = (float)v;
    uint32_t u;
    std::memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

// Operands of the split on the tensor-core encoder: row r < m of the rotation holds row r of
// the outer group's H diag(eps) at the outer channels, row m + r the inner group's at the
// inner channels (+-1: the 1/sqrt(d_g) of each group cancels in y / ||y_g||); then S of the
// two groups on the diagonal blocks.
void split_tc_operands(const tq_state* outer, const tq_state* inner, const std::vector<int32_t>& maps,
                       std::vector<uint16_t>& ops) {
    ops.assign(2 * 128 * 128, 0);
    const tq_state* st[2] = {outer, inner};
    int off = 0;
    for (int g = 0; g < 2; ++g) {
        const tq_state* s = st[g];
        const int dg = s->p.d;
        for (int n = 0; n < dg; ++n) {
            for (int k = 0; k < dg; ++k) {
                const bool eps_neg = (s->dev.signs[k >> 5] >> (k & 31)) & 1u;
                ops[(size_t)(off + n) * 128 + maps[off + k]] = (hadamard_negative(s, n, k) ^ eps_neg) ? 0xBF80u : 0x3F80u;
                if (s->p.mode == TQ_PROD)
                    ops[128 * 128 + (size_t)(off + n) * 128 + off + k] = bf16_bits_exact(s->s[(size_t)n * dg + k]);
            }
        }
        off += dg;
    }
}
}  // namespace

int tq_split_create(const tq_state* outer, const tq_state* inner, const int32_t* h_channels, int m,
                    tq_split** out) {
    if (!outer || !inner || !out || m < 1) return TQ_EINVAL;
    *out = nullptr;
    if (outer->p.d != m || outer->p.mode != inner->p.mode || outer->p.device != inner->p.device) return TQ_EINVAL;
    if (!h_channels) return TQ_EINVAL;
    const int d = m + inner->p.d;
    std::vector<int32_t> maps(d);
    for (int i = 0; i < m; ++i) {
        if (h_channels[i] < 0 || h_channels[i] >= d || (i > 0 && h_channels[i] <= h_channels[i - 1])) return TQ_EINVAL;
        maps[i] = h_channels[i];
    }
    for (int c = 0, j = 0, k = m; c < d; ++c) {   // the inner map: every channel not listed, ascending
        if (j < m && h_channels[j] == c) ++j;
        else maps[k++] = c;
    }
    DeviceGuard g(outer->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    auto* sp = new tq_split;
    sp->outer = outer;
    sp->inner = inner;
    sp->d = d;
    sp->channels.assign(h_channels, h_channels + m);
    cudaError_t e = cudaMalloc(&sp->d_chan, (size_t)d * sizeof(int32_t));
    if (e == cudaSuccess) e = cudaMemcpy(sp->d_chan, maps.data(), (size_t)d * sizeof(int32_t), cudaMemcpyHostToDevice);
    if (e == cudaSuccess && d == 128 && tq::split_tc_supported(outer->dev, inner->dev, m)) {
        std::vector<uint16_t> ops;
        split_tc_operands(outer, inner, maps, ops);
        e = cudaMalloc(&sp->d_tc, ops.size() * sizeof(uint16_t));
        if (e == cudaSuccess) e = cudaMemcpy(sp->d_tc, ops.data(), ops.size() * sizeof(uint16_t), cudaMemcpyHostToDevice);
    }
    if (e != cudaSuccess) {
        if (sp->d_chan) cudaFree(sp->d_chan);
        if (sp->d_tc) cudaFree(sp->d_tc);
        delete sp;
        return cuda_status(e);
    }
    *out = sp;
    return TQ_OK;
}

void tq_split_destroy(tq_split* sp) {
    if (!sp) return;
    if (sp->d_chan || sp->d_tc) {
        DeviceGuard g(sp->outer->p.device);
        if (sp->d_chan) cudaFree(sp->d_chan);
        if (sp->d_tc) cudaFree(sp->d_tc);
    }
    delete sp;
}

int tq_split_quantize(const tq_split* sp, const void* x, int dtype, int64_t n, int64_t ld,
                      const tq_planes* outer, const tq_planes* inner, void* stream) {
    if (!sp || n < 0) return TQ_EINVAL;
    if (dtype != TQ_F32 && dtype != TQ_BF16) return TQ_EINVAL;
    if (n == 0) return TQ_OK;
    const size_t es = (dtype == TQ_F32) ? 4 : 2;
    if (!x || ld < sp->d || !aligned16(x) || ((size_t)ld * es) % 16) return TQ_EINVAL;
    if (!planes_ok(sp->outer, outer) || !planes_ok(sp->inner, inner)) return TQ_EINVAL;
    DeviceGuard g(sp->outer->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    const bool prod = sp->outer->p.mode == TQ_PROD;
    const int m = sp->outer->p.d;
    if (sp->d_tc && dtype == TQ_BF16 && n < ((int64_t)1 << 31)) {
        uint8_t* const codes[2] = {outer->codes, inner->codes};
        uint8_t* const qjl[2] = {prod ? outer->qjl : nullptr, prod ? inner->qjl : nullptr};
        float* const norms[2] = {outer->norms, inner->norms};
        float* const rnorms[2] = {prod ? outer->rnorms : nullptr, prod ? inner->rnorms : nullptr};
        return cuda_status((cudaError_t)tq::launch_encode_split_tc(sp->outer->dev, sp->inner->dev, sp->d_tc,
                                                                   sp->d_tc + 128 * 128, x, n, ld, codes, qjl, norms,
                                                                   rnorms, stream));
    }
    int e = launch_encode_channels(sp->outer->dev, x, dtype, n, ld, sp->d_chan, outer->codes,
                                   prod ? outer->qjl : nullptr, outer->norms, prod ? outer->rnorms : nullptr, stream);
    if (e == 0)
        e = launch_encode_channels(sp->inner->dev, x, dtype, n, ld, sp->d_chan + m, inner->codes,
                                   prod ? inner->qjl : nullptr, inner->norms, prod ? inner->rnorms : nullptr, stream);
    return cuda_status((cudaError_t)e);
}

int tq_split_dequant(const tq_split* sp, const tq_planes* outer, const tq_planes* inner, int64_t n, float* out,
                     void* stream) {
    if (!sp || n < 0) return TQ_EINVAL;
    if (n == 0) return TQ_OK;
    if (!out || !aligned16(out) || !planes_ok(sp->outer, outer) || !planes_ok(sp->inner, inner)) return TQ_EINVAL;
    DeviceGuard g(sp->outer->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    const bool prod = sp->outer->p.mode == TQ_PROD;
    const int m = sp->outer->p.d;
    int e = launch_dequant(sp->outer->dev, outer->codes, prod ? outer->qjl : nullptr, outer->norms,
                           prod ? outer->rnorms : nullptr, n, sp->d_chan, sp->d, out, stream);
    if (e == 0)
        e = launch_dequant(sp->inner->dev, inner->codes, prod ? inner->qjl : nullptr, inner->norms,
                           prod ? inner->rnorms : nullptr, n, sp->d_chan + m, sp->d, out, stream);
    return cuda_status((cudaError_t)e);
}

namespace {
// tq_split_score's workspace: the queries' outer channels [rows][m], their inner channels
// [rows][d - m] (each 256-byte aligned), then one region for the groups' score tables
// (used by the two score launches in turn).
size_t split_score_ws(const tq_split* sp, int qdtype, int64_t groups, int64_t nq, size_t* q_inner_off,
                      size_t* tables_off) {
    const int m = sp->outer->p.d, r = sp->d - m;
    const size_t rows = (size_t)groups * nq, es = (qdtype == TQ_F32) ? 4 : 2;
    const size_t b_out = (rows * m * es + 255) & ~(size_t)255;
    const size_t b_in = (rows * r * es + 255) & ~(size_t)255;
    if (q_inner_off) *q_inner_off = b_out;
    if (tables_off) *tables_off = b_out + b_in;
    return b_out + b_in + std::max(score_ws_bytes(sp->outer->dev, groups, nq), score_ws_bytes(sp->inner->dev, groups, nq));
}
}  // namespace

int tq_split_score_workspace(const tq_split* sp, int qdtype, int64_t groups, int64_t nq, size_t* bytes) {
    if (!sp || !bytes || groups < 0 || nq < 0 || (qdtype != TQ_F32 && qdtype != TQ_BF16)) return TQ_EINVAL;
    *bytes = (groups == 0 || nq == 0) ? 0 : split_score_ws(sp, qdtype, groups, nq, nullptr, nullptr);
    return TQ_OK;
}

int tq_split_score(const tq_split* sp, const void* q, int qdtype, int64_t groups, int64_t nq,
                   const tq_planes* outer, const tq_planes* inner, int64_t n, float* scores, void* workspace,
                   size_t ws_bytes, void* stream) {
    if (!sp || groups < 0 || nq < 0 || n < 0) return TQ_EINVAL;
    if (qdtype != TQ_F32 && qdtype != TQ_BF16) return TQ_EINVAL;
    if (groups == 0 || nq == 0 || n == 0) return TQ_OK;
    if (groups > 65535) return TQ_EUNSUPPORTED;
    if (!q || !scores || !aligned16(q) || !planes_ok(sp->outer, outer) || !planes_ok(sp->inner, inner))
        return TQ_EINVAL;
    size_t q_in_off = 0, tab_off = 0;
    const size_t need = split_score_ws(sp, qdtype, groups, nq, &q_in_off, &tab_off);
    if (!workspace || ((uintptr_t)workspace & 255u)) return TQ_EINVAL;
    if (ws_bytes < need) return TQ_ENOMEM;
    DeviceGuard g(sp->outer->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    const bool prod = sp->outer->p.mode == TQ_PROD;
    const int m = sp->outer->p.d, r = sp->d - m;
    const int64_t rows = groups * nq;
    unsigned char* w = reinterpret_cast<unsigned char*>(workspace);
    void* q_out = w;
    void* q_in = w + q_in_off;
    void* tables = w + tab_off;
    int e = launch_gather_rows(q, qdtype, rows, sp->d, sp->d_chan, m, q_out, stream);
    if (e == 0) e = launch_gather_rows(q, qdtype, rows, sp->d, sp->d_chan + m, r, q_in, stream);
    if (e == 0)
        e = launch_score(sp->outer->dev, q_out, qdtype, groups, nq, outer->codes, prod ? outer->qjl : nullptr,
                         outer->norms, prod ? outer->rnorms : nullptr, n, 0, scores, tables, stream);
    if (e == 0)
        e = launch_score(sp->inner->dev, q_in, qdtype, groups, nq, inner->codes, prod ? inner->qjl : nullptr,
                         inner->norms, prod ? inner->rnorms : nullptr, n, 1, scores, tables, stream);
    return cuda_status((cudaError_t)e);
}

int tq_split_attend_workspace(const tq_split* ks, const tq_split* vs, int H, int64_t T, size_t* bytes) {
    if (!ks || !vs || !bytes || H < 0 || T < 0) return TQ_EINVAL;
    *bytes = split_attend_ws_bytes(ks->outer->dev, ks->inner->dev, vs->outer->p.d, vs->d, H, T);
    return TQ_OK;
}

int tq_split_attend_decode(const tq_split* ks, const tq_split* vs, const void* q, int qdtype, int H, int64_t T,
                           const tq_planes* k_outer, const tq_planes* k_inner, const tq_planes* v_outer,
                           const tq_planes* v_inner, float scale, float* out, void* workspace, size_t ws_bytes,
                           void* stream) {
    if (!ks || !vs || H < 0 || T < 0) return TQ_EINVAL;
    if (qdtype != TQ_F32 && qdtype != TQ_BF16) return TQ_EINVAL;
    if (vs->outer->p.mode != TQ_MSE || ks->d != vs->d || ks->outer->p.device != vs->outer->p.device)
        return TQ_EINVAL;
    if (!std::isfinite(scale)) return TQ_EINVAL;
    if (H == 0) return TQ_OK;
    if (T == 0 || H > 65535) return T == 0 ? TQ_EINVAL : TQ_EUNSUPPORTED;
    if (!q || !out || !aligned16(q) || !aligned16(out)) return TQ_EINVAL;
    if (!planes_ok(ks->outer, k_outer) || !planes_ok(ks->inner, k_inner) || !planes_ok(vs->outer, v_outer) ||
        !planes_ok(vs->inner, v_inner))
        return TQ_EINVAL;
    const size_t need = split_attend_ws_bytes(ks->outer->dev, ks->inner->dev, vs->outer->p.d, vs->d, H, T);
    if (!workspace || ws_bytes < need || ((uintptr_t)workspace & 255u)) return TQ_EINVAL;
    DeviceGuard g(ks->outer->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    const bool prod = ks->outer->p.mode == TQ_PROD;
    SplitPlanes kp{{k_outer->codes, k_inner->codes},
                   {prod ? k_outer->qjl : nullptr, prod ? k_inner->qjl : nullptr},
                   {k_outer->norms, k_inner->norms},
                   {prod ? k_outer->rnorms : nullptr, prod ? k_inner->rnorms : nullptr}};
    SplitPlanes vp{{v_outer->codes, v_inner->codes}, {nullptr, nullptr}, {v_outer->norms, v_inner->norms},
                   {nullptr, nullptr}};
    return cuda_status((cudaError_t)launch_split_attend(ks->outer->dev, ks->inner->dev, ks->d_chan, vs->outer->dev,
                                                         vs->inner->dev, vs->d_chan, q, qdtype, H, T, kp, vp, scale,
                                                         out, workspace, stream));
}

int tq_attend_workspace(const tq_state* ks, const tq_state* vs, int H, int64_t T, size_t* bytes) {
    if (!ks || !vs || !bytes || H < 0 || T < 0) return TQ_EINVAL;
    *bytes = attend_workspace_bytes(ks->dev, H, T);
    return TQ_OK;
}

int tq_attend_decode(const tq_state* ks, const tq_state* vs, const void* q, int qdtype, int H,
                     int64_t T, const uint8_t* kcodes, const uint8_t* kqjl, const float* knorms,
                     const float* krnorms, const uint8_t* vcodes, const float* vnorms, float scale,
                     float* out, void* workspace, size_t ws_bytes, void* stream) {
    if (!ks || !vs || H < 0 || T < 0) return TQ_EINVAL;
    if (qdtype != TQ_F32 && qdtype != TQ_BF16) return TQ_EINVAL;
    if (vs->p.mode != TQ_MSE || ks->p.d != vs->p.d || ks->p.device != vs->p.device) return TQ_EINVAL;
    if (!std::isfinite(scale)) return TQ_EINVAL;
    if (H == 0) return TQ_OK;
    if (T == 0) return TQ_EINVAL;   // softmax over no tokens is undefined
    const bool prod = ks->p.mode == TQ_PROD;
    if (!q || !out || !knorms || !vnorms || (ks->b_mse > 0 && !kcodes) || !vcodes ||
        (prod && (!kqjl || !krnorms)))
        return TQ_EINVAL;
    if (!aligned16(q) || !aligned16(out)) return TQ_EINVAL;
    const size_t need = attend_workspace_bytes(ks->dev, H, T);
    if (need > 0 && (!workspace || ((uintptr_t)workspace & 255u))) return TQ_EINVAL;
    if (ws_bytes < need) return TQ_ENOMEM;
    DeviceGuard g(ks->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    return cuda_status((cudaError_t)launch_attend(ks->dev, vs->dev, q, qdtype, H, T, 1, T, kcodes,
                                                  prod ? kqjl : nullptr, knorms, prod ? krnorms : nullptr, vcodes,
                                                  vnorms, scale, out, workspace, ws_bytes, stream));
}

namespace {
// Checks shared by the grouped and appending decode steps.
int check_grouped(const tq_state* ks, const tq_state* vs, const void* q, int qdtype, int H, int G, int64_t T,
                  int64_t Tcap, const uint8_t* kcodes, const uint8_t* kqjl, const float* knorms,
                  const float* krnorms, const uint8_t* vcodes, const float* vnorms, float scale, const float* out) {
    if (!ks || !vs || H < 1 || G < 1 || H % G != 0 || T < 1 || Tcap < T) return TQ_EINVAL;
    if (qdtype != TQ_F32 && qdtype != TQ_BF16) return TQ_EINVAL;
    if (vs->p.mode != TQ_MSE || ks->p.d != vs->p.d || ks->p.device != vs->p.device) return TQ_EINVAL;
    if (!std::isfinite(scale)) return TQ_EINVAL;
    const bool prod = ks->p.mode == TQ_PROD;
    if (!q || !out || !knorms || !vnorms || (ks->b_mse > 0 && !kcodes) || !vcodes ||
        (prod && (!kqjl || !krnorms)))
        return TQ_EINVAL;
    if (!aligned16(q) || !aligned16(out)) return TQ_EINVAL;
    return TQ_OK;
}
}  // namespace

int tq_attend_decode_grouped(const tq_state* ks, const tq_state* vs, const void* q, int qdtype, int H, int G,
                             int64_t T, int64_t Tcap, const uint8_t* kcodes, const uint8_t* kqjl,
                             const float* knorms, const float* krnorms, const uint8_t* vcodes, const float* vnorms,
                             float scale, float* out, void* workspace, size_t ws_bytes, void* stream) {
    int rc = check_grouped(ks, vs, q, qdtype, H, G, T, Tcap, kcodes, kqjl, knorms, krnorms, vcodes, vnorms, scale,
                           out);
    if (rc != TQ_OK) return rc;
    const size_t need = attend_workspace_bytes(ks->dev, H, T);
    if (need > 0 && (!workspace || ((uintptr_t)workspace & 255u))) return TQ_EINVAL;
    if (ws_bytes < need) return TQ_ENOMEM;
    DeviceGuard g(ks->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    const bool prod = ks->p.mode == TQ_PROD;
    return cuda_status((cudaError_t)launch_attend(ks->dev, vs->dev, q, qdtype, H, T, G, Tcap, kcodes,
                                                  prod ? kqjl : nullptr, knorms, prod ? krnorms : nullptr, vcodes,
                                                  vnorms, scale, out, workspace, ws_bytes, stream));
}

int tq_attend_append_decode(const tq_state* ks, const tq_state* vs, const void* q, int qdtype, int H, int G,
                            const void* k_new, const void* v_new, int kvdtype, int64_t T, int64_t Tcap,
                            uint8_t* kcodes, uint8_t* kqjl, float* knorms, float* krnorms, uint8_t* vcodes,
                            float* vnorms, float scale, float* out, void* workspace, size_t ws_bytes, void* stream) {
    if (T < 0 || T >= Tcap) return TQ_EINVAL;
    int rc = check_grouped(ks, vs, q, qdtype, H, G, T + 1, Tcap, kcodes, kqjl, knorms, krnorms, vcodes, vnorms,
                           scale, out);
    if (rc != TQ_OK) return rc;
    if (kvdtype != TQ_F32 && kvdtype != TQ_BF16) return TQ_EINVAL;
    if (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)) return TQ_EINVAL;
    const size_t need = attend_workspace_bytes(ks->dev, H, T + 1);
    if (need > 0 && (!workspace || ((uintptr_t)workspace & 255u))) return TQ_EINVAL;
    if (ws_bytes < need) return TQ_ENOMEM;
    DeviceGuard g(ks->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    const bool prod = ks->p.mode == TQ_PROD;
    // the new token of every KV head goes into row T of that head's planes inside the decode
    // step (d = 128: by the launch that builds the query tables), then attention over T + 1
    AppendRow app = {};
    app.k_new = k_new;
    app.v_new = v_new;
    app.dtype = kvdtype;
    app.G = G;
    app.Tcap = Tcap;
    app.kcodes = kcodes ? kcodes + T * ks->dev.code_bytes : nullptr;
    app.kqjl = prod ? kqjl + T * ks->dev.qjl_bytes : nullptr;
    app.knorms = knorms + T;
    app.krnorms = prod ? krnorms + T : nullptr;
    app.vcodes = vcodes + T * vs->dev.code_bytes;
    app.vnorms = vnorms + T;
    const int e = launch_attend(ks->dev, vs->dev, q, qdtype, H, T + 1, G, Tcap, kcodes, prod ? kqjl : nullptr, knorms,
                                prod ? krnorms : nullptr, vcodes, vnorms, scale, out, workspace, ws_bytes, stream, &app);
    return cuda_status((cudaError_t)e);
}

int tq_attend_decode_noalloc(const tq_state* ks, const tq_state* vs, const void* q, int qdtype, int H, int64_t T,
                             const uint8_t* kcodes, const uint8_t* kqjl, const float* knorms, const float* krnorms,
                             const uint8_t* vcodes, const float* vnorms, float scale, float* out, void* stream) {
    if (!ks || !vs || H < 0 || T < 0) return TQ_EINVAL;
    if (qdtype != TQ_F32 && qdtype != TQ_BF16) return TQ_EINVAL;
    if (vs->p.mode != TQ_MSE || ks->p.d != vs->p.d || ks->p.device != vs->p.device) return TQ_EINVAL;
    if (!std::isfinite(scale)) return TQ_EINVAL;
    if (H == 0) return TQ_OK;
    if (T == 0) return TQ_EINVAL;
    const bool prod = ks->p.mode == TQ_PROD;
    if (!q || !out || !knorms || !vnorms || (ks->b_mse > 0 && !kcodes) || !vcodes ||
        (prod && (!kqjl || !krnorms)))
        return TQ_EINVAL;
    if (!aligned16(q) || !aligned16(out)) return TQ_EINVAL;
    const size_t need = attend_workspace_bytes(ks->dev, H, T);
    if (need > kAttendStaticScratchBytes) return TQ_EUNSUPPORTED;   // beyond the fixed 4 MiB array
    DeviceGuard g(ks->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    void* scratch = nullptr;
    int e = attend_static_scratch(&scratch);
    if (e != 0) return cuda_status((cudaError_t)e);
    return cuda_status((cudaError_t)launch_attend(ks->dev, vs->dev, q, qdtype, H, T, 1, T, kcodes,
                                                  prod ? kqjl : nullptr, knorms, prod ? krnorms : nullptr, vcodes,
                                                  vnorms, scale, out, scratch, kAttendStaticScratchBytes, stream));
}

int tq_ip_stats(const float* x, const float* xt, int64_t n, int d, const float* q, int64_t nq, double* out,
                void* stream, int device) {
    if (n < 0 || nq < 0 || d < 1 || !out || device < 0) return TQ_EINVAL;
    if (d > 256) return TQ_EUNSUPPORTED;
    if (n > 0 && (!x || !xt)) return TQ_EINVAL;
    if (nq > 0 && !q) return TQ_EINVAL;
    DeviceGuard g(device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    return cuda_status((cudaError_t)launch_ip_stats(x, xt, n, d, q, nq, out, stream));
}

int tq_search_workspace(const tq_state* st, int64_t nq, int64_t n, int k, size_t* bytes) {
    if (!st || !bytes || nq < 0 || n < 0 || k < 1 || k > 64) return TQ_EINVAL;
    *bytes = search_workspace_bytes(st->dev, nq, n, k);
    return TQ_OK;
}

int tq_search_topk(const tq_state* st, const void* q, int qdtype, int64_t nq, const uint8_t* codes,
                   const uint8_t* qjl, const float* norms, const float* rnorms, int64_t n, int k,
                   int64_t* idx, float* vals, void* workspace, size_t ws_bytes, void* stream) {
    if (!st || nq < 0 || n < 0 || k < 1 || k > 64) return TQ_EINVAL;
    if (qdtype != TQ_F32 && qdtype != TQ_BF16) return TQ_EINVAL;
    if (nq == 0) return TQ_OK;
    if (k > n) return TQ_EINVAL;
    const bool prod = st->p.mode == TQ_PROD;
    if (!q || !idx || !vals || !norms || (st->b_mse > 0 && !codes) || (prod && (!qjl || !rnorms)))
        return TQ_EINVAL;
    if (!aligned16(q)) return TQ_EINVAL;
    const size_t need = search_workspace_bytes(st->dev, nq, n, k);
    if (need > 0 && (!workspace || ((uintptr_t)workspace & 255u))) return TQ_EINVAL;
    if (ws_bytes < need) return TQ_ENOMEM;
    DeviceGuard g(st->p.device);
    if (!g.ok) return cuda_status(cudaGetLastError());
    return cuda_status((cudaError_t)launch_search(st->dev, q, qdtype, nq, codes, prod ? qjl : nullptr, norms,
                                                  prod ? rnorms : nullptr, n, k, idx, vals, workspace, ws_bytes,
                                                  stream));
}

}  // extern "C"
