// Internal declarations shared by the host library and the kernels of libtq.
// Not part of the public ABI (include/tq.h is).
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>

#include "../../include/tq.h"

namespace tq {

constexpr int kMaxLevels = 256;      // 2^b_mse with b_mse <= 8
constexpr int kMaxDim = 2048;        // largest d the kernels accept
constexpr int kMaxDevices = 64;
// Size of the fixed device array behind tq_attend_decode_noalloc (4 MiB).
constexpr size_t kAttendStaticScratchBytes = (size_t)4 << 20;

// Everything a kernel needs about a state, passed by value as a kernel parameter
// (lives in the constant bank: uniform reads of the codebook are broadcasts).
struct DevState {
    int d;
    int b_mse;          // bits of MSE code per coordinate (0 for prod b=1)
    int L;              // 2^b_mse
    int mode;           // TQ_MSE / TQ_PROD
    int rot;            // TQ_ROT_DENSE / TQ_ROT_RHT
    int mat_dtype;      // TQ_F32 / TQ_BF16
    int code_bytes;     // ceil(b_mse*d/8)
    int qjl_bytes;      // d/8 (prod) or 0
    float qjl_scale;    // sqrt(pi/2)/d
    float rsqrt_d;      // 1/sqrt(d) (RHT normalisation)
    const void* pi;     // Pi, row-major [d][d] (dense)
    const void* piT;    // Pi^T, row-major [d][d] (dense)
    const void* s;      // S, row-major [d][d] (prod)
    const void* sT;     // S^T, row-major [d][d] (prod)
    uint32_t signs[kMaxDim / 32];  // RHT: bit j set <=> eps_j = -1
    uint32_t h12[12];              // RHT with d = 12 * 2^k: bit c of row a set <=> H_12[a][c] = -1
    float c[kMaxLevels];           // centroids (fp32 stored values)
    float t[kMaxLevels];           // boundaries t[0..L-2]
};

}  // namespace tq

struct tq_state {
    tq_params p;
    int b_mse;
    double dmse;
    std::vector<double> centroids;   // fp64 Lloyd-Max centroids
    std::vector<double> bounds;      // fp64 boundaries
    std::vector<double> pi;          // stored Pi values (after rounding), row-major
    std::vector<int8_t> signs;       // RHT signs
    std::vector<double> s;           // stored S values (after rounding), row-major
    void* d_mem = nullptr;           // one device allocation holding pi, piT, s, sT
    tq::DevState dev;                // kernel view
};

// Canonical prefix code of the codebook indices (see entropy.cpp).
namespace tq {
constexpr int kMaxCodeLen = 32;
struct EntropyTable {
    int L;
    int maxlen;
    double mean_bits;
    uint8_t len[kMaxLevels];           // codeword length of each index
    uint32_t word[kMaxLevels];         // canonical codeword (first bit = most significant)
    uint32_t rword[kMaxLevels];        // the codeword bit-reversed (first bit = bit 0)
    uint16_t sym[kMaxLevels];          // indices in canonical (length, index) order
    uint32_t first[kMaxCodeLen + 2];   // first codeword of each length
    uint16_t count[kMaxCodeLen + 2];   // number of codewords of each length
    uint16_t start[kMaxCodeLen + 2];   // position in sym of the first codeword of each length
};
int build_prefix_code(const tq_state* st, EntropyTable* tab);
size_t entropy_ws_bytes(int64_t n);
int launch_entropy_encode(const DevState& st, const EntropyTable& tab, const uint8_t* codes, int64_t n,
                          uint64_t* offsets, uint8_t* stream, size_t capacity, void* ws, void* cuda_stream);
int launch_entropy_decode(const DevState& st, const EntropyTable& tab, const uint8_t* stream, const uint64_t* offsets,
                          int64_t n, uint8_t* codes, void* cuda_stream);
}  // namespace tq

struct tq_split {
    const tq_state* outer;           // channels `chan_outer`, dimension m
    const tq_state* inner;           // the other channels, ascending, dimension d - m
    int d;
    std::vector<int32_t> channels;   // host copy of the outer channel list
    int32_t* d_chan = nullptr;       // device: outer map [m], then inner map [d - m]
    uint16_t* d_tc = nullptr;        // tensor-core encoder operands (or null): rotation [128][128], then S [128][128], bf16
};

namespace tq {

// ---- host helpers (host.cpp / codebook.cpp / linalg.cpp) ----
int build_codebook(int d, int b, double* c, double* t, double* dmse);
void philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);
void philox_gaussian(uint64_t seed, size_t count, double* out);
void philox_signs(uint64_t seed, size_t count, int8_t* out);
int haar_from_gaussian(int d, const double* g, double* pi_out);
float bf16_round_host(float x);
void paley_hadamard12_rows(uint32_t rows[12]);
void set_cuda_error(int err);

// ---- kernel launchers (kernels .cu files); all return a cudaError_t value ----
// Workspace bytes of launch_encode for n vectors (0 when the configuration needs none; with
// less than this, down to encode_ws_min_bytes, the encoder takes more passes).
size_t encode_ws_bytes(const DevState& st, int dtype, int64_t n, int64_t ld);
size_t encode_ws_min_bytes(const DevState& st, int dtype, int64_t n, int64_t ld);
int launch_encode(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld,
                  uint8_t* codes, uint8_t* qjl, float* norms, float* rnorms, void* ws, size_t ws_bytes,
                  void* stream);
int launch_encode_strided(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, int64_t ostride,
                          uint8_t* codes, uint8_t* qjl, float* norms, float* rnorms, void* stream);
int launch_encode_channels(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, const int32_t* chan,
                           uint8_t* codes, uint8_t* qjl, float* norms, float* rnorms, void* stream);
// out row stride ldo; chan (optional): element j of a vector goes to column chan[j]
int launch_dequant(const DevState& st, const uint8_t* codes, const uint8_t* qjl,
                   const float* norms, const float* rnorms, int64_t n, const int32_t* chan, int64_t ldo,
                   float* out, void* stream);
// Workspace bytes of launch_score for groups * nq queries (the per-query lookup tables; 0
// for the general kernel, which prepares each query in shared memory).
size_t score_ws_bytes(const DevState& st, int64_t groups, int64_t nq);
// accumulate != 0: scores += estimates (else scores = estimates); ws: score_ws_bytes, 256-aligned
int launch_score(const DevState& st, const void* q, int qdtype, int64_t groups, int64_t nq,
                 const uint8_t* codes, const uint8_t* qjl, const float* norms,
                 const float* rnorms, int64_t n, int accumulate, float* scores, void* ws, void* stream);
// rows of q [count][ldq] gathered at columns chan[0..m) into out [count][m] (same dtype)
int launch_gather_rows(const void* q, int dtype, int64_t count, int64_t ldq, const int32_t* chan, int m, void* out,
                       void* stream);
// Outlier-channel split on the two-team tensor-core encoder (d = 128, bf16 input, both groups
// RHT at 1 or 2 bits, m a multiple of 32): pmat / sbd are the [128][128] bf16 rotation and
// block-diagonal S operands built by the host; planes index 0 = outer group, 1 = inner.
bool split_tc_supported(const DevState& so, const DevState& si, int m);
int launch_encode_split_tc(const DevState& so, const DevState& si, const uint16_t* pmat, const uint16_t* sbd,
                           const void* x, int64_t n, int64_t ld, uint8_t* const codes[2], uint8_t* const qjl[2],
                           float* const norms[2], float* const rnorms[2], void* stream);
// Planes of the two channel groups of a split (index 0: outer, 1: inner).
struct SplitPlanes {
    const uint8_t* codes[2];
    const uint8_t* qjl[2];
    const float* norms[2];
    const float* rnorms[2];
};
size_t split_attend_ws_bytes(const DevState& ko, const DevState& ki, int dv_outer, int dv, int H, int64_t T);
int launch_split_attend(const DevState& ko, const DevState& ki, const int32_t* kchan, const DevState& vo,
                        const DevState& vi, const int32_t* vchan, const void* q, int qdtype, int H, int64_t T,
                        const SplitPlanes& kp, const SplitPlanes& vp, float scale, float* out, void* ws,
                        void* stream);
int launch_expired_wait(uint64_t limit_ns, void* stream);
int read_device_error(int* flag);
int take_device_error_gemm(int* flag);
int take_device_error_search(int* flag);
int launch_ip_stats(const float* x, const float* xt, int64_t n, int d, const float* q, int64_t nq, double* out,
                    void* stream);
size_t attend_workspace_bytes(const DevState& ks, int H, int64_t T);
// The new token of a streaming decode step: row 0 of KV head g's planes is at g * Tcap rows
// from the pointers (already offset to the appended row); k_new / v_new are [H / G][d].
struct AppendRow {
    const void* k_new;
    const void* v_new;
    int dtype;          // of k_new / v_new
    int G;              // query heads per KV head
    int64_t Tcap;
    uint8_t* kcodes;
    uint8_t* kqjl;
    float* knorms;
    float* krnorms;
    uint8_t* vcodes;
    uint8_t* vqjl;
    float* vnorms;
    float* vrnorms;
};
int launch_append_tables128(const DevState& ks, const DevState& vs, const void* q, int qdtype, int64_t count,
                            float* luts, const AppendRow& app, void* stream);
// Per-query lookup tables of the d = 128 scorers (rotated query against code groups, and
// QJL nibbles): floats per query, and a launch building them for `count` query rows.
size_t query_table_floats(const DevState& st);
int launch_query_tables128(const DevState& st, const void* q, int qdtype, int64_t count, float* luts, void* stream);
// H query heads, G of them per KV head; the planes of KV head g start at row g * Tcap
// app (optional): encode the new token of every KV head into its row before attending
int launch_attend(const DevState& ks, const DevState& vs, const void* q, int qdtype, int H,
                  int64_t T, int G, int64_t Tcap, const uint8_t* kcodes, const uint8_t* kqjl, const float* knorms,
                  const float* krnorms, const uint8_t* vcodes, const float* vnorms, float scale,
                  float* out, void* ws, size_t ws_bytes, void* stream, const AppendRow* app = nullptr);
int attend_static_scratch(void** out);
size_t search_workspace_bytes(const DevState& st, int64_t nq, int64_t n, int k);
int launch_search(const DevState& st, const void* q, int qdtype, int64_t nq,
                  const uint8_t* codes, const uint8_t* qjl, const float* norms,
                  const float* rnorms, int64_t n, int k, int64_t* idx, float* vals, void* ws,
                  size_t ws_bytes, void* stream);

}  // namespace tq
