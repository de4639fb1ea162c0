/*
 * tq.h - C ABI of libtq: TurboQuant-style online vector quantization on B200 (sm_100a).
 *
 * The operations follow the TurboQuant review (Jump2Paper, arXiv 2504.19874):
 *   - Lemma 1 / Theorem 1 (MSE): a random rotation Pi makes every coordinate of a unit
 *     vector follow f_X(x) ~ (1 - x^2)^((d-3)/2); each coordinate then gets a b-bit
 *     Lloyd-Max code for f_X, and x~ = ||x|| Pi^T c[idx].
 *   - Definition 1 (QJL) and Theorem 2 (prod): the prod quantizer keeps (b-1)-bit MSE
 *     codes plus sign(S r) of the residual r and ||r||, S i.i.d. N(0,1) d x d; its
 *     inner-product estimate is unbiased.
 *   - Problem statement: Q maps R^d to B = b*d bits; Q^{-1} reconstructs.
 * and the AI Trends summary of the TurboQuant video (chapter "L2 normalize + RHT
 * matrix": store the norm, normalise, rotate by a randomized Hadamard transform whose
 * inverse is its transpose).
 *
 * Conventions for every call:
 *   - Every function returns an int status (TQ_OK = 0). Nothing is thrown across the ABI.
 *     Arguments are validated before any launch; on an error nothing is launched and
 *     no output is touched. tq_status_string() gives the text.
 *   - Pointers named h_* are host pointers; every other buffer pointer is a device
 *     pointer on the state's device. The caller owns all data buffers and workspaces; the
 *     library owns tq_state and tq_split objects (free with tq_state_destroy /
 *     tq_split_destroy). Device memory is allocated only when a state or split is created;
 *     every other call works in the caller's buffers (calls that need scratch space take a
 *     workspace argument sized by a matching *_workspace query).
 *   - Device work is asynchronous on the given cudaStream_t (passed as void*; NULL is
 *     the legacy default stream). Buffers must stay valid until the stream reaches it.
 *   - A CUDA error seen at launch is returned as TQ_ECUDA; tq_last_cuda_error() gives
 *     the cudaError_t value of the calling thread's last such error.
 *   - Distinct states may be used from distinct threads. A state is read-only after
 *     creation, so concurrent calls on one state are safe as long as their output
 *     buffers and workspaces differ.
 *
 * Data layout (structure of arrays, n vectors):
 *   codes   uint8 [n][code_bytes], code_bytes = ceil(b_mse * d / 8): each vector's
 *           codes form one LSB-first bit stream, code j in bits [j*b_mse, j*b_mse+b_mse)
 *           (bit i of byte k is stream bit 8k+i). b_mse = b (MSE) or b-1 (prod).
 *   qjl     uint8 [n][d/8] (prod only): bit j = 1 iff (S r)_j >= 0.
 *   norms   float [n]: ||x||.     rnorms  float [n] (prod only): ||r|| of the unit vector.
 *   vectors fp32 or bf16 rows of d elements, row stride ld elements (ld >= d); rows must
 *           start on 16-byte boundaries (ld*elem_size and the base pointer multiples of 16).
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------------------- */
#define TQ_OK            0
#define TQ_EINVAL        1  /* a null pointer, size, stride, alignment or value is invalid */
#define TQ_EUNSUPPORTED  2  /* valid but not supported here (e.g. RHT with d not a power of 2) */
#define TQ_ENOMEM        3  /* host or device allocation failed, or a workspace is too small */
#define TQ_ECUDA         4  /* the CUDA runtime returned an error */
#define TQ_EDEVICE       5  /* a kernel reported an error through its status word */

/* ---- enums --------------------------------------------------------------------------- */
#define TQ_MSE        0     /* TurboQuant_mse: b-bit codes + ||x||                          */
#define TQ_PROD       1     /* TurboQuant_prod: (b-1)-bit codes + QJL signs + ||x|| + ||r|| */
#define TQ_ROT_DENSE  0     /* Pi = Haar-random orthogonal matrix (QR of a Gaussian matrix)  */
#define TQ_ROT_RHT    1     /* Pi = H_d diag(eps) / sqrt(d), Sylvester Hadamard H_d          */
#define TQ_F32        0
#define TQ_BF16       1

/*
 * Host utilities (no device work): the draws and the rotation that tq_state_create uses
 * when it is given no draws, so that a caller can reproduce or inspect them.
 *   tq_draw_gaussian  count N(0,1) draws of Philox4x32-10 keyed by seed (Box-Muller).
 *   tq_draw_signs     count signs (+1/-1) of Philox4x32-10 keyed by seed.
 *   tq_haar_rotation  Pi = Q diag(sign(diag R)) from the Householder QR of the row-major
 *                     d x d matrix h_g, in fp64 (before any rounding to mat_dtype).
 * Errors: TQ_EINVAL for NULL pointers, d < 2, or a singular h_g.
 */
int tq_draw_gaussian(uint64_t seed, size_t count, double* h_out);
int tq_draw_signs(uint64_t seed, size_t count, int8_t* h_out);
int tq_haar_rotation(int d, const double* h_g, double* h_pi);

/* Which host copy tq_state_copy() returns. */
#define TQ_FIELD_CENTROIDS 0  /* 2^b_mse fp64 centroids (ascending)                */
#define TQ_FIELD_BOUNDS    1  /* 2^b_mse - 1 fp64 boundaries                       */
#define TQ_FIELD_PI        2  /* d*d row-major Pi, the values stored on the device */
#define TQ_FIELD_SIGNS     3  /* d RHT signs (+1/-1)                               */
#define TQ_FIELD_S         4  /* d*d row-major S, the values stored on the device  */

typedef struct tq_params {
    int32_t d;          /* dimension, 2 <= d; kernels: d in {32,64,128,256,512,1024,1536,2048} */
    int32_t b;          /* bits per coordinate: MSE 1..8, prod 1..9 (prod b=1 is pure QJL)    */
    int32_t mode;       /* TQ_MSE or TQ_PROD                                                  */
    int32_t rot;        /* TQ_ROT_DENSE or TQ_ROT_RHT (d a power of two)                       */
    int32_t mat_dtype;  /* device storage of dense Pi and of S: TQ_F32 or TQ_BF16              */
    int32_t device;     /* CUDA device ordinal that holds the state                           */
    uint64_t seed_pi;   /* Philox key used when no rotation draws are supplied                 */
    uint64_t seed_s;    /* Philox key used when S is not supplied                              */
} tq_params;

typedef struct tq_state tq_state;

/* Text of a status code (static string, never NULL). */
const char* tq_status_string(int status);

/* cudaError_t value of the calling thread's last TQ_ECUDA (0 if none). */
int tq_last_cuda_error(void);

/*
 * Synchronise `device` and report kernel-side errors: TQ_EDEVICE if a kernel of this
 * library gave up a bounded wait (it then recorded an error word and returned without
 * finishing); the word is cleared by this call. TQ_OK otherwise; TQ_ECUDA on a CUDA error.
 */
int tq_device_status(int device);

/*
 * Exercise the failure path of the bounded waits without a fault: on `device` (default
 * stream) a kernel waits on an mbarrier phase that nothing completes, gives up after
 * limit_us (1 .. 1e6 microseconds) and records the kernel error word. The next
 * tq_device_status(device) then returns TQ_EDEVICE (and clears the word); the context stays
 * usable. Returns the launch status.
 */
int tq_check_error_path(int device, uint32_t limit_us);

/* Library version as major*10000 + minor*100 + patch. */
int tq_version(void);

/*
 * Lloyd-Max codebook of the Lemma-1 law f_X for dimension d and b bits (host only, fp64).
 * Jump2Paper review, Theorem 1 (MSE): continuous 1-D k-means on f_X; the optimal MSE is
 * D_mse = d * C(f_X, b). Writes 2^b centroids (ascending; antisymmetric about 0), 2^b-1
 * boundaries (midpoints) and D_mse. Any output pointer may be NULL.
 * Errors: TQ_EINVAL if d < 2 or b outside 1..8.
 */
int tq_build_codebook(int d, int b, double* h_centroids, double* h_bounds, double* h_dmse);

/*
 * Create a state: codebook, rotation, and (prod) the QJL matrix S, copied to the device.
 *   h_gauss_pi  TQ_ROT_DENSE: d*d row-major N(0,1) draws G; Pi = Q diag(sign(diag R)) from
 *               the Householder QR of G (Jump2Paper: the paper's rotation is a QR rotation).
 *               NULL: G is drawn from Philox4x32-10 keyed by seed_pi (Box-Muller).
 *   h_signs     TQ_ROT_RHT: d signs (+1/-1). NULL: drawn from Philox keyed by seed_pi.
 *   h_s         TQ_PROD: d*d row-major S (Definition 1). NULL: drawn from Philox keyed by seed_s.
 * Pi and S are rounded once to mat_dtype; those stored values define the transform.
 * Pointers that the mode does not use are ignored. The state is owned by the caller and
 * freed with tq_state_destroy().
 * Errors: TQ_EINVAL (bad params / NULL out), TQ_EUNSUPPORTED (RHT with d not a power of 2,
 * or d not supported by the kernels), TQ_ENOMEM, TQ_ECUDA.
 */
int tq_state_create(const tq_params* p, const double* h_gauss_pi, const int8_t* h_signs,
                    const double* h_s, tq_state** out);

/* Free a state and its device memory (NULL is allowed). */
int tq_state_destroy(tq_state* st);

/* Copy of the parameters the state was created with. */
int tq_state_params(const tq_state* st, tq_params* out);

/* Bits of MSE code per coordinate (b or b-1), and D_mse of that codebook. */
int tq_state_codebook_info(const tq_state* st, int* b_mse, double* dmse);

/* Host copy of one field as fp64 (see TQ_FIELD_*). `count` is the capacity of h_out in
 * elements; TQ_EINVAL if it is smaller than the field or the field is absent. */
int tq_state_copy(const tq_state* st, int field, double* h_out, size_t count);

/* Serialise a state into h_buf (checkpoint). With h_buf NULL, *bytes receives the size.
 * Errors: TQ_ENOMEM if *bytes is smaller than needed (then *bytes is set to the size). */
int tq_state_export(const tq_state* st, void* h_buf, size_t* bytes);

/* Rebuild a state from tq_state_export() output on `device` (-1: the exported device). */
int tq_state_import(const void* h_buf, size_t bytes, int device, tq_state** out);

/* Per-vector plane widths in bytes: codes (ceil(b_mse*d/8)) and qjl (d/8 or 0). */
int tq_code_layout(const tq_state* st, size_t* code_bytes, size_t* qjl_bytes);

/*
 * Workspace bytes that tq_quantize_mse / tq_quantize_prod need for n vectors of dtype with
 * row stride ld (0 when the configuration needs none). Only the d >= 512 tensor-core encoders
 * (bf16 input with dense bf16 Pi, or with the randomized Hadamard rotation, prod) need one:
 * between their two passes each vector keeps a bf16 pair per coordinate of its residual and
 * one partial norm per 256 coordinates, (4 d + 4 d / 256) bytes, for up to 65536 vectors at a
 * time. A smaller workspace (at least the size for min(n, 128) vectors) is accepted and makes
 * the encoder take more passes; this call returns the size that gives the fewest.
 */
int tq_quantize_workspace(const tq_state* st, int dtype, int64_t n, int64_t ld, size_t* bytes);

/*
 * TurboQuant_mse encode of n vectors x (dtype TQ_F32 / TQ_BF16, row stride ld elements):
 * norms[i] = ||x_i||, y = Pi x_i / ||x_i||, codes = b-bit Lloyd-Max cell of each y_j
 * (the upper cell on a tie), packed as in the layout above. The state must be TQ_MSE.
 * workspace: device memory of ws_bytes (see tq_quantize_workspace; 256-byte aligned; may be
 * NULL when that size is 0). The library allocates nothing.
 * n = 0 is a no-op. Errors: TQ_EINVAL, TQ_ENOMEM (workspace below the minimum), TQ_ECUDA.
 */
int tq_quantize_mse(const tq_state* st, const void* x, int dtype, int64_t n, int64_t ld,
                    uint8_t* codes, float* norms, void* workspace, size_t ws_bytes, void* stream);

/*
 * TurboQuant_prod encode (Jump2Paper, Theorem 2): (b-1)-bit MSE codes of y = Pi x/||x||,
 * residual r = y - c[idx] (rotated domain), rnorms[i] = ||r||, qjl bits of sign(S r).
 * The state must be TQ_PROD. A zero vector stores norm 0, the codes of y = 0, r = 0.
 * workspace as for tq_quantize_mse.
 */
int tq_quantize_prod(const tq_state* st, const void* x, int dtype, int64_t n, int64_t ld,
                     uint8_t* codes, uint8_t* qjl, float* norms, float* rnorms, void* workspace,
                     size_t ws_bytes, void* stream);

/*
 * Reconstruction Q^{-1}: out[i] = ||x|| Pi^T (c[idx] + ||r|| sqrt(pi/2)/d S^T (2z - 1))
 * (the QJL term only for prod; qjl and rnorms are ignored for MSE and may be NULL).
 * out is fp32 [n][d], row stride d.
 */
int tq_dequant(const tq_state* st, const uint8_t* codes, const uint8_t* qjl,
               const float* norms, const float* rnorms, int64_t n, float* out, void* stream);

/*
 * Workspace bytes that tq_score needs for groups * nq queries: the per-query lookup tables of
 * the table scorer (d = 32, 64, 96, 128, 256 with 1 to 4 code bits), built once per query;
 * 0 for the other configurations, whose kernel prepares each query in shared memory.
 */
int tq_score_workspace(const tq_state* st, int64_t groups, int64_t nq, size_t* bytes);

/*
 * Inner-product estimates <q, x~> straight from the packed codes, grouped:
 *   queries q [groups][nq][d] (dtype TQ_F32/TQ_BF16, contiguous rows),
 *   keys (codes/qjl/norms/rnorms) [groups][n],
 *   scores fp32 [groups][nq][n]: scores[g][i][k] = <q[g][i], x~[g][k]>.
 * Computed through the rotated query q' = Pi q and u = S q':
 *   <q, x~> = ||x|| ( sum_j q'_j c[idx_j] + ||r|| sqrt(pi/2)/d sum_j u_j (2 z_j - 1) ).
 * groups = 1 is plain all-pairs scoring; groups = heads with nq = 1 is one decode query
 * per head against that head's keys.
 * workspace: at least tq_score_workspace() bytes of device memory, 256-byte aligned (NULL
 * allowed when that size is 0). Errors: TQ_ENOMEM if ws_bytes is too small.
 */
int tq_score(const tq_state* st, const void* q, int qdtype, int64_t groups, int64_t nq,
             const uint8_t* codes, const uint8_t* qjl, const float* norms, const float* rnorms,
             int64_t n, float* scores, void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes that tq_attend_decode needs for H heads and T tokens. */
int tq_attend_workspace(const tq_state* ks, const tq_state* vs, int H, int64_t T, size_t* bytes);

/*
 * One decode step of attention over a compressed cache (per head h, T tokens):
 *   s_t = scale * <q_h, k~_t>,  p = softmax(s),  out_h = sum_t p_t v~_t.
 * K is compressed by `ks` (MSE or prod), V by `vs` (MSE). Both states must have the same d.
 * Planes are [H][T] (token-major within a head); q is [H][d] (TQ_F32/TQ_BF16); out fp32 [H][d].
 * The value sum is accumulated in the rotated domain and Pi_V^T is applied once per head.
 * workspace: device memory of at least tq_attend_workspace() bytes, 256-byte aligned.
 * Errors: TQ_ENOMEM if ws_bytes is too small.
 */
int tq_attend_decode(const tq_state* ks, const tq_state* vs, const void* q, int qdtype, int H,
                     int64_t T, const uint8_t* kcodes, const uint8_t* kqjl, const float* knorms,
                     const float* krnorms, const uint8_t* vcodes, const float* vnorms,
                     float scale, float* out, void* workspace, size_t ws_bytes, void* stream);

/*
 * tq_attend_decode without a workspace argument, for callers that cannot allocate device
 * memory: runtimes that hand all device memory to their own pool allocator and forbid
 * other allocations, and latency-critical decode loops where an allocation's cost or
 * possible failure is not acceptable. (No counterpart on the reference pages: this is an
 * interface convenience around the decode step above, with the same arguments and result.)
 * The scratch that tq_attend_decode takes from its workspace (the split partials and, for
 * d = 128 keys at 2 to 4 bits, the per-head query tables) goes to a fixed device array of
 * 4 MiB inside the library, which every GPU that loads the library holds until the process
 * exits; the entry point itself allocates nothing. A call is accepted when
 * tq_attend_workspace(ks, vs, H, T) <= 4 MiB and returns TQ_EUNSUPPORTED otherwise (nothing
 * is launched). That size grows with H and d, and the number of token splits grows with
 * the device's SM count, so the largest accepted H differs between GPUs; query
 * tq_attend_workspace on the device in use.
 * All calls on a device share the array and it keeps the last call's contents, so calls
 * whose work overlaps on the GPU (concurrent streams or threads) race and must be
 * serialised by the caller. The first call on each device looks up the array's device
 * address with that device current; make that first call before any stream capture.
 */
int tq_attend_decode_noalloc(const tq_state* ks, const tq_state* vs, const void* q, int qdtype, int H,
                             int64_t T, const uint8_t* kcodes, const uint8_t* kqjl, const float* knorms,
                             const float* krnorms, const uint8_t* vcodes, const float* vnorms,
                             float scale, float* out, void* stream);

/*
 * Distortion and inner-product error statistics of reconstructions, for the distortion /
 * bias sweep (Jump2Paper review: Theorem 1 gives D_mse = E||x - x~||^2; Theorem 2 gives an
 * unbiased <q, x~> for prod; the motivation paragraph gives the 2/pi slope of the 1-bit MSE
 * quantizer). Inputs fp32 row-major: x and xt [n][d] (original and reconstruction, e.g. from
 * tq_dequant), q [nq][d]. Writes 6 fp64 sums to the device buffer `out`:
 *   out[0] = sum_i ||x_i - xt_i||^2     out[1] = sum_i ||x_i||^2
 *   out[2] = sum_{q,i} e                out[3] = sum e^2          with a = <q, x_i>,
 *   out[4] = sum a b                    out[5] = sum a^2               b = <q, xt_i>, e = b - a.
 * `out` is zeroed first on `stream`. d <= 256 (TQ_EUNSUPPORTED above). The fp64 sums are
 * accumulated with atomics, so their last bits can vary from run to run.
 */
int tq_ip_stats(const float* x, const float* xt, int64_t n, int d, const float* q, int64_t nq, double* out,
                void* stream, int device);

/* Workspace bytes that tq_search_topk needs. */
int tq_search_workspace(const tq_state* st, int64_t nq, int64_t n, int k, size_t* bytes);

/*
 * Top-k database vectors by estimated inner product for each of nq queries
 * (Jump2Paper: nearest-neighbour search over compressed vectors). Planes as tq_score with
 * groups = 1. idx int64 [nq][k] and vals fp32 [nq][k], best first; ties to the lower index.
 * 1 <= k <= 64 and k <= n.
 */
int tq_search_topk(const tq_state* st, const void* q, int qdtype, int64_t nq,
                   const uint8_t* codes, const uint8_t* qjl, const float* norms,
                   const float* rnorms, int64_t n, int k, int64_t* idx, float* vals,
                   void* workspace, size_t ws_bytes, void* stream);

/*
 * Decode step with grouped queries: H query heads, G of them per KV head (H % G == 0;
 * query head h reads KV head h / G). The planes of KV head g are rows g*Tcap .. g*Tcap+T-1
 * (Tcap >= T: a cache with room to grow); q [H][d], out fp32 [H][d]. Workspace as
 * tq_attend_workspace(ks, vs, H, T). G = 1 and Tcap = T is tq_attend_decode.
 */
int tq_attend_decode_grouped(const tq_state* ks, const tq_state* vs, const void* q, int qdtype, int H, int G,
                             int64_t T, int64_t Tcap, const uint8_t* kcodes, const uint8_t* kqjl,
                             const float* knorms, const float* krnorms, const uint8_t* vcodes, const float* vnorms,
                             float scale, float* out, void* workspace, size_t ws_bytes, void* stream);

/*
 * Streaming decode step (the "online" setting: one new token per step): encode the new key
 * and value of every KV head (k_new, v_new: [H/G][d], dtype kvdtype, contiguous) into row T
 * of that head's planes (0 <= T < Tcap), then run tq_attend_decode_grouped over the T + 1
 * tokens. Both launches go on `stream` in that order. Workspace as
 * tq_attend_workspace(ks, vs, H, T + 1).
 */
int tq_attend_append_decode(const tq_state* ks, const tq_state* vs, const void* q, int qdtype, int H, int G,
                            const void* k_new, const void* v_new, int kvdtype, int64_t T, int64_t Tcap,
                            uint8_t* kcodes, uint8_t* kqjl, float* knorms, float* krnorms, uint8_t* vcodes,
                            float* vnorms, float scale, float* out, void* workspace, size_t ws_bytes, void* stream);

/* ---- prefix coding of the indices -----------------------------------------------------
 * TurboQuant review (Jump2Paper), limitations: an optimal prefix code on the b = 4 indices
 * averages about 3.8 bits. The code is Huffman's code of the one-coordinate index law under
 * Lemma 1 (cell probabilities of the state's Lloyd-Max boundaries), fixed per state: ties
 * in the merges go to the lower node id (leaves 0..L-1, merged nodes L, L+1, ... in creation
 * order); codewords are canonical. Stream layout: each vector's codes in coordinate order,
 * each codeword first bit (most significant) first, vectors back to back, bit j of the
 * stream = bit j % 8 of byte j / 8; offsets[k] = first bit of vector k, offsets[n] = total.
 */

/* Codeword lengths and canonical codewords (host arrays of 2^b_mse), and the mean length in
   bits per coordinate under the index law. Any output may be NULL. */
int tq_entropy_table(const tq_state* st, int* h_lengths, uint32_t* h_words, double* h_mean_bits);

/* Stream capacity in bytes that tq_entropy_encode requires for n vectors (the longest
   codeword for every coordinate, in whole 32-bit words, plus 16 bytes). */
int tq_entropy_max_bytes(const tq_state* st, int64_t n, size_t* bytes);

/* Workspace bytes that tq_entropy_encode needs for n vectors. */
int tq_entropy_workspace(const tq_state* st, int64_t n, size_t* bytes);

/*
 * Encode the packed codes planes [n][code_bytes] (16-byte aligned) into `stream` (device,
 * 4-byte aligned, `capacity` >= tq_entropy_max_bytes; zeroed here first) and offsets
 * (device uint64 [n + 1], 8-byte aligned). workspace: >= tq_entropy_workspace bytes,
 * 256-byte aligned. TQ_ENOMEM if capacity or workspace is too small.
 */
int tq_entropy_encode(const tq_state* st, const uint8_t* codes, int64_t n, uint64_t* offsets, uint8_t* stream,
                      size_t capacity, void* workspace, size_t ws_bytes, void* cuda_stream);

/* Decode n vectors of `stream` (offsets as written by tq_entropy_encode) back into packed
   codes planes [n][code_bytes] (16-byte aligned). */
int tq_entropy_decode(const tq_state* st, const uint8_t* stream, const uint64_t* offsets, int64_t n, uint8_t* codes,
                      void* cuda_stream);

/* ---- outlier-channel split ------------------------------------------------------------
 * TurboQuant review (Jump2Paper), experiment settings ("KV bit settings": 2.5 and 3.5 bits
 * with outlier and non-outlier channels separated; "outlier handling": 32 of 128 channels at
 * 3 bits, 96 at 2 bits). A split quantizes the m channels listed in `channels` with the
 * state `outer` (dimension m) and the other d - m channels, in ascending order, with `inner`
 * (dimension d - m): two independent quantizers, each with its own rotation, codebook, QJL
 * matrix and norms. The reconstruction puts each group back into its channels, so an
 * estimate <q, x~> is the sum of the two groups' estimates.
 */
typedef struct tq_split tq_split;

/* Device planes of one channel group (qjl and rnorms NULL for an MSE state). */
typedef struct tq_planes {
    uint8_t* codes;
    uint8_t* qjl;
    float* norms;
    float* rnorms;
} tq_planes;

/*
 * Create a split of d = outer.d + inner.d channels. h_channels: host array of m = outer.d
 * distinct channel indices in [0, d), ascending. Both states must have the same mode and
 * device; the split keeps pointers to them (they must outlive it) and a device copy of the
 * two channel maps. TQ_EINVAL on any mismatch.
 */
int tq_split_create(const tq_state* outer, const tq_state* inner, const int32_t* h_channels, int m,
                    tq_split** out);

/* Free a split (NULL is allowed). */
void tq_split_destroy(tq_split* sp);

/*
 * Quantize n rows x [n][ld] (dtype TQ_F32/TQ_BF16, row stride ld >= d elements, 16-byte
 * aligned base and stride): the outer group into `outer`'s planes [n], the inner group into
 * `inner`'s planes [n]. Plane pointers 16-byte aligned, as for tq_quantize_*.
 */
int tq_split_quantize(const tq_split* sp, const void* x, int dtype, int64_t n, int64_t ld,
                      const tq_planes* outer, const tq_planes* inner, void* stream);

/* Reconstruct rows out fp32 [n][d] (16-byte aligned) from both groups' planes. */
int tq_split_dequant(const tq_split* sp, const tq_planes* outer, const tq_planes* inner, int64_t n,
                     float* out, void* stream);

/* Workspace bytes that tq_split_score needs: the queries' two channel groups, gathered, and
   the groups' score tables. */
int tq_split_score_workspace(const tq_split* sp, int qdtype, int64_t groups, int64_t nq, size_t* bytes);

/*
 * Estimates as tq_score (queries [groups][nq][d], planes [groups][n], scores fp32
 * [groups][nq][n]), summed over the two groups. workspace: at least tq_split_score_workspace()
 * bytes, 256-byte aligned. Errors: TQ_ENOMEM if ws_bytes is too small.
 */
int tq_split_score(const tq_split* sp, const void* q, int qdtype, int64_t groups, int64_t nq,
                   const tq_planes* outer, const tq_planes* inner, int64_t n, float* scores,
                   void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes that tq_split_attend_decode needs for H heads and T tokens. */
int tq_split_attend_workspace(const tq_split* ks, const tq_split* vs, int H, int64_t T, size_t* bytes);

/*
 * One decode step of attention (as tq_attend_decode) over channel-split caches: K split `ks`
 * (MSE or prod groups), V split `vs` (MSE groups), both over the same d channels (their
 * outlier lists may differ). s_t = scale * (sum over the K groups of <q_group, k~_t,group>),
 * p = softmax(s), out_h = sum_t p_t v~_t with each V group reconstructed in its own
 * channels. Planes [H][T] per group; q [H][d]; out fp32 [H][d]; workspace of at least
 * tq_split_attend_workspace() bytes, 256-byte aligned.
 */
int tq_split_attend_decode(const tq_split* ks, const tq_split* vs, const void* q, int qdtype, int H, int64_t T,
                           const tq_planes* k_outer, const tq_planes* k_inner, const tq_planes* v_outer,
                           const tq_planes* v_inner, float scale, float* out, void* workspace,
                           size_t ws_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H */
