// Host-side random draws and the QR rotation for state creation (fp64, one-off).
//
// Random numbers: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers:
// as easy as 1, 2, 3", SC 2011), a counter-based generator; normal deviates by the
// Box-Muller transform (Box and Muller, 1958). Draw i of a stream uses counter
// (i/2, 0, 0, 0) with key (seed low 32 bits, seed high 32 bits); the four output words
// make two 53-bit uniforms u1, u2 in (0, 1], and the pair (r cos, r sin) with
// r = sqrt(-2 ln u1), angle 2 pi u2 gives draws 2(i/2) and 2(i/2)+1.
//
// Rotation: the TurboQuant review (Jump2Paper) uses a QR rotation of a Gaussian
// matrix; here Householder QR, then Pi = Q diag(sign(R_ii)) so that the factorisation
// (and with it Pi) is unique.
#include <cmath>
#include <cstring>
#include <vector>

#include "internal.h"

namespace tq {

void philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
    uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
    uint32_t k0 = key_in[0], k1 = key_in[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += W0;
            k1 += W1;
        }
        uint64_t p0 = (uint64_t)M0 * c0;
        uint64_t p1 = (uint64_t)M1 * c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        c0 = n0;
        c1 = lo1;
        c2 = n2;
        c3 = lo0;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

static double uniform53(uint32_t hi, uint32_t lo) {
    // 53 random bits -> (0, 1]
    uint64_t v = ((uint64_t)(hi >> 5) << 26) | (lo >> 6);
    return ((double)v + 1.0) * (1.0 / 9007199254740992.0);
}

void philox_gaussian(uint64_t seed, size_t count, double* out) {
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    for (size_t i = 0; i < count; i += 2) {
        const uint32_t ctr[4] = {(uint32_t)(i / 2), (uint32_t)((i / 2) >> 32), 0u, 0u};
        uint32_t r[4];
        philox4x32_10(ctr, key, r);
        double u1 = uniform53(r[0], r[1]);
        double u2 = uniform53(r[2], r[3]);
        double rad = std::sqrt(-2.0 * std::log(u1));
        double ang = 2.0 * M_PI * u2;
        out[i] = rad * std::cos(ang);
        if (i + 1 < count) out[i + 1] = rad * std::sin(ang);
    }
}

void philox_signs(uint64_t seed, size_t count, int8_t* out) {
    const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    for (size_t i = 0; i < count; ++i) {
        const uint32_t ctr[4] = {(uint32_t)i, (uint32_t)(i >> 32), 1u, 0u};
        uint32_t r[4];
        philox4x32_10(ctr, key, r);
        out[i] = (r[0] & 1u) ? (int8_t)-1 : (int8_t)1;
    }
}

int haar_from_gaussian(int d, const double* g, double* pi_out) {
    // Householder QR of G (row-major d x d). A is overwritten by R; the reflectors are kept.
    std::vector<double> A(g, g + (size_t)d * d);
    std::vector<double> V((size_t)d * d, 0.0);   // V[k][i] = reflector k, entries i >= k
    std::vector<double> rdiag(d);
    std::vector<double> w(d);
    for (int k = 0; k < d; ++k) {
        double nrm = 0.0;
        for (int i = k; i < d; ++i) nrm += A[(size_t)i * d + k] * A[(size_t)i * d + k];
        nrm = std::sqrt(nrm);
        if (nrm == 0.0) return TQ_EINVAL;   // singular draw
        double x0 = A[(size_t)k * d + k];
        double alpha = (x0 >= 0.0) ? -nrm : nrm;
        double* v = &V[(size_t)k * d];
        for (int i = k; i < d; ++i) v[i] = A[(size_t)i * d + k];
        v[k] -= alpha;
        double vn = 0.0;
        for (int i = k; i < d; ++i) vn += v[i] * v[i];
        vn = std::sqrt(vn);
        for (int i = k; i < d; ++i) v[i] /= vn;
        // A[k:, k:] -= 2 v (v^T A[k:, k:])
        for (int j = k; j < d; ++j) w[j] = 0.0;
        for (int i = k; i < d; ++i) {
            const double vi = v[i];
            const double* row = &A[(size_t)i * d];
            for (int j = k; j < d; ++j) w[j] += vi * row[j];
        }
        for (int i = k; i < d; ++i) {
            const double vi2 = 2.0 * v[i];
            double* row = &A[(size_t)i * d];
            for (int j = k; j < d; ++j) row[j] -= vi2 * w[j];
        }
        rdiag[k] = alpha;
    }
    // Q = H_0 H_1 ... H_{d-1}: apply the reflectors to I from the last one back.
    std::vector<double> Q((size_t)d * d, 0.0);
    for (int i = 0; i < d; ++i) Q[(size_t)i * d + i] = 1.0;
    for (int k = d - 1; k >= 0; --k) {
        const double* v = &V[(size_t)k * d];
        for (int j = 0; j < d; ++j) w[j] = 0.0;
        for (int i = k; i < d; ++i) {
            const double vi = v[i];
            const double* row = &Q[(size_t)i * d];
            for (int j = 0; j < d; ++j) w[j] += vi * row[j];
        }
        for (int i = k; i < d; ++i) {
            const double vi2 = 2.0 * v[i];
            double* row = &Q[(size_t)i * d];
            for (int j = 0; j < d; ++j) row[j] -= vi2 * w[j];
        }
    }
    // Pi = Q diag(sign(R_kk))
    for (int i = 0; i < d; ++i)
        for (int k = 0; k < d; ++k) pi_out[(size_t)i * d + k] = Q[(size_t)i * d + k] * (rdiag[k] < 0.0 ? -1.0 : 1.0);
    return TQ_OK;
}

float bf16_round_host(float x) {
    uint32_t u;
    std::memcpy(&u, &x, 4);
    if ((u & 0x7F800000u) == 0x7F800000u) return x;   // inf / nan unchanged
    u = (u + 0x7FFFu + ((u >> 16) & 1u)) & 0xFFFF0000u;
    float r;
    std::memcpy(&r, &u, 4);
    return r;
}

// Paley's Hadamard matrix of order 12 (q = 11, q = 3 mod 4): H = I + [[0, 1^T], [-1, Q]],
// Q[i][j] = chi(j - i) with chi the quadratic character of GF(11). rows[a] has bit c set
// where H[a][c] = -1.
void paley_hadamard12_rows(uint32_t rows[12]) {
    constexpr int q = 11;
    int chi[q] = {0};
    for (int a = 1; a < q; ++a) chi[a] = -1;
    for (int x = 1; x < q; ++x) chi[(x * x) % q] = 1;
    for (int a = 0; a < 12; ++a) {
        rows[a] = 0;
        for (int c = 0; c < 12; ++c) {
            int v;
            if (a == 0) v = (c == 0) ? 1 : 1;                       // I + border row of ones
            else if (c == 0) v = -1;                                 // border column of -1
            else v = chi[((c - 1) - (a - 1) + q) % q] + (a == c ? 1 : 0);
            if (v < 0) rows[a] |= 1u << c;
        }
    }
}

}  // namespace tq
