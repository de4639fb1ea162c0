// Prefix coding of the packed codebook indices on the GPU (TurboQuant review, Jump2Paper,
// limitations paragraph: an optimal prefix code on the b = 4 indices averages about 3.8
// bits). Encode: per-vector code lengths and per-block totals; an exclusive scan of the
// totals; then each vector's offset (block scan) and its bits, written with word-wise ORs
// into a zeroed stream (neighbouring vectors share the boundary words). Decode: one thread
// per vector walks its bits with the canonical (first, count, start) tables and repacks the
// fixed-width codes.
#include "common.cuh"

namespace tq {
namespace {

constexpr int kEThreads = 256;
constexpr int kEPer = 4;                        // vectors per thread
constexpr int kEBlock = kEThreads * kEPer;      // vectors per block

// Code j of a packed LSB-first row of b-bit codes, read through a 64-bit window.
struct CodeReader {
    const uint32_t* row;
    uint64_t buf = 0;
    int have = 0, wi = 0;
    __device__ explicit CodeReader(const uint32_t* r) : row(r) {}
    __device__ __forceinline__ uint32_t next(int b) {
        if (have < b) {
            buf |= (uint64_t)__ldg(row + wi++) << have;
            have += 32;
        }
        const uint32_t c = (uint32_t)buf & ((1u << b) - 1u);
        buf >>= b;
        have -= b;
        return c;
    }
};

__device__ __forceinline__ uint32_t vector_bits(const uint8_t* codes, int64_t v, int d, int b, int code_bytes,
                                                const uint8_t* len) {
    CodeReader rd(reinterpret_cast<const uint32_t*>(codes + v * code_bytes));
    uint32_t s = 0;
    for (int j = 0; j < d; ++j) s += len[rd.next(b)];
    return s;
}

__global__ void __launch_bounds__(kEThreads)
entropy_bits_kernel(const EntropyTable tab, const uint8_t* __restrict__ codes, int64_t n, int d, int b,
                    int code_bytes, uint32_t* __restrict__ bits, uint64_t* __restrict__ block_tot) {
    __shared__ uint8_t len[kMaxLevels];
    __shared__ uint64_t red[kEThreads / 32];
    for (int i = threadIdx.x; i < tab.L; i += kEThreads) len[i] = tab.len[i];
    __syncthreads();
    uint64_t tot = 0;
    for (int i = 0; i < kEPer; ++i) {
        const int64_t v = (int64_t)blockIdx.x * kEBlock + (int64_t)threadIdx.x * kEPer + i;
        if (v < n) {
            const uint32_t s = vector_bits(codes, v, d, b, code_bytes, len);
            bits[v] = s;
            tot += s;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = tot;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint64_t t = 0;
        for (int w = 0; w < kEThreads / 32; ++w) t += red[w];
        block_tot[blockIdx.x] = t;
    }
}

// In place exclusive scan of nb block totals (one block of 1024 threads); the grand total
// goes to offsets[n].
__global__ void __launch_bounds__(1024)
scan_totals_kernel(uint64_t* __restrict__ tot, int64_t nb, uint64_t* __restrict__ total_out) {
    __shared__ uint64_t warp_sums[32];
    __shared__ uint64_t carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t c0 = 0; c0 < nb; c0 += 1024) {
        const int64_t i = c0 + threadIdx.x;
        const uint64_t x = (i < nb) ? tot[i] : 0;
        uint64_t incl = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_sums[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            uint64_t ws = warp_sums[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint64_t y = __shfl_up_sync(0xffffffffu, ws, o);
                if (lane >= o) ws += y;
            }
            warp_sums[lane] = ws;   // inclusive over warps
        }
        __syncthreads();
        const uint64_t before = carry + (warp > 0 ? warp_sums[warp - 1] : 0) + incl - x;
        if (i < nb) tot[i] = before;
        __syncthreads();
        if (threadIdx.x == 1023) carry = before + x;
        __syncthreads();
    }
    if (threadIdx.x == 0) *total_out = carry;
}

__global__ void __launch_bounds__(kEThreads)
entropy_write_kernel(const EntropyTable tab, const uint8_t* __restrict__ codes, int64_t n, int d, int b,
                     int code_bytes, const uint32_t* __restrict__ bits, const uint64_t* __restrict__ block_off,
                     uint64_t* __restrict__ offsets, uint32_t* __restrict__ stream32) {
    __shared__ uint8_t len[kMaxLevels];
    __shared__ uint32_t rword[kMaxLevels];
    __shared__ uint64_t warp_sums[kEThreads / 32];
    for (int i = threadIdx.x; i < tab.L; i += kEThreads) {
        len[i] = tab.len[i];
        rword[i] = tab.rword[i];
    }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t v0 = (int64_t)blockIdx.x * kEBlock + (int64_t)threadIdx.x * kEPer;
    uint32_t mine[kEPer];
    uint64_t tsum = 0;
#pragma unroll
    for (int i = 0; i < kEPer; ++i) {
        mine[i] = (v0 + i < n) ? bits[v0 + i] : 0u;
        tsum += mine[i];
    }
    uint64_t incl = tsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    uint64_t before = block_off[blockIdx.x] + incl - tsum;
    for (int w = 0; w < warp; ++w) before += warp_sums[w];
    for (int i = 0; i < kEPer; ++i) {
        const int64_t v = v0 + i;
        if (v >= n) break;
        offsets[v] = before;
        // the vector's codewords, first bit first, from bit `before` on
        CodeReader rd(reinterpret_cast<const uint32_t*>(codes + v * code_bytes));
        int64_t w = (int64_t)(before >> 5);
        uint64_t acc = 0;
        int acc_bits = (int)(before & 31);
        for (int j = 0; j < d; ++j) {
            const uint32_t c = rd.next(b);
            acc |= (uint64_t)rword[c] << acc_bits;
            acc_bits += len[c];
            if (acc_bits >= 32) {
                atomicOr(stream32 + w, (uint32_t)acc);
                ++w;
                acc >>= 32;
                acc_bits -= 32;
            }
        }
        if (acc_bits > 0) atomicOr(stream32 + w, (uint32_t)acc);
        before += mine[i];
    }
}

__global__ void __launch_bounds__(kEThreads)
entropy_decode_kernel(const EntropyTable tab, const uint32_t* __restrict__ stream32,
                      const uint64_t* __restrict__ offsets, int64_t n, int d, int b, int code_bytes,
                      uint8_t* __restrict__ codes) {
    __shared__ uint32_t first[kMaxCodeLen + 2];
    __shared__ uint16_t count[kMaxCodeLen + 2];
    __shared__ uint16_t start[kMaxCodeLen + 2];
    __shared__ uint16_t sym[kMaxLevels];
    for (int i = threadIdx.x; i < kMaxCodeLen + 2; i += kEThreads) {
        first[i] = tab.first[i];
        count[i] = tab.count[i];
        start[i] = tab.start[i];
    }
    for (int i = threadIdx.x; i < tab.L; i += kEThreads) sym[i] = tab.sym[i];
    __syncthreads();
    const int64_t nwords = (int64_t)((offsets[n] + 31) >> 5);   // words holding stream bits
    for (int64_t v = (int64_t)blockIdx.x * kEThreads + threadIdx.x; v < n; v += (int64_t)gridDim.x * kEThreads) {
        const uint64_t off = offsets[v];
        int64_t w = (int64_t)(off >> 5);
        uint64_t buf = (w < nwords) ? __ldg(stream32 + w) : 0u;
        ++w;
        buf >>= (off & 31);
        int have = 32 - (int)(off & 31);
        uint32_t* out = reinterpret_cast<uint32_t*>(codes + v * code_bytes);
        uint64_t obuf = 0;
        int obits = 0, ow = 0;
        for (int j = 0; j < d; ++j) {
            uint32_t code = 0;
            uint32_t s = 0;
            for (int l = 1; l <= kMaxCodeLen; ++l) {
                if (have == 0) {
                    buf = (w < nwords) ? __ldg(stream32 + w) : 0u;
                    ++w;
                    have = 32;
                }
                code = (code << 1) | (uint32_t)(buf & 1u);
                buf >>= 1;
                --have;
                if (count[l] != 0 && code - first[l] < count[l]) {
                    s = sym[start[l] + (code - first[l])];
                    break;
                }
            }
            obuf |= (uint64_t)s << obits;
            obits += b;
            if (obits >= 32) {
                out[ow++] = (uint32_t)obuf;
                obuf >>= 32;
                obits -= 32;
            }
        }
        if (obits > 0) out[ow] = (uint32_t)obuf;
    }
}

}  // namespace

size_t entropy_ws_bytes(int64_t n) {
    const int64_t nb = (n + kEBlock - 1) / kEBlock;
    return ((size_t)n * 4 + 255) / 256 * 256 + (size_t)nb * 8;
}

int launch_entropy_encode(const DevState& st, const EntropyTable& tab, const uint8_t* codes, int64_t n,
                          uint64_t* offsets, uint8_t* stream, size_t capacity, void* ws, void* cuda_stream) {
    cudaStream_t s = (cudaStream_t)cuda_stream;
    const int64_t nb = (n + kEBlock - 1) / kEBlock;
    uint32_t* bits = reinterpret_cast<uint32_t*>(ws);
    uint64_t* tot = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(ws) + ((size_t)n * 4 + 255) / 256 * 256);
    cudaError_t e = cudaMemsetAsync(stream, 0, capacity, s);
    if (e != cudaSuccess) return (int)e;
    entropy_bits_kernel<<<(unsigned)nb, kEThreads, 0, s>>>(tab, codes, n, st.d, st.b_mse, st.code_bytes, bits, tot);
    scan_totals_kernel<<<1, 1024, 0, s>>>(tot, nb, offsets + n);
    entropy_write_kernel<<<(unsigned)nb, kEThreads, 0, s>>>(tab, codes, n, st.d, st.b_mse, st.code_bytes, bits, tot,
                                                            offsets, reinterpret_cast<uint32_t*>(stream));
    return (int)cudaGetLastError();
}

int launch_entropy_decode(const DevState& st, const EntropyTable& tab, const uint8_t* stream, const uint64_t* offsets,
                          int64_t n, uint8_t* codes, void* cuda_stream) {
    cudaStream_t s = (cudaStream_t)cuda_stream;
    const int64_t need = (n + kEThreads - 1) / kEThreads;
    const int64_t blocks = need < ((int64_t)1 << 20) ? need : ((int64_t)1 << 20);
    entropy_decode_kernel<<<(unsigned)blocks, kEThreads, 0, s>>>(tab, reinterpret_cast<const uint32_t*>(stream),
                                                                 offsets, n, st.d, st.b_mse, st.code_bytes, codes);
    return (int)cudaGetLastError();
}

}  // namespace tq
