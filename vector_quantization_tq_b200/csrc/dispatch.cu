// Chooses the encoder for a state: the tensor-core encoder where one exists for the
// configuration, else the general kernel.
#include "common.cuh"

namespace tq {

int launch_encode_generic(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, uint8_t* codes,
                          uint8_t* qjl, float* norms, float* rnorms, void* stream);

bool encode_tc_supported(const DevState& st, int dtype, int64_t n, int64_t ld);
int launch_encode_tc(const DevState& st, const void* x, int64_t n, int64_t ld, uint8_t* codes, uint8_t* qjl,
                     float* norms, float* rnorms, void* stream);

int launch_encode(const DevState& st, const void* x, int dtype, int64_t n, int64_t ld, uint8_t* codes,
                  uint8_t* qjl, float* norms, float* rnorms, void* stream) {
    if (encode_tc_supported(st, dtype, n, ld))
        return launch_encode_tc(st, x, n, ld, codes, qjl, norms, rnorms, stream);
    return launch_encode_generic(st, x, dtype, n, ld, codes, qjl, norms, rnorms, stream);
}

}  // namespace tq
