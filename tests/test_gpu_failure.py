"""Failure detection without a GPU fault: a bounded wait that runs out records the kernel
error word, tq_device_status reports TQ_EDEVICE once (and clears it), and the context keeps
working (an encode afterwards matches the same encode before)."""
import numpy as np
import pytest

import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu
tq = pytest.importorskip("vector_quantization_tq_b200")


def test_expired_wait_is_reported_and_the_context_survives():
    st = tq.State(128, 3, tq.PROD, tq.ROT_RHT, tq.BF16, signs=synth.rht_signs(128), s=synth.gaussian_matrix(128, 1))
    bits = synth.kv_prefill_batch(1, 777, 128, seed=9)[0]
    x = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)

    def encode():
        planes = st.empty_planes(777)
        tq.quantize_prod(st, x, *planes)
        torch.cuda.synchronize()
        return [p.cpu().numpy() for p in planes]

    before = encode()
    tq.device_status(0)
    assert tq.lib().tq_check_error_path(0, 2000) == 0
    assert tq.lib().tq_device_status(0) == 5          # TQ_EDEVICE
    assert tq.lib().tq_device_status(0) == 0          # read once, then cleared
    after = encode()
    tq.device_status(0)
    for a, b in zip(before, after):
        np.testing.assert_array_equal(a, b)
