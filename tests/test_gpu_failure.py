"""Failure detection without a GPU fault: every wait inside the kernels is bounded, and a
wait that runs out records a status for the host instead of hanging.

qlora_selftest_wait_timeout launches one kernel whose only wait is on an mbarrier that
nothing arrives at. The wait must give up after the library's limit (2 s), the host
must read QLORA_ERR_TIMEOUT from the device error word, and the context must stay usable."""
import time

import numpy as np
import pytest
import torch

from bit_nf4_quantized_unpack_b200 import inputs, qlora
from oracle import nf4_oracle as O
from tests.gpu_util import need_gpu

pytestmark = pytest.mark.gpu

TIMEOUT = 7  # QLORA_ERR_TIMEOUT


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    need_gpu()
    assert qlora.qlora_device_error() == 0
    try:
        torch.cuda.synchronize()
        t0 = time.monotonic()
        qlora.qlora_selftest_wait_timeout()
        torch.cuda.synchronize()
        waited = time.monotonic() - t0
        assert 1.9 < waited < 60.0, waited           # the 2 s limit, then the kernel exits
        assert qlora.qlora_device_error(clear=False) == TIMEOUT
        assert "timed out" in qlora.lib().qlora_last_error().decode()
    finally:
        qlora.qlora_device_error(clear=True)
    assert qlora.qlora_device_error() == 0           # cleared once read
    # the same context still computes: a quantization and its double dequantization,
    # bit for bit against the oracle
    rng = np.random.default_rng(31)
    W = inputs.to_bf16_values(rng.normal(0, 0.02, (64, 1024)).astype(np.float32))
    q = qlora.qlora_quantize_nf4_dq(torch.from_numpy(W).cuda().to(torch.bfloat16))
    wd = qlora.qlora_dequant(q)
    torch.cuda.synchronize()
    ref = O.quantize_nf4_dq(W)
    assert np.array_equal(q.codes.cpu().numpy(), ref["codes"])
    got = wd.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, O.bf16_bits(O.double_dequant(ref)))
    assert qlora.qlora_device_error() == 0
