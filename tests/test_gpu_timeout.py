"""Failure detection on the GPU without a fault: the library's bounded
device-side wait gives up after the host-set limit, the host reads
TL_ETIMEOUT, and the CUDA context stays usable.

The wait that runs out is the one of tl_wait_probe: a single thread waits,
through the same bounded-wait code the tensor-core kernels use, on an
mbarrier that nothing ever arrives on ("a flag that nothing sets"); no copy
or MMA is in flight while it waits."""
import time

import pytest
import torch

import transformer_layer_pre_b200 as tlp
from parity import check_layer, run_gpu, run_oracle
from transformer_layer_pre_b200.synthetic import Workload, make_inputs

pytestmark = pytest.mark.gpu

TL_ETIMEOUT = 5
SMALL = Workload("timeout-check-f16", 2, 64, 128, 2, 256, "f16", 0.1, 0.1, lengths=(40, 64))


def test_bounded_wait_gives_up_and_the_context_survives():
    torch.cuda.init()
    tlp.device_check()                       # nothing pending before
    limit_ns = 20_000_000                    # 20 ms
    tlp.set_wait_limit(limit_ns)
    try:
        t0 = time.perf_counter()
        tlp.wait_probe()
        with pytest.raises(tlp.TlError) as ei:
            tlp.device_check()
        waited = time.perf_counter() - t0
        assert ei.value.status == TL_ETIMEOUT
        assert 0.9 * limit_ns * 1e-9 <= waited < 1.5, waited   # gave up after the limit, not the 2 s default
    finally:
        tlp.set_wait_limit(0)
    tlp.device_check()                       # the flag was cleared by the read
    # the context still runs the layer, and correctly
    inp = make_inputs(SMALL)
    check_layer(run_gpu(inp), run_oracle(inp), run_oracle(inp, storage_rounded=True), "f16")
    tlp.device_check()
