"""Failure detection on the GPU without a fault: a bounded wait is made to run out.

fq_debug_arm_stall makes the next tensor-core launch issue no x loads, so stage A's wait
for its first tile has nothing to wait for. With a 50 ms limit the kernel must give up,
let every role leave, free its TMEM and return; the host then reads the expiry from the
handle's status word, and the same context runs the next call correctly."""

import time

import pytest
import torch

from rotation_bit_quantization_token_b200 import FlatQuant, FQError, _lib
from rotation_bit_quantization_token_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,K", [("mx_case3_32768x128x112", 300), ("per_token_int32_4096x64x64", 64)])
def test_bounded_wait_expires_and_context_survives(name, K):
    w = WORKLOADS[name].with_tokens(K)
    x, P1, P2 = (t.cuda() for t in make_inputs(w, seed=7))
    fq = FlatQuant(w.K, w.M, w.N)
    fq.set_kernel("tcgen05")

    def call():
        if w.mode == "mx":
            return fq.quantize_mx(x, P1, P2, w.dst_type_max)
        return fq.quantize_per_token(x, P1, P2, w.clip_ratio, w.out)

    ref = call()
    torch.cuda.synchronize()
    assert fq.device_status() == 0

    fq.debug_arm_stall(0.05)
    t0 = time.monotonic()
    call()
    torch.cuda.synchronize()
    elapsed = time.monotonic() - t0
    status = fq.device_status()
    assert status != 0, "the stalled launch did not report its expired wait"
    assert status & 2, f"stage A's wait for the x tile is not among the expired waits ({status:#x})"
    assert elapsed < 2.0, f"the stalled launch took {elapsed:.2f} s to give up"

    again = call()
    torch.cuda.synchronize()
    assert fq.device_status() == 0
    assert torch.equal(again[0], ref[0]) and torch.equal(again[1], ref[1])


def test_arm_stall_rejects_bad_limits():
    fq = FlatQuant(4, 32, 64)
    for bad in (0.0, -1.0, 11.0, float("nan")):
        with pytest.raises(FQError) as e:
            fq.debug_arm_stall(bad)
        assert e.value.status == _lib.FQ_ERR_INVALID
