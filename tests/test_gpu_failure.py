"""Failure detection on the GPU without faulting it: the tensor-core kernel's
bounded waits expire when its input loads are withheld (a wait that nothing
completes); the kernel records the timeout, frees its resources and exits, the
host reads DN_ERR_TIMEOUT, and the context stays usable for correct work."""
import pytest
import torch

import delta_rule_recurrent_02_b200 as dn
from delta_rule_recurrent_02_b200 import workloads as W
from _util import assert_close, oracle_prefill, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("gate", ["scalar", "per_key"])
def test_bounded_wait_timeout_is_reported_and_context_survives(cuda_device, gate):
    inp = W.gen_prefill(1, 2, 130, 128, 128, dtype="bf16", gate=gate, seed=31, s0_std=0.1)
    d = to_dev(inp)
    sc = 128 ** -0.5
    dn.dn_device_status()                      # clean start
    o = torch.full((1, 2, 130, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    S = torch.full((1, 2, 128, 128), 7.0, device="cuda")
    dn.dn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], o, S, scale=sc, path="tc_stall_test")
    with pytest.raises(dn.DNError) as ei:
        dn.dn_device_status()
    assert ei.value.status == dn.DN_ERR_TIMEOUT
    dn.dn_device_status()                      # the status word was cleared by the read
    # the same inputs on the normal path: correct results, no timeout
    o2, S2 = dn.chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], scale=sc, path="tc")
    dn.dn_device_status()
    ro, rS = oracle_prefill(inp, sc)
    assert_close(o2, ro, "bf16", "o after a timeout")
    assert_close(S2, rS, "bf16", "S_T after a timeout")
