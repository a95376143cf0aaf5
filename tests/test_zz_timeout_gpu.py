"""The bounded-wait failure path on the GPU, without a fault: with the test
hook on, the MMA warp waits on a barrier nothing arrives at, so every wait of
every CTA runs out after a short limit.  The call must return (no hang), the
device status word must read SK_ERR_DEVICE_TIMEOUT, and the context must stay
usable: the next normal call matches the oracle and leaves the status clean."""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sk():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from varlen_flash_attention_b200 import build

    build.build()
    import varlen_flash_attention_b200 as m

    return m


def test_wait_runs_out_and_context_survives(sk):
    w = workloads.get("tiny")
    t = workloads.make_inputs(w)
    d = {k: v.cuda() for k, v in t.items()}
    assert sk.sk_device_status(clear=True) == 0
    sk.sk_set_wait_timeout_ms(20)
    sk.sk_test_stall_mma(True)
    try:
        sk.attn_fwd_split_kv(d["q"], d["k_prefix"], d["v_prefix"], d["k_suffix"], d["v_suffix"])
        torch.cuda.synchronize()
        assert sk.sk_device_status(clear=True) == 4  # SK_ERR_DEVICE_TIMEOUT
    finally:
        sk.sk_test_stall_mma(False)
        sk.sk_set_wait_timeout_ms(2000)
    out = sk.attn_fwd_split_kv(d["q"], d["k_prefix"], d["v_prefix"], d["k_suffix"], d["v_suffix"])
    torch.cuda.synchronize()
    assert sk.sk_device_status() == 0
    ref = oracle.attn_split_kv(**t)
    assert float(np.abs(out.float().cpu().numpy() - ref).max()) <= 2e-2
