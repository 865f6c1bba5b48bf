"""The failure path of the library's bounded device waits, run on purpose
without a fault: a wait on an mbarrier that nothing arrives at gives up after
its limit, the other waiting role of the CTA leaves on the abort flag, the
copy in flight lands, the TMEM is freed, and attnqat_device_status() reports
ATTNQAT_ETIMEOUT once (then clears).  The context stays usable: an ordinary
forward and backward right after still match the oracle."""
import time

import pytest

import oracle
from quantization_aware_attention_nvfp4_b200 import workloads as W
from tests.helpers import assert_close, run_attention, to_f64

pytestmark = pytest.mark.gpu


def test_timed_out_wait_is_reported_and_the_context_stays_usable():
    import torch
    import quantization_aware_attention_nvfp4_b200 as A
    A.attnqat_device_status()  # starts clear
    t0 = time.perf_counter()
    ended = A.attnqat_selftest_wait_timeout(2_000_000)  # 2 ms
    dt = time.perf_counter() - t0
    assert ended == 2, "both waiting roles must leave their wait"
    assert dt < 1.0
    with pytest.raises(A.AttnQatError) as err:
        A.attnqat_device_status()
    assert err.value.status == A.ETIMEOUT
    assert A.attnqat_device_status() == A.OK  # reported once, then cleared

    w = W.get("tiny")
    inp = W.inputs(w)
    got = run_attention(inp, w.sm_scale, A.QUANT_ALL)
    ref = oracle.attention(inp["q"], inp["k"], inp["v"], w.sm_scale, oracle.QUANT_ALL, inp["do"])
    for name, key in (("O", "o"), ("dQ", "dq"), ("dK", "dk"), ("dV", "dv")):
        assert_close(name, to_f64(got[key]), ref[name])
    torch.cuda.synchronize()
