"""Parity of causal masking (flag ATTNQAT_CAUSAL on attnqat_fwd / attnqat_bwd,
through the C ABI) with the float64 oracle: full comparisons with ragged,
exact-multiple, single-tile and tiny lengths, both head dimensions and the
fp16 P V route with every quantizer on, and the flag sets with some quantizer
off (whose unquantized operands reach the MMAs as power-of-two-scaled fp16
copies).  The first keys' gradients gather every later row's contribution, so
they are heavy-tailed: these cases check that dS and the dV operand keep
enough precision.  Bar as for dense attention."""
import pytest

import oracle
from quantization_aware_attention_nvfp4_b200 import workloads as W
from tests.helpers import assert_close, run_attention, to_f64

pytestmark = pytest.mark.gpu


def _full_compare(w, flags):
    inp = W.inputs(w)
    got = run_attention(inp, w.sm_scale, flags | oracle.CAUSAL)
    ref = oracle.attention(inp["q"], inp["k"], inp["v"], w.sm_scale, flags | oracle.CAUSAL, inp["do"])
    assert_close("O", to_f64(got["o"]), ref["O"])
    assert_close("LSE", to_f64(got["lse"]), ref["lse"])
    assert_close("m", to_f64(got["m"]), ref["m"])
    assert_close("dQ", to_f64(got["dq"]), ref["dQ"])
    assert_close("dK", to_f64(got["dk"]), ref["dK"])
    assert_close("dV", to_f64(got["dv"]), ref["dV"])


@pytest.mark.parametrize("L,D,flags", [
    (1000, 128, oracle.QUANT_ALL),    # ragged last tile (104 rows and keys)
    (1024, 128, oracle.QUANT_ALL),    # whole tiles
    (1040, 128, oracle.QUANT_ALL),    # L % 32 == 16: the fp16 P V route
    (600, 64, oracle.QUANT_ALL),
    (128, 128, oracle.QUANT_ALL),     # the diagonal tile alone
    (7, 128, oracle.QUANT_ALL),
    (1, 64, oracle.QUANT_ALL),
    (500, 128, 0),                                    # no quantizer
    (500, 128, oracle.QUANT_Q | oracle.QUANT_K),
    (500, 128, oracle.QUANT_P),
    (500, 128, oracle.QUANT_V | oracle.QUANT_P),
    (1000, 64, oracle.QUANT_Q | oracle.QUANT_V),
    (1024, 128, oracle.QUANT_ALL & ~oracle.QUANT_P),
])
def test_causal_full(L, D, flags):
    w = W.custom(1, 2, L, L, D, seed_index=900 + L % 97 + D + flags)
    _full_compare(w, flags)
