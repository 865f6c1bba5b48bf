"""Property check of the oracle's block-sparse and causal masking over random
shapes, tile sizes (16, 32 and the tile-64 profile's 64) and selections
(hypothesis): every query tile's outputs equal dense attention against its
gathered key tiles, and with causal masking every row equals dense attention
against its key prefix (quantizers off there, so the prefix problem needs no
fq(V) of the whole V)."""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle
from quantization_aware_attention_nvfp4_b200 import workloads as W


def _bits(rng, shape):
    return W.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32))


@settings(max_examples=12, deadline=None)
@given(seed=st.integers(0, 2 ** 31 - 1), nq=st.integers(1, 3), nk=st.integers(1, 4),
       tile=st.sampled_from([16, 32, 64]), rq=st.integers(1, 16), rk=st.integers(1, 16),
       flags=st.sampled_from([oracle.QUANT_ALL, oracle.QUANT_Q | oracle.QUANT_K | oracle.QUANT_P, 0]))
def test_sparse_tile_outputs_equal_gathered_dense(seed, nq, nk, tile, rq, rk, flags):
    rng = np.random.default_rng(seed)
    Lq, Lk, D = (nq - 1) * tile + rq, (nk - 1) * tile + rk, 16
    q, k, v, dO = _bits(rng, (Lq, D)), _bits(rng, (Lk, D)), _bits(rng, (Lk, D)), _bits(rng, (Lq, D))
    sel = (rng.random((nq, nk)) < 0.6).astype(np.uint8)
    sp = oracle.Head(q, k, v, 0.25, flags, dO, sel=sel, tile=tile)
    st_sp = sp.stats()
    dQ, dK, dV = sp.backward()
    for I in range(nq):
        rows = np.arange(I * tile, min((I + 1) * tile, Lq))
        js = np.nonzero(sel[I])[0]
        if js.size == 0:
            assert np.all(st_sp["O"][rows] == 0) and np.all(np.isneginf(st_sp["lse"][rows]))
            continue
        keys = np.concatenate([np.arange(J * tile, min((J + 1) * tile, Lk)) for J in js])
        hd = oracle.Head(q[rows], k[keys], v[keys], 0.25, flags, dO[rows])
        ref = hd.stats()
        assert np.allclose(st_sp["O"][rows], ref["O"], rtol=0, atol=1e-12 * max(1.0, np.abs(ref["O"]).max()))
        assert np.allclose(dQ[rows], hd.dq_rows(), rtol=0, atol=1e-11 * max(1.0, np.abs(dQ[rows]).max()))


@settings(max_examples=10, deadline=None)
@given(seed=st.integers(0, 2 ** 31 - 1), L=st.integers(1, 40))
def test_causal_rows_equal_prefix_dense_quantizers_off(seed, L):
    rng = np.random.default_rng(seed)
    D = 16
    q, k, v = _bits(rng, (L, D)), _bits(rng, (L, D)), _bits(rng, (L, D))
    ca = oracle.Head(q, k, v, 0.3, oracle.CAUSAL).stats()
    for i in range(L):
        ref = oracle.Head(q[i:i + 1], k[: i + 1], v[: i + 1], 0.3, 0).stats()
        assert np.allclose(ca["O"][i], ref["O"][0], rtol=0, atol=1e-12 * max(1.0, np.abs(ref["O"]).max()))
        assert abs(ca["lse"][i] - ref["lse"][0]) <= 1e-12
